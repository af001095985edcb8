// topk_kernel.cuh -- per-row top-k of the lightning-indexer scores.
//
// Per query row: the set of the index_topk valid slots with the largest
// scores, -1 padded when the row has fewer valid slots (DeepSeek-V3.2 Sparse
// Indexer Kernel API Reference: [n_tokens, index_topk] int32, an unordered
// set; NeMo AutoModel optimized_kernels: -1 masks an entry). Validity comes
// from positions / the causal rule, never from the values.
//
// Radix select on a monotone 32-bit key of each fp32 score, most significant
// digit first (11, 11, 10 bits), with the digit histogram in shared memory.
// Once the bin that holds the k-th key is small enough, its keys are copied
// into shared memory and the remaining digits run there. A final ordered pass
// writes every slot whose key is above the threshold and, among slots equal
// to it, the lowest indices (so the set is deterministic), in slot order.
#pragma once

#include <cstdint>

namespace dsa {

constexpr int kTopkThreads = 512;
constexpr int kTopkWarps = kTopkThreads / 32;
constexpr int kTopkBins = 2048;
constexpr int kTopkCap = 16384;        // candidate keys kept in shared memory

struct TopkParams {
  int mode;                 // kModePositions / kModeCausal
  int T;
  int64_t S;                // POSITIONS row length
  int num_seqs;
  const int *cu_seqlens;
  const int *positions;
  const float *scores;
  int *topk;
  int k;
};

struct TopkSmem {
  uint32_t hist[kTopkBins];
  uint32_t cand[kTopkCap];
  uint32_t warp_sums[kTopkWarps];
  uint32_t ncand;
  uint32_t sel_bin, sel_above;
  int seq;
  long long seq_off;
};

// Order-preserving key: larger float -> larger unsigned key; -0 maps to +0.
__device__ __forceinline__ uint32_t score_key(float f) {
  uint32_t u = __float_as_uint(f);
  if (u == 0x80000000u) u = 0u;
  return (u & 0x80000000u) ? ~u : (u | 0x80000000u);
}

// Inclusive block-wide prefix sum of v; *total receives the block sum.
__device__ __forceinline__ uint32_t block_incl_scan(uint32_t v, TopkSmem &sm,
                                                    uint32_t *total) {
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
#pragma unroll
  for (int off = 1; off < 32; off <<= 1) {
    const uint32_t n = __shfl_up_sync(0xffffffffu, v, off);
    if (lane >= off) v += n;
  }
  if (lane == 31) sm.warp_sums[warp] = v;
  __syncthreads();
  if (warp == 0) {
    uint32_t x = lane < kTopkWarps ? sm.warp_sums[lane] : 0u;
#pragma unroll
    for (int off = 1; off < 32; off <<= 1) {
      const uint32_t n = __shfl_up_sync(0xffffffffu, x, off);
      if (lane >= off) x += n;
    }
    if (lane < kTopkWarps) sm.warp_sums[lane] = x;
  }
  __syncthreads();
  const uint32_t res = v + (warp > 0 ? sm.warp_sums[warp - 1] : 0u);
  *total = sm.warp_sums[kTopkWarps - 1];
  __syncthreads();
  return res;
}

// Find the bin b holding the need-th largest key: sum(hist[b+1..]) < need <=
// sum(hist[b..]). Writes sm.sel_bin and sm.sel_above = sum(hist[b+1..]).
__device__ __forceinline__ void select_bin(TopkSmem &sm, uint32_t need,
                                           int nbins) {
  constexpr int kPer = kTopkBins / kTopkThreads;          // 4 bins a thread
  const int b0 = threadIdx.x * kPer;
  uint32_t own = 0;
#pragma unroll
  for (int i = 0; i < kPer; ++i) own += (b0 + i < nbins) ? sm.hist[b0 + i] : 0u;
  uint32_t total;
  const uint32_t incl = block_incl_scan(own, sm, &total);
  const uint32_t suffix_from_me = total - (incl - own);   // bins >= b0
  const uint32_t suffix_after_me = suffix_from_me - own;  // bins >= b0 + kPer
  if (suffix_after_me < need && need <= suffix_from_me) {
    uint32_t acc = suffix_after_me;
#pragma unroll
    for (int i = kPer - 1; i >= 0; --i) {
      const uint32_t h = (b0 + i < nbins) ? sm.hist[b0 + i] : 0u;
      if (acc + h >= need) {
        sm.sel_bin = b0 + i;
        sm.sel_above = acc;
        break;
      }
      acc += h;
    }
  }
  __syncthreads();
}

__global__ void __launch_bounds__(kTopkThreads)
    topk_kernel(const TopkParams p) {
  extern __shared__ uint8_t smem_raw[];
  TopkSmem &sm = *reinterpret_cast<TopkSmem *>(smem_raw);
  const int t = blockIdx.x;
  const int tid = threadIdx.x;

  // ---- row geometry ----
  const float *row;
  int64_t nvalid;
  if (p.mode == kModePositions) {
    row = p.scores + static_cast<int64_t>(t) * p.S;
    const int pos = __ldg(p.positions + t);
    nvalid = pos < 0 ? 0 : (static_cast<int64_t>(pos) + 1 < p.S ? pos + 1 : p.S);
  } else {
    if (tid == 0) {            // largest i with cu[i] <= t (cu non-decreasing)
      int lo = 0, hi = p.num_seqs - 1;
      while (lo < hi) {
        const int mid = (lo + hi + 1) / 2;
        if (__ldg(p.cu_seqlens + mid) <= t) lo = mid; else hi = mid - 1;
      }
      sm.seq = lo;
    }
    __syncthreads();
    const int i = sm.seq;
    // sum_{j < i} L_j^2: strided over threads, reduced per warp, then summed
    // into shared memory
    long long part = 0;
    for (int j = tid; j < i; j += kTopkThreads) {
      const long long L = __ldg(p.cu_seqlens + j + 1) - __ldg(p.cu_seqlens + j);
      part += L * L;
    }
#pragma unroll
    for (int off = 16; off > 0; off >>= 1) part += __shfl_xor_sync(0xffffffffu, part, off);
    if (tid == 0) sm.seq_off = 0;
    __syncthreads();
    if ((tid & 31) == 0 && part)
      atomicAdd(reinterpret_cast<unsigned long long *>(&sm.seq_off),
                static_cast<unsigned long long>(part));
    __syncthreads();
    const int a = __ldg(p.cu_seqlens + i);
    const int64_t L = __ldg(p.cu_seqlens + i + 1) - a;
    row = p.scores + sm.seq_off + static_cast<int64_t>(t - a) * L;
    nvalid = t - a + 1;
  }
  int *out = p.topk + static_cast<int64_t>(t) * p.k;
  const uint32_t k = static_cast<uint32_t>(p.k);

  if (nvalid <= static_cast<int64_t>(k)) {
    for (uint32_t i = tid; i < k; i += kTopkThreads)
      out[i] = i < nvalid ? static_cast<int>(i) : -1;
    return;
  }
  const uint32_t n = static_cast<uint32_t>(nvalid);

  // ---- radix select of the threshold key ----
  uint32_t prefix = 0, pmask = 0, need = k;
  bool in_smem = false;
  if (tid == 0) sm.ncand = 0;
  constexpr int kShift[3] = {21, 10, 0};
  constexpr int kBits[3] = {11, 11, 10};
#pragma unroll 1
  for (int d = 0; d < 3; ++d) {
    const int shift = kShift[d];
    const uint32_t dmask = (1u << kBits[d]) - 1u;
    for (int b = tid; b < kTopkBins; b += kTopkThreads) sm.hist[b] = 0;
    __syncthreads();
    if (!in_smem) {
      for (uint32_t s = tid; s < n; s += kTopkThreads) {
        const uint32_t key = score_key(__ldg(row + s));
        if ((key & pmask) == prefix) atomicAdd(&sm.hist[(key >> shift) & dmask], 1u);
      }
    } else {
      const uint32_t nc = sm.ncand;
      for (uint32_t i = tid; i < nc; i += kTopkThreads) {
        const uint32_t key = sm.cand[i];
        if ((key & pmask) == prefix) atomicAdd(&sm.hist[(key >> shift) & dmask], 1u);
      }
    }
    __syncthreads();
    select_bin(sm, need, 1 << kBits[d]);
    const uint32_t b = sm.sel_bin;
    need -= sm.sel_above;
    prefix |= b << shift;
    pmask |= dmask << shift;
    const uint32_t remaining = sm.hist[b];
    __syncthreads();
    if (!in_smem && d < 2 && remaining <= kTopkCap) {
      for (uint32_t s = tid; s < n; s += kTopkThreads) {
        const uint32_t key = score_key(__ldg(row + s));
        if ((key & pmask) == prefix) sm.cand[atomicAdd(&sm.ncand, 1u)] = key;
      }
      __syncthreads();
      in_smem = true;
    }
  }
  const uint32_t tau = prefix;

  // ---- ordered output: keys > tau, then the first `need` keys == tau ----
  uint32_t base_gt = 0, base_eq = 0;
  for (uint32_t c0 = 0; c0 < n; c0 += 4 * kTopkThreads) {
    uint32_t gt = 0, eq = 0;          // bit i: element c0 + 4*tid + i
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      const uint32_t s = c0 + 4 * tid + i;
      if (s < n) {
        const uint32_t key = score_key(__ldg(row + s));
        gt |= static_cast<uint32_t>(key > tau) << i;
        eq |= static_cast<uint32_t>(key == tau) << i;
      }
    }
    const uint32_t own = (__popc(gt) << 16) | __popc(eq);
    uint32_t total;
    const uint32_t excl = block_incl_scan(own, sm, &total) - own;
    uint32_t G = base_gt + (excl >> 16);
    uint32_t E = base_eq + (excl & 0xFFFFu);
    uint32_t pos = G + min(E, need);
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      const uint32_t s = c0 + 4 * tid + i;
      if (gt >> i & 1u) {
        if (pos < k) out[pos] = static_cast<int>(s);
        ++pos;
      } else if (eq >> i & 1u) {
        if (E < need) {
          if (pos < k) out[pos] = static_cast<int>(s);
          ++pos;
        }
        ++E;
      }
    }
    base_gt += total >> 16;
    base_eq += total & 0xFFFFu;
  }
}

}  // namespace dsa
