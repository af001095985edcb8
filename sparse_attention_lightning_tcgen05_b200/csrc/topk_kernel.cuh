// topk_kernel.cuh -- per-row top-k of the lightning-indexer scores.
//
// Per query row: the set of the index_topk valid slots with the largest
// scores, -1 padded when the row has fewer valid slots (DeepSeek-V3.2 Sparse
// Indexer Kernel API Reference: [n_tokens, index_topk] int32, an unordered
// set; NeMo AutoModel optimized_kernels: -1 masks an entry). Validity comes
// from positions / the causal rule, never from the values.
//
// One CTA per row. Each valid score becomes a monotone 32-bit key (larger
// score, larger key; -0 == +0). The row's keys are staged in shared memory
// with 16-byte loads when they fit (otherwise every pass streams the row
// from L2), and the same pass finds the row's smallest and largest key.
// Radix select then runs on u = key - kmin, most significant digit first,
// with digits placed from the top set bit of kmax - kmin: the 2048 bins of
// the first digit span the row's actual range, so few keys share a bin and
// the bin holding the k-th key is small. Its keys are compacted into shared
// memory and the remaining digits run on that list; once at most 32 remain,
// one warp finishes by rank counting. The output pass writes every slot
// whose key is above the threshold (warp-aggregated atomics, any order) and
// the slots equal to it: all of them, or the lowest indices when only some
// are taken (a deterministic set).
#pragma once

#include <cstdint>

#include "sm100_ptx.cuh"
#include "row_rule.cuh"

namespace dsa {

constexpr int kTopkBins = 2048;          // first-digit bins (11 bits)
constexpr int kTopkCand = 4096;          // compacted candidate keys

struct TopkParams {
  int mode;                 // kModePositions / kModeCausal
  int T;
  int64_t S;                // POSITIONS row length
  int num_seqs;
  const int *cu_seqlens;
  const int *positions;     // POSITIONS
  int compressed;           // POSITIONS rows that end by the compressed rule
  CompressedRule comp;
  const float *scores;
  int *topk;
  int k;
  int stage_cap;            // keys a CTA may stage in shared memory
  const unsigned int *cu_bad;   // CAUSAL: set by the cu_seqlens check -> no work
  unsigned int *err;        // device status word (first failure kept)
};

template <int NT>
struct TopkShared {
  uint32_t hist[kTopkBins];
  uint32_t cand[kTopkCand];
  uint32_t warp_a[NT / 32];
  uint32_t warp_b[NT / 32];
  uint32_t ncand;
  uint32_t sel_bin, sel_above;
  uint32_t kmin, kmax;
  uint32_t ckmin, ckmax;         // key range of the compacted candidates
  uint32_t tau, need, n_eq;      // threshold key, ties to take, ties in the row
  uint32_t out_gt, out_eq;       // output cursors of the unordered pass
  uint32_t tie_idx[32];          // slots of the ties (when at most 32)
  uint32_t small[32];            // the last <= 32 candidates
  uint32_t nsmall;
  int seq;
  long long seq_off;
  // followed by the staged keys (dynamic size)
};

// Order-preserving key: larger float -> larger unsigned key; -0 maps to +0.
__device__ __forceinline__ uint32_t score_key(float f) {
  uint32_t u = __float_as_uint(f);
  if (u == 0x80000000u) u = 0u;
  return (u & 0x80000000u) ? ~u : (u | 0x80000000u);
}

// Inclusive block-wide prefix sum of v; *total receives the block sum.
template <int NT, typename SM>
__device__ __forceinline__ uint32_t block_incl_scan(uint32_t v, SM &sm, uint32_t *total) {
  constexpr int kWarps = NT / 32;
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
#pragma unroll
  for (int off = 1; off < 32; off <<= 1) {
    const uint32_t n = __shfl_up_sync(0xffffffffu, v, off);
    if (lane >= off) v += n;
  }
  if (lane == 31) sm.warp_a[warp] = v;
  __syncthreads();
  if (warp == 0) {
    uint32_t x = lane < kWarps ? sm.warp_a[lane] : 0u;
#pragma unroll
    for (int off = 1; off < 32; off <<= 1) {
      const uint32_t n = __shfl_up_sync(0xffffffffu, x, off);
      if (lane >= off) x += n;
    }
    if (lane < kWarps) sm.warp_a[lane] = x;
  }
  __syncthreads();
  const uint32_t res = v + (warp > 0 ? sm.warp_a[warp - 1] : 0u);
  *total = sm.warp_a[kWarps - 1];
  __syncthreads();
  return res;
}

// Block-wide min and max of the keys each thread saw (into sm.kmin/kmax).
template <int NT, typename SM>
__device__ __forceinline__ void block_minmax(uint32_t lo, uint32_t hi, SM &sm) {
  constexpr int kWarps = NT / 32;
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
#pragma unroll
  for (int off = 16; off > 0; off >>= 1) {
    lo = min(lo, __shfl_xor_sync(0xffffffffu, lo, off));
    hi = max(hi, __shfl_xor_sync(0xffffffffu, hi, off));
  }
  if (lane == 0) {
    sm.warp_a[warp] = lo;
    sm.warp_b[warp] = hi;
  }
  __syncthreads();
  if (warp == 0) {
    lo = lane < kWarps ? sm.warp_a[lane] : 0xffffffffu;
    hi = lane < kWarps ? sm.warp_b[lane] : 0u;
#pragma unroll
    for (int off = 16; off > 0; off >>= 1) {
      lo = min(lo, __shfl_xor_sync(0xffffffffu, lo, off));
      hi = max(hi, __shfl_xor_sync(0xffffffffu, hi, off));
    }
    if (lane == 0) {
      sm.kmin = lo;
      sm.kmax = hi;
    }
  }
  __syncthreads();
}

// The bin b holding the need-th largest entry: sum(hist[b+1..]) < need <=
// sum(hist[b..]). Writes sm.sel_bin and sm.sel_above = sum(hist[b+1..]).
template <int NT, typename SM>
__device__ __forceinline__ void select_bin(SM &sm, const uint32_t *hist, uint32_t need,
                                           int nbins) {
  constexpr int kPer = (kTopkBins + NT - 1) / NT;
  const int b0 = threadIdx.x * kPer;
  uint32_t own = 0;
#pragma unroll
  for (int i = 0; i < kPer; ++i) own += (b0 + i < nbins) ? hist[b0 + i] : 0u;
  uint32_t total;
  const uint32_t incl = block_incl_scan<NT>(own, sm, &total);
  const uint32_t suffix_from_me = total - (incl - own);   // bins >= b0
  const uint32_t suffix_after_me = suffix_from_me - own;  // bins >= b0 + kPer
  if (own > 0 && suffix_after_me < need && need <= suffix_from_me) {
    uint32_t acc = suffix_after_me;
#pragma unroll
    for (int i = kPer - 1; i >= 0; --i) {
      const uint32_t h = (b0 + i < nbins) ? hist[b0 + i] : 0u;
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

// Entry s of the row: staged in shared memory or read from the row.
struct RowSrc {
  const float *row;
  const float *staged;      // nullptr: stream from global memory
  __device__ __forceinline__ float val(uint32_t s) const {
    return staged ? staged[s] : __ldg(row + s);
  }
  __device__ __forceinline__ uint32_t key(uint32_t s) const { return score_key(val(s)); }
};

// First-level bin of a score (see topk_kernel): monotone in v.
__device__ __forceinline__ int value_bin(float v, float vmin, float vscale) {
  return min(kTopkBins - 1, static_cast<int>((v - vmin) * vscale));
}

// Inverse of score_key.
__device__ __forceinline__ float key_value(uint32_t key) {
  return __uint_as_float((key & 0x80000000u) ? (key & 0x7fffffffu) : ~key);
}

// Row t's scores and its valid length: POSITIONS rows of S slots (valid up to
// the position, or the compressed rule's last pooled slot); CAUSAL rows of
// their sequence's L x L block (valid up to the diagonal). All threads of the
// block call it (CAUSAL synchronises).
template <int NT, typename SM>
__device__ __forceinline__ void topk_row_geometry(const TopkParams &p, int t, SM &sm,
                                                  const float *&row, int64_t &nvalid) {
  const int tid = threadIdx.x;
  if (p.mode == kModePositions) {
    row = p.scores + static_cast<int64_t>(t) * p.S;
    const int64_t pos = p.compressed ? compressed_last_slot(p.comp, t) : __ldg(p.positions + t);
    nvalid = pos < 0 ? 0 : (pos + 1 < p.S ? pos + 1 : p.S);
    return;
  }
  if (tid == 0) {            // largest i with cu[i] <= t (cu non-decreasing)
    int lo = 0, hi = p.num_seqs - 1;
    while (lo < hi) {
      const int mid = (lo + hi + 1) / 2;
      if (__ldg(p.cu_seqlens + mid) <= t) lo = mid; else hi = mid - 1;
    }
    sm.seq = lo;
    sm.seq_off = 0;
  }
  __syncthreads();
  const int i = sm.seq;
  // sum_{j < i} L_j^2: strided over threads, reduced per warp, then summed
  long long part = 0;
  for (int j = tid; j < i; j += NT) {
    const long long L = __ldg(p.cu_seqlens + j + 1) - __ldg(p.cu_seqlens + j);
    part += L * L;
  }
#pragma unroll
  for (int off = 16; off > 0; off >>= 1) part += __shfl_xor_sync(0xffffffffu, part, off);
  if ((tid & 31) == 0 && part)
    atomicAdd(reinterpret_cast<unsigned long long *>(&sm.seq_off),
              static_cast<unsigned long long>(part));
  __syncthreads();
  const int a = __ldg(p.cu_seqlens + i);
  const int64_t L = __ldg(p.cu_seqlens + i + 1) - a;
  row = p.scores + sm.seq_off + static_cast<int64_t>(t - a) * L;
  nvalid = t - a + 1;
}

// Stage the row's values [0, n) in shared memory (if keys != nullptr) and
// find the smallest and largest key. Vector loads on the 16-byte aligned body.
template <int NT>
__device__ void stage_row(const float *row, uint32_t n, float *keys, TopkShared<NT> &sm) {
  uint32_t lo = 0xffffffffu, hi = 0u;
  const uint32_t head =
      min(n, static_cast<uint32_t>((16u - (reinterpret_cast<uintptr_t>(row) & 15u)) & 15u) / 4u);
  for (uint32_t s = threadIdx.x; s < head; s += NT) {
    const float v = __ldg(row + s);
    const uint32_t kk = score_key(v);
    if (keys) keys[s] = v;
    lo = min(lo, kk);
    hi = max(hi, kk);
  }
  const uint32_t nvec = (n - head) / 4;
  const float4 *v4 = reinterpret_cast<const float4 *>(row + head);
#pragma unroll 4
  for (uint32_t i = threadIdx.x; i < nvec; i += NT) {
    const float4 v = __ldg(v4 + i);
    const uint32_t k0 = score_key(v.x), k1 = score_key(v.y), k2 = score_key(v.z),
                   k3 = score_key(v.w);
    if (keys) {
      const uint32_t s = head + 4 * i;
      keys[s] = v.x;
      keys[s + 1] = v.y;
      keys[s + 2] = v.z;
      keys[s + 3] = v.w;
    }
    lo = min(min(lo, min(k0, k1)), min(k2, k3));
    hi = max(max(hi, max(k0, k1)), max(k2, k3));
  }
  for (uint32_t s = head + 4 * nvec + threadIdx.x; s < n; s += NT) {
    const float v = __ldg(row + s);
    const uint32_t kk = score_key(v);
    if (keys) keys[s] = v;
    lo = min(lo, kk);
    hi = max(hi, kk);
  }
  block_minmax<NT>(lo, hi, sm);
}

// The selection of one row of n > k valid scores into out[0, k): the whole
// block, smem `sm` and a stage of p.stage_cap floats. Every thread returns.
template <int NT>
__device__ void topk_row_full(const TopkParams &p, TopkShared<NT> &sm, float *staged_keys,
                              const float *row, uint32_t n, int *out) {
  const int tid = threadIdx.x;
  const uint32_t k = static_cast<uint32_t>(p.k);
  const bool staged = n <= static_cast<uint32_t>(p.stage_cap);

  // ---- stage (or scan) the row: keys and their range ----
  stage_row<NT>(row, n, staged ? staged_keys : nullptr, sm);
  const RowSrc src{row, staged ? staged_keys : nullptr};
  uint32_t kmin = sm.kmin;
  uint32_t range = sm.kmax - kmin;
  uint32_t need = k;
  bool in_cand = false;
  uint32_t n_match = n;    // entries that can still hold the threshold

  // ---- first level: bins linear in the score value ----
  // bin(v) = min(2047, (v - vmin) * 2048 / (vmax - vmin)) is monotone in v
  // under fp32 rounding, so it is a valid selection digit; unlike the
  // exponent-dominated bits of a key it spreads the scores evenly, so the
  // bin holding the k-th score is small and the histogram atomics rarely
  // collide.
  const float vmin = key_value(kmin), vmax = key_value(sm.kmax);
  const float vscale = 2048.f / (vmax - vmin);
  if (range != 0 && isfinite(vscale) && vscale > 0.f) {
    for (int b = tid; b < kTopkBins; b += NT) sm.hist[b] = 0;
    if (tid == 0) { sm.ncand = 0; sm.ckmin = 0xffffffffu; sm.ckmax = 0u; }
    __syncthreads();
#pragma unroll 4
    for (uint32_t s = tid; s < n; s += NT) {
      atomicAdd(&sm.hist[value_bin(src.val(s), vmin, vscale)], 1u);
    }
    __syncthreads();
    select_bin<NT>(sm, sm.hist, need, kTopkBins);
    const int b1 = static_cast<int>(sm.sel_bin);
    need -= sm.sel_above;
    n_match = sm.hist[b1];
    if (n_match <= static_cast<uint32_t>(kTopkCand)) {
      for (uint32_t s = tid; s < n; s += NT) {
        const float v = src.val(s);
        if (value_bin(v, vmin, vscale) == b1) {
          const uint32_t key = score_key(v);
          sm.cand[atomicAdd(&sm.ncand, 1u)] = key;
          atomicMin(&sm.ckmin, key);
          atomicMax(&sm.ckmax, key);
        }
      }
      __syncthreads();
      in_cand = true;
      kmin = sm.ckmin;                 // the key digits below work on the bin
      range = sm.ckmax - kmin;
    } else {
      need = k;                        // too many: digits over the whole row
      n_match = n;
      __syncthreads();
    }
  }
  const int bits = range == 0 ? 0 : 32 - __clz(range);   // significant bits of u

  // ---- radix select on u = key - kmin ----
  // Digits from the top: [bits-11, bits), then 11 bits at a time down to 0.
  // Once the keys that share the resolved prefix are compacted into shared
  // memory and number at most 32, one warp finishes by rank counting.
  uint32_t prefix = 0;     // resolved high part of u, right-aligned
  int lo_bit = bits;       // surviving keys have u >> lo_bit == prefix
  if (!in_cand && tid == 0) sm.ncand = 0;
#pragma unroll 1
  while (lo_bit > 0) {
    if (in_cand && n_match <= 32) break;
    const int dbits = lo_bit >= 11 ? 11 : lo_bit;
    const int shift = lo_bit - dbits;
    const uint32_t dmask = (1u << dbits) - 1u;
    for (int b = tid; b < kTopkBins; b += NT) sm.hist[b] = 0;
    __syncthreads();
    if (in_cand) {
      const uint32_t nc = sm.ncand;
      for (uint32_t i = tid; i < nc; i += NT) {
        const uint32_t u = sm.cand[i] - kmin;
        if ((u >> lo_bit) == prefix) atomicAdd(&sm.hist[(u >> shift) & dmask], 1u);
      }
    } else {
#pragma unroll 4
      for (uint32_t s = tid; s < n; s += NT) {
        const uint32_t u = src.key(s) - kmin;
        if (lo_bit >= 32 || (u >> lo_bit) == prefix)
          atomicAdd(&sm.hist[(u >> shift) & dmask], 1u);
      }
    }
    __syncthreads();
    select_bin<NT>(sm, sm.hist, need, 1 << dbits);
    const uint32_t b = sm.sel_bin;
    need -= sm.sel_above;
    prefix = (lo_bit >= 32 ? 0u : (prefix << dbits)) | b;
    lo_bit = shift;
    n_match = sm.hist[b];
    __syncthreads();
    if (!in_cand && lo_bit > 0 && n_match <= kTopkCand) {
      for (uint32_t s = tid; s < n; s += NT) {
        const uint32_t key = src.key(s);
        if (((key - kmin) >> lo_bit) == prefix) sm.cand[atomicAdd(&sm.ncand, 1u)] = key;
      }
      __syncthreads();
      in_cand = true;
    }
  }
  if (lo_bit > 0) {
    // <= 32 candidates share the prefix: the need-th largest of them, by
    // counting for each candidate the ones above it. The block collects them
    // (the list may still hold keys compacted under a shorter prefix), then
    // one warp ranks them.
    if (tid == 0) sm.nsmall = 0;
    __syncthreads();
    const uint32_t nc = sm.ncand;
    for (uint32_t i = tid; i < nc; i += NT) {
      const uint32_t key = sm.cand[i];
      if (((key - kmin) >> lo_bit) == prefix) {
        const uint32_t slot = atomicAdd(&sm.nsmall, 1u);
        if (slot < 32) sm.small[slot] = key;
      }
    }
    __syncthreads();
    if (tid < 32) {
      const uint32_t live_n = min(sm.nsmall, 32u);
      const bool live = static_cast<uint32_t>(tid) < live_n;
      const uint32_t mine = live ? sm.small[tid] : 0u;
      uint32_t above = 0, equal = 0;
      for (uint32_t l = 0; l < live_n; ++l) {
        const uint32_t other = sm.small[l];
        above += other > mine;
        equal += other == mine;
      }
      const bool is_tau = live && above < need && need <= above + equal;
      const unsigned who = __ballot_sync(0xffffffffu, is_tau);
      if (tid == __ffs(who) - 1) {
        sm.tau = mine;
        sm.need = need - above;
        sm.n_eq = equal;
      }
    }
    __syncthreads();
  } else {
    if (tid == 0) {
      sm.tau = kmin + prefix;
      sm.need = need;
      sm.n_eq = n_match;
    }
    __syncthreads();
  }
  const uint32_t tau = sm.tau;       // the k-th largest key
  need = sm.need;                    // ties at tau to take (>= 1)
  const uint32_t n_eq = sm.n_eq;     // ties at tau in the row

  if (need == n_eq || n_eq <= 32) {
    // ---- unordered output: every key > tau, and the ties ----
    // All ties are taken, or they are few enough to order in one warp.
    if (tid == 0) { sm.out_gt = 0; sm.out_eq = 0; }
    __syncthreads();
    const uint32_t n_gt = k - need;          // keys above tau
    const int lane = tid & 31;
    for (uint32_t c0 = 0; c0 < n; c0 += NT) {
      const uint32_t s = c0 + tid;
      const uint32_t key = s < n ? src.key(s) : 0u;
      const bool gt = s < n && key > tau;
      const bool eq = s < n && key == tau;
      const unsigned mgt = __ballot_sync(0xffffffffu, gt);
      if (mgt) {
        uint32_t base = 0;
        if (lane == 0) base = atomicAdd(&sm.out_gt, __popc(mgt));
        base = __shfl_sync(0xffffffffu, base, 0);
        const uint32_t o = base + __popc(mgt & ((1u << lane) - 1u));
        if (gt && o < k) out[o] = static_cast<int>(s);
      }
      const unsigned meq = __ballot_sync(0xffffffffu, eq);
      if (meq) {
        uint32_t base = 0;
        if (lane == 0) base = atomicAdd(&sm.out_eq, __popc(meq));
        base = __shfl_sync(0xffffffffu, base, 0);
        const uint32_t r = base + __popc(meq & ((1u << lane) - 1u));
        if (eq) {
          if (need == n_eq) {
            if (n_gt + r < k) out[n_gt + r] = static_cast<int>(s);
          }
          else if (r < 32) sm.tie_idx[r] = static_cast<uint32_t>(s);
        }
      }
    }
    if (need != n_eq) {
      __syncthreads();
      if (tid < 32) {            // the `need` lowest slots among <= 32 ties
        const uint32_t mine = tid < static_cast<int>(n_eq) ? sm.tie_idx[tid] : 0xffffffffu;
        uint32_t below = 0;
        for (int l = 0; l < 32; ++l) below += __shfl_sync(0xffffffffu, mine, l) < mine;
        if (tid < static_cast<int>(n_eq) && below < need && n_gt + below < k)
          out[n_gt + below] = static_cast<int>(mine);
      }
    }
    return;
  }

  // ---- ordered output (many ties, only some taken): keys > tau, then the
  // first `need` keys == tau in slot order ----
  uint32_t base_gt = 0, base_eq = 0;
  for (uint32_t c0 = 0; c0 < n; c0 += 4 * NT) {
    uint32_t gt = 0, eq = 0;          // bit i: entry c0 + 4*tid + i
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      const uint32_t s = c0 + 4 * tid + i;
      if (s < n) {
        const uint32_t key = src.key(s);
        gt |= static_cast<uint32_t>(key > tau) << i;
        eq |= static_cast<uint32_t>(key == tau) << i;
      }
    }
    const uint32_t own = (__popc(gt) << 16) | __popc(eq);
    uint32_t total;
    const uint32_t excl = block_incl_scan<NT>(own, sm, &total) - own;
    const uint32_t E0 = base_eq + (excl & 0xFFFFu);
    uint32_t E = E0;
    uint32_t pos = base_gt + (excl >> 16) + min(E0, need);
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

template <int NT>
__global__ void __launch_bounds__(NT) topk_kernel(const TopkParams p) {
  extern __shared__ uint8_t smem_raw[];
  TopkShared<NT> &sm = *reinterpret_cast<TopkShared<NT> *>(smem_raw);
  float *staged_keys = reinterpret_cast<float *>(smem_raw + sizeof(TopkShared<NT>));
  const int t = blockIdx.x;
  const int tid = threadIdx.x;
  // scores (and positions) come from earlier work on the stream
  grid_dep_wait();
  grid_dep_launch_dependents();
  // CAUSAL: a cu_seqlens array that failed its check -> write nothing
  if (p.mode == kModeCausal && *p.cu_bad) return;

  const float *row;
  int64_t nvalid;
  topk_row_geometry<NT>(p, t, sm, row, nvalid);
  int *out = p.topk + static_cast<int64_t>(t) * p.k;
  const uint32_t k = static_cast<uint32_t>(p.k);

  if (nvalid <= static_cast<int64_t>(k)) {
    for (uint32_t i = tid; i < k; i += NT) out[i] = i < nvalid ? static_cast<int>(i) : -1;
    return;
  }
  topk_row_full<NT>(p, sm, staged_keys, row, static_cast<uint32_t>(nvalid), out);
}

}  // namespace dsa
