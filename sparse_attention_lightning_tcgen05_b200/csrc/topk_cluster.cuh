// topk_cluster.cuh -- top-k of decode score rows: one thread-block cluster of
// C CTAs (C <= 8) per row.
//
// Same result as topk_kernel (DeepSeek-V3.2 Sparse Indexer Kernel API
// Reference: [n_tokens, index_topk] int32, an unordered set; ties at the k-th
// score go to the lower slot), for rows that are few and long: a decode batch
// has one row per sequence, so one CTA per row would leave most SMs idle.
// Rank r of the cluster stages the r-th 1/C of the row's valid slots as
// monotone keys in its shared memory. The ranks then agree on the threshold
// through distributed shared memory (DSMEM), with few cluster barriers (each
// costs about as much as a few hundred cycles of work):
//   1. every rank publishes its key range and reads all of them (barrier A);
//   2. while the candidates are too many to gather, a histogram round: every
//      rank counts its candidates in 256 bins (the first round linear in the
//      score value over the row's range, later rounds 8-bit key digits),
//      then copies every rank's histogram (barrier per round), so every rank
//      selects the same bin and knows, per rank, how many keys lie above it
//      and in it;
//   3. every rank writes its candidates into every rank's list at offsets
//      known from those counts (barrier C), and each rank resolves the exact
//      threshold key tau, and how many keys equal to it are taken, from the
//      same list;
//   4. the per-rank counts above and at tau give every rank its output
//      offsets without a further exchange: keys above tau are written in any
//      order, ties in slot order when only some are taken.
// All branches around a cluster barrier depend only on values every rank
// computes identically, so every CTA reaches every barrier; no CTA exits
// while another may still read its shared memory.
#pragma once

#include <cstdint>

#include "sm100_ptx.cuh"
#include "topk_kernel.cuh"

namespace dsa {

constexpr int kClusterMaxRanks = 8;    // portable cluster size
constexpr int kClusterBins = 256;      // bins of a histogram round
constexpr int kClusterCand = 1024;     // candidates every rank gathers

template <int NT>
struct ClusterTopkShared {
  alignas(16) uint32_t hist[2][kClusterBins];                 // this CTA's (hist[0] reused)
  // every rank's histogram of the round, pushed here by its owner before the
  // round's barrier; by round parity, so that a rank already pushing the
  // next round never overwrites one still being read
  alignas(16) uint32_t part[2][kClusterMaxRanks][kClusterBins];
  uint32_t rk_min[kClusterMaxRanks], rk_max[kClusterMaxRanks];  // pushed key ranges
  uint32_t ghist[kClusterBins];                               // their sum
  uint32_t cand[kClusterCand];          // the candidates of all ranks, rank by rank
  uint32_t gt_above[kClusterMaxRanks];  // per rank: keys above the selected bins
  uint32_t cnt_sel[kClusterMaxRanks];   // per rank: keys in the selected bin
  uint32_t cnt_gt[kClusterMaxRanks];    // per rank: keys above tau
  uint32_t cnt_eq[kClusterMaxRanks];    // per rank: keys equal to tau
  uint32_t warp_a[NT / 32], warp_b[NT / 32];
  uint32_t kmin, kmax;                  // block_minmax result
  uint32_t gkmin, gkmax;                // the row's key range
  uint32_t sel_bin, sel_above;
  uint32_t tau, need_eq;
  uint32_t cursor, nsmall;
  uint32_t out_gt, out_eq;              // output cursors
  uint32_t small[32];
};

// Key i of this CTA's chunk: staged in shared memory or read from the row.
struct ChunkKeys {
  const float *src;
  const uint32_t *staged;
  __device__ __forceinline__ uint32_t operator()(uint32_t i) const {
    return staged ? staged[i] : score_key(__ldg(src + i));
  }
};

// Stage src[0, n) as keys (when keys != nullptr) and find their range
// (sm.kmin, sm.kmax). 16-byte loads on the aligned body.
template <int NT, typename SM>
__device__ void stage_keys(const float *src, uint32_t n, uint32_t *keys, SM &sm) {
  uint32_t lo = 0xffffffffu, hi = 0u;
  const uint32_t head =
      min(n, static_cast<uint32_t>((16u - (reinterpret_cast<uintptr_t>(src) & 15u)) & 15u) / 4u);
  for (uint32_t s = threadIdx.x; s < head; s += NT) {
    const uint32_t kk = score_key(__ldg(src + s));
    if (keys) keys[s] = kk;
    lo = min(lo, kk);
    hi = max(hi, kk);
  }
  const uint32_t nvec = (n - head) / 4;
  const float4 *v4 = reinterpret_cast<const float4 *>(src + head);
#pragma unroll 4
  for (uint32_t i = threadIdx.x; i < nvec; i += NT) {
    const float4 v = __ldg(v4 + i);
    const uint32_t k0 = score_key(v.x), k1 = score_key(v.y), k2 = score_key(v.z),
                   k3 = score_key(v.w);
    if (keys) {
      const uint32_t s = head + 4 * i;
      keys[s] = k0;
      keys[s + 1] = k1;
      keys[s + 2] = k2;
      keys[s + 3] = k3;
    }
    lo = min(min(lo, min(k0, k1)), min(k2, k3));
    hi = max(max(hi, max(k0, k1)), max(k2, k3));
  }
  for (uint32_t s = head + 4 * nvec + threadIdx.x; s < n; s += NT) {
    const uint32_t kk = score_key(__ldg(src + s));
    if (keys) keys[s] = kk;
    lo = min(lo, kk);
    hi = max(hi, kk);
  }
  block_minmax<NT>(lo, hi, sm);
}

// Among the m candidate keys sm.cand[0, m): the need-th largest (sm.tau)
// and how many keys equal to it are taken (sm.need_eq = need minus the keys
// above it). 8-bit digits from the top of the candidates' range until at
// most 32 share the resolved prefix; one warp then ranks those. Whole CTA.
template <int NT, typename SM>
__device__ void cand_select(SM &sm, uint32_t m, uint32_t need) {
  const int tid = threadIdx.x;
  uint32_t lo = 0xffffffffu, hi = 0u;
  for (uint32_t i = tid; i < m; i += NT) {
    lo = min(lo, sm.cand[i]);
    hi = max(hi, sm.cand[i]);
  }
  block_minmax<NT>(lo, hi, sm);
  const uint32_t cmin = sm.kmin, crange = sm.kmax - sm.kmin;
  int lo_bit = crange == 0 ? 0 : 32 - __clz(crange);
  uint32_t prefix = 0, nmatch = m;
#pragma unroll 1
  while (lo_bit > 0 && nmatch > 32) {
    const int dbits = lo_bit >= 8 ? 8 : lo_bit;
    const int shift = lo_bit - dbits;
    const uint32_t dmask = (1u << dbits) - 1u;
    for (int b = tid; b < kClusterBins; b += NT) sm.hist[0][b] = 0;
    __syncthreads();
    for (uint32_t i = tid; i < m; i += NT) {
      const uint32_t u = sm.cand[i] - cmin;
      if (lo_bit >= 32 || (u >> lo_bit) == prefix) atomicAdd(&sm.hist[0][(u >> shift) & dmask], 1u);
    }
    __syncthreads();
    select_bin<NT>(sm, sm.hist[0], need, 1 << dbits);
    const uint32_t bin = sm.sel_bin;
    need -= sm.sel_above;
    nmatch = sm.hist[0][bin];
    prefix = (lo_bit >= 32 ? 0u : (prefix << dbits)) | bin;
    lo_bit = shift;
    __syncthreads();
  }
  if (lo_bit == 0) {
    if (tid == 0) {
      sm.tau = cmin + prefix;
      sm.need_eq = need;
    }
    __syncthreads();
    return;
  }
  // at most 32 keys share the prefix: collect them, then one warp ranks them
  if (tid == 0) sm.nsmall = 0;
  __syncthreads();
  for (uint32_t i = tid; i < m; i += NT) {
    const uint32_t key = sm.cand[i];
    if (lo_bit >= 32 || ((key - cmin) >> lo_bit) == prefix) {
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
      sm.need_eq = need - above;
    }
  }
  __syncthreads();
}

// First-round bin of a key: linear in its score value over [vmin, vmax].
__device__ __forceinline__ int cluster_value_bin(uint32_t key, float vmin, float vscale) {
  return min(kClusterBins - 1, static_cast<int>((key_value(key) - vmin) * vscale));
}

template <int NT>
__global__ void __launch_bounds__(NT) topk_cluster_kernel(const TopkParams p) {
  static_assert(NT >= 64 * kClusterMaxRanks && NT / 32 >= kClusterMaxRanks, "threads");
  extern __shared__ __align__(16) uint8_t smem_raw[];
  ClusterTopkShared<NT> &sm = *reinterpret_cast<ClusterTopkShared<NT> *>(smem_raw);
  uint32_t *staged_keys = reinterpret_cast<uint32_t *>(smem_raw + sizeof(ClusterTopkShared<NT>));
  const uint32_t C = cluster_size(), r = cluster_rank();
  const int t = static_cast<int>(blockIdx.x / C);
  const int tid = threadIdx.x;
  const int lane = tid & 31, warp = tid >> 5;
  // scores and positions come from earlier work on the stream
  grid_dep_wait();
  grid_dep_launch_dependents();

  const float *row = p.scores + static_cast<int64_t>(t) * p.S;
  const int64_t pos = p.compressed ? compressed_last_slot(p.comp, t) : __ldg(p.positions + t);
  const int64_t nvalid = pos < 0 ? 0 : (pos + 1 < p.S ? pos + 1 : p.S);
  int *out = p.topk + static_cast<int64_t>(t) * p.k;
  const uint32_t k = static_cast<uint32_t>(p.k);
  if (nvalid <= static_cast<int64_t>(k)) {   // the same in every rank
    if (r == 0)
      for (uint32_t i = tid; i < k; i += NT) out[i] = i < nvalid ? static_cast<int>(i) : -1;
    return;
  }
  const uint32_t n = static_cast<uint32_t>(nvalid);
  const uint32_t chunk = (n + C - 1) / C;
  const uint32_t lo = min(n, r * chunk);
  const uint32_t m = min(n, lo + chunk) - lo;
  const bool staged = chunk <= static_cast<uint32_t>(p.stage_cap);   // the same in every rank
  const ChunkKeys key{row + lo, staged ? staged_keys : nullptr};
  if (static_cast<uint32_t>(tid) < C) {   // each rank's share, until a round counts it
    const uint32_t l = min(n, tid * chunk);
    sm.cnt_sel[tid] = min(n, l + chunk) - l;
    sm.gt_above[tid] = 0;
  }
  if (tid == 0) {
    sm.cursor = 0;
    sm.out_gt = 0;
    sm.out_eq = 0;
  }

  // ---- 1. stage the chunk; the row's key range (barrier A) ----
  // Exchanges push: each rank stores its data into every rank's shared
  // memory before the barrier (the barrier's release/acquire makes it
  // visible), so nothing waits on a remote load after it.
  stage_keys<NT>(row + lo, m, staged ? staged_keys : nullptr, sm);
  if (static_cast<uint32_t>(tid) < C) {
    dsmem_st(dsmem_addr(smem_u32(&sm.rk_min[r]), tid), sm.kmin);
    dsmem_st(dsmem_addr(smem_u32(&sm.rk_max[r]), tid), sm.kmax);
  }
  cluster_sync();
  if (tid < 32) {
    uint32_t a = 0xffffffffu, b = 0u;
    if (static_cast<uint32_t>(lane) < C) {
      a = sm.rk_min[lane];
      b = sm.rk_max[lane];
    }
#pragma unroll
    for (int off = 16; off > 0; off >>= 1) {
      a = min(a, __shfl_xor_sync(0xffffffffu, a, off));
      b = max(b, __shfl_xor_sync(0xffffffffu, b, off));
    }
    if (tid == 0) {
      sm.gkmin = a;
      sm.gkmax = b;
    }
  }
  __syncthreads();
  const uint32_t gkmin = sm.gkmin, range = sm.gkmax - sm.gkmin;

  // ---- 2. histogram rounds while the candidates are too many ----
  // Candidates: keys in value bin b1 (once that round ran) whose
  // u = key - gkmin satisfies u >> lo_bit == prefix.
  uint32_t need = k, cnt = n, prefix = 0;
  int lo_bit = range == 0 ? 0 : 32 - __clz(range);
  int b1 = -1, buf = 0;
  const float vmin = key_value(gkmin), vmax = key_value(sm.gkmax);
  const float vscale = static_cast<float>(kClusterBins) / (vmax - vmin);
  auto matches = [&](uint32_t kk) -> bool {
    if (b1 >= 0 && cluster_value_bin(kk, vmin, vscale) != b1) return false;
    return lo_bit >= 32 || ((kk - gkmin) >> lo_bit) == prefix;
  };
  bool value_round =
      range != 0 && isfinite(vscale) && vscale > 0.f && n > static_cast<uint32_t>(kClusterCand);
#pragma unroll 1
  while (value_round || (cnt > static_cast<uint32_t>(kClusterCand) && lo_bit > 0)) {
    const int dbits = value_round ? 8 : (lo_bit >= 8 ? 8 : lo_bit);
    const int shift = value_round ? 0 : lo_bit - dbits;
    const uint32_t dmask = (1u << dbits) - 1u;
    uint32_t *h = sm.hist[0];
    for (int b = tid; b < kClusterBins; b += NT) h[b] = 0;
    __syncthreads();
    for (uint32_t i = tid; i < m; i += NT) {
      const uint32_t kk = key(i);
      if (matches(kk))
        atomicAdd(&h[value_round ? cluster_value_bin(kk, vmin, vscale)
                                 : static_cast<int>(((kk - gkmin) >> shift) & dmask)],
                  1u);
    }
    __syncthreads();
    uint32_t (*part)[kClusterBins] = sm.part[buf];
    if (static_cast<uint32_t>(tid) < 64u * C) {   // push this histogram to every rank
      const int dst = tid >> 6, q = tid & 63;
      dsmem_st4(dsmem_addr(smem_u32(&part[r][4 * q]), dst),
                *reinterpret_cast<const uint4 *>(&h[4 * q]));
    }
    cluster_sync();
    if (tid < kClusterBins) {
      uint32_t sum = 0;
      for (uint32_t j = 0; j < C; ++j) sum += part[j][tid];
      sm.ghist[tid] = sum;
    }
    __syncthreads();
    select_bin<NT>(sm, sm.ghist, need, 1 << dbits);
    const uint32_t bin = sm.sel_bin;
    if (static_cast<uint32_t>(warp) < C) {        // per rank: above the bin, in it
      uint32_t above = 0;
      for (int b = static_cast<int>(bin) + 1 + lane; b < (1 << dbits); b += 32) above += part[warp][b];
      above = __reduce_add_sync(0xffffffffu, above);
      if (lane == 0) {
        sm.gt_above[warp] += above;
        sm.cnt_sel[warp] = part[warp][bin];
      }
    }
    __syncthreads();
    need -= sm.sel_above;
    cnt = sm.ghist[bin];
    if (value_round) {
      b1 = static_cast<int>(bin);
      value_round = false;
    } else {
      prefix = (lo_bit >= 32 ? 0u : (prefix << dbits)) | bin;
      lo_bit = shift;
    }
    buf ^= 1;
  }

  // ---- 3. the exact threshold ----
  uint32_t tau, need_eq;
  if (lo_bit == 0) {
    // every candidate key is the same: tau itself
    tau = gkmin + prefix;
    need_eq = need;
    if (static_cast<uint32_t>(tid) < C) {
      sm.cnt_gt[tid] = sm.gt_above[tid];
      sm.cnt_eq[tid] = sm.cnt_sel[tid];
    }
    cluster_sync();   // other ranks are done reading this CTA's histograms
  } else {
    // every rank's candidates into every rank's list (barrier C)
    uint32_t off = 0;
    for (uint32_t j = 0; j < r; ++j) off += sm.cnt_sel[j];
    uint32_t dst[kClusterMaxRanks];
#pragma unroll
    for (int d = 0; d < kClusterMaxRanks; ++d)
      dst[d] = d < static_cast<int>(C) ? dsmem_addr(smem_u32(&sm.cand[0]), d) : 0u;
    for (uint32_t i = tid; i < m; i += NT) {
      const uint32_t kk = key(i);
      if (matches(kk)) {
        const uint32_t slot = off + atomicAdd(&sm.cursor, 1u);
        if (slot < static_cast<uint32_t>(kClusterCand)) {
#pragma unroll
          for (int d = 0; d < kClusterMaxRanks; ++d)
            if (d < static_cast<int>(C)) dsmem_st(dst[d] + 4u * slot, kk);
        }
      }
    }
    cluster_sync();   // no shared memory of another CTA is touched after this
    cand_select<NT>(sm, cnt, need);
    tau = sm.tau;
    need_eq = sm.need_eq;
    if (static_cast<uint32_t>(warp) < C) {   // per rank: its candidates above / at tau
      uint32_t o = 0;
      for (int j = 0; j < warp; ++j) o += sm.cnt_sel[j];
      uint32_t g = 0, e = 0;
      for (uint32_t j = lane; j < sm.cnt_sel[warp]; j += 32) {
        const uint32_t kk = sm.cand[o + j];
        g += kk > tau;
        e += kk == tau;
      }
      g = __reduce_add_sync(0xffffffffu, g);
      e = __reduce_add_sync(0xffffffffu, e);
      if (lane == 0) {
        sm.cnt_gt[warp] = sm.gt_above[warp] + g;
        sm.cnt_eq[warp] = e;
      }
    }
    __syncthreads();
  }

  // ---- 4. output ----
  uint32_t gt_off = 0, eq_off = 0, n_gt = 0, tot_eq = 0;
  for (uint32_t j = 0; j < C; ++j) {
    if (j < r) {
      gt_off += sm.cnt_gt[j];
      eq_off += sm.cnt_eq[j];
    }
    n_gt += sm.cnt_gt[j];
    tot_eq += sm.cnt_eq[j];
  }
  if (need_eq == tot_eq) {
    // every key above tau and every tie: any order
    for (uint32_t c0 = 0; c0 < m; c0 += NT) {
      const uint32_t i = c0 + tid;
      const uint32_t kk = i < m ? key(i) : 0u;
      const bool gt = i < m && kk > tau;
      const bool eq = i < m && kk == tau;
      const unsigned mgt = __ballot_sync(0xffffffffu, gt);
      if (mgt) {
        uint32_t base = 0;
        if (lane == 0) base = atomicAdd(&sm.out_gt, __popc(mgt));
        base = __shfl_sync(0xffffffffu, base, 0);
        const uint32_t o = gt_off + base + __popc(mgt & ((1u << lane) - 1u));
        if (gt && o < k) out[o] = static_cast<int>(lo + i);
      }
      const unsigned meq = __ballot_sync(0xffffffffu, eq);
      if (meq) {
        uint32_t base = 0;
        if (lane == 0) base = atomicAdd(&sm.out_eq, __popc(meq));
        base = __shfl_sync(0xffffffffu, base, 0);
        const uint32_t o = n_gt + eq_off + base + __popc(meq & ((1u << lane) - 1u));
        if (eq && o < k) out[o] = static_cast<int>(lo + i);
      }
    }
    return;
  }
  // only some ties are taken: the lowest slots, so ties go in slot order
  uint32_t eq_base = eq_off;
  for (uint32_t c0 = 0; c0 < m; c0 += 4 * NT) {
    uint32_t gtm = 0, eqm = 0;        // bit j: entry c0 + 4*tid + j
#pragma unroll
    for (int j = 0; j < 4; ++j) {
      const uint32_t i = c0 + 4 * tid + j;
      if (i < m) {
        const uint32_t kk = key(i);
        gtm |= static_cast<uint32_t>(kk > tau) << j;
        eqm |= static_cast<uint32_t>(kk == tau) << j;
      }
    }
    if (gtm) {
      uint32_t o = gt_off + atomicAdd(&sm.out_gt, __popc(gtm));
#pragma unroll
      for (int j = 0; j < 4; ++j)
        if (gtm >> j & 1u) {
          if (o < k) out[o] = static_cast<int>(lo + c0 + 4 * tid + j);
          ++o;
        }
    }
    uint32_t total;
    const uint32_t own = __popc(eqm);
    uint32_t e = eq_base + block_incl_scan<NT>(own, sm, &total) - own;
#pragma unroll
    for (int j = 0; j < 4; ++j)
      if (eqm >> j & 1u) {
        if (e < need_eq && n_gt + e < k) out[n_gt + e] = static_cast<int>(lo + c0 + 4 * tid + j);
        ++e;
      }
    eq_base += total;
  }
}

}  // namespace dsa
