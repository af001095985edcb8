// topk_rows.cuh -- per-row top-k with the row held in registers.
//
// The same selection as topk_kernel (the index_topk valid slots with the
// largest scores; ties at the threshold go to the lowest slots; -1 padding
// when a row has fewer valid slots), for decode-style rows of at most
// NT*KPT slots, such as the rows of a pooled (compressed) key cache. One CTA
// per row. Each thread copies its chunks of the row (chunk j of thread tid
// holds slots 4*(j*NT + tid) - h .. +3, h = the row's misalignment in
// floats; chunk rows past the row's end are skipped by the whole block)
// into its own shared-memory slots, then into registers with a validity
// mask, so that every pass reads registers:
//   1. the row's smallest and largest score;
//   2. a 2048-bin histogram linear in the score value; the bin holding the
//      k-th score is found with one exchange of warp partials;
//   3. its members, when at most 32 (the usual case), go to shared memory and
//      one warp ranks them: the threshold tau and the ties it takes, which
//      that warp writes itself (the lowest slots first);
//   4. each thread marks its scores above tau; one exchange of warp totals
//      gives every warp its output offset, and for each register slot in
//      turn the warp's selected lanes write one contiguous run.
// The common path takes eight block barriers. When the bin holds more than
// 32 scores, 11-bit radix digits of their keys narrow it further; many equal
// keys at the threshold (more than 32, only some taken) go through an
// ordered pass that ranks the ties by slot.
#pragma once

#include <cstdint>

#include "topk_kernel.cuh"

namespace dsa {

constexpr int kRowsSmall = 32;

template <int NT>
struct RowsShared {
  uint32_t hist[kTopkBins];
  uint32_t part_a[NT / 32];       // per-warp partials of one phase ...
  uint32_t part_b[NT / 32];       // ... and of the next (no barrier between reuses)
  uint32_t warp_a[NT / 32];       // block_minmax / block_incl_scan / select_bin
  uint32_t warp_b[NT / 32];
  uint32_t sel_bin, sel_above;
  uint32_t kmin, kmax;
  uint32_t nsmall;
  uint32_t small_key[kRowsSmall];
  uint32_t small_slot[kRowsSmall];
  uint32_t tau, need;
};

// Warp-wide reductions and scans.
__device__ __forceinline__ uint32_t warp_sum(uint32_t v) {
#pragma unroll
  for (int off = 16; off > 0; off >>= 1) v += __shfl_xor_sync(0xffffffffu, v, off);
  return v;
}
__device__ __forceinline__ uint32_t warp_incl_scan_u32(uint32_t v, int lane) {
#pragma unroll
  for (int off = 1; off < 32; off <<= 1) {
    const uint32_t n = __shfl_up_sync(0xffffffffu, v, off);
    if (lane >= off) v += n;
  }
  return v;
}
// Sum over lanes l' >= lane.
__device__ __forceinline__ uint32_t warp_suffix_scan_u32(uint32_t v, int lane) {
#pragma unroll
  for (int off = 1; off < 32; off <<= 1) {
    const uint32_t n = __shfl_down_sync(0xffffffffu, v, off);
    if (lane + off < 32) v += n;
  }
  return v;
}

// Row t's scores and valid length, computed by every warp on its own (no
// block barrier): POSITIONS rows of S slots; CAUSAL rows of their sequence's
// L x L block, valid up to the diagonal.
__device__ __forceinline__ void rows_geometry(const TopkParams &p, int t, int lane,
                                              const float *&row, int64_t &nvalid) {
  if (p.mode == kModePositions) {
    row = p.scores + static_cast<int64_t>(t) * p.S;
    const int64_t pos = p.compressed ? compressed_last_slot(p.comp, t) : __ldg(p.positions + t);
    nvalid = pos < 0 ? 0 : (pos + 1 < p.S ? pos + 1 : p.S);
    return;
  }
  int lo = 0, hi = p.num_seqs - 1;       // largest i with cu[i] <= t
  while (lo < hi) {
    const int mid = (lo + hi + 1) / 2;
    if (__ldg(p.cu_seqlens + mid) <= t) lo = mid; else hi = mid - 1;
  }
  long long part = 0;                    // sum_{j < lo} L_j^2
  for (int j = lane; j < lo; j += 32) {
    const long long L = __ldg(p.cu_seqlens + j + 1) - __ldg(p.cu_seqlens + j);
    part += L * L;
  }
#pragma unroll
  for (int off = 16; off > 0; off >>= 1) part += __shfl_xor_sync(0xffffffffu, part, off);
  const int a = __ldg(p.cu_seqlens + lo);
  const int64_t L = __ldg(p.cu_seqlens + lo + 1) - a;
  row = p.scores + part + static_cast<int64_t>(t - a) * L;
  nvalid = t - a + 1;
}

// One row of the persistent loop: where its scores are, where its set goes,
// and what it needs.
struct RowJob {
  const float *row;
  int *out;
  uint32_t n;          // valid slots
  int kind;            // 0: too long for this instance, 1: n <= k (no selection), 2: select
};

// Floats of a row's buffer that its valid slots occupy: the buffer starts at
// the 16-byte boundary at or before the row, h = 0..3 floats earlier.
__device__ __forceinline__ int64_t rows_span(const float *row, int64_t nvalid) {
  return nvalid + static_cast<int64_t>((reinterpret_cast<uintptr_t>(row) & 15u) / 4u);
}

template <int NT, int KPT>
__device__ __forceinline__ RowJob rows_job(const TopkParams &p, int t, int lane) {
  RowJob j;
  int64_t nvalid;
  rows_geometry(p, t, lane, j.row, nvalid);
  j.out = p.topk + static_cast<int64_t>(t) * p.k;
  j.n = static_cast<uint32_t>(nvalid < 0 ? 0 : (nvalid > 0x7fffffff ? 0x7fffffff : nvalid));
  j.kind = nvalid <= p.k ? 1 : (rows_span(j.row, nvalid) > static_cast<int64_t>(NT) * KPT ? 0 : 2);
  return j;
}

// Start this thread's copies of its chunks of a row into its own slots of
// buffer `buf` (chunk j of thread tid -> buf[j*NT + tid]); whole chunks by
// one 16-byte copy, the row's ragged ends slot by slot.
template <int NT, int KPT>
__device__ __forceinline__ void rows_prefetch(const RowJob &job, float4 *buf) {
  constexpr int KV = KPT / 4;
  if (job.kind != 2) return;
  const int tid = threadIdx.x;
  const uint32_t n = job.n;
  const uint32_t h = static_cast<uint32_t>(reinterpret_cast<uintptr_t>(job.row) & 15u) / 4u;
  const float *arow = job.row - h;
  const uint32_t jmax = (h + n + 4u * NT - 1u) / (4u * NT);
#pragma unroll
  for (int j = 0; j < KV; ++j) {
    if (static_cast<uint32_t>(j) >= jmax) break;
    const uint32_t e0 = 4u * static_cast<uint32_t>(j * NT + tid);
    float4 *dst = buf + j * NT + tid;
    if (e0 >= h && e0 + 4u <= h + n) {
      cp_async16(dst, arow + e0);
    } else {
#pragma unroll
      for (int q = 0; q < 4; ++q) {
        const uint32_t s = e0 + q - h;     // wraps to a large value before the row
        if (s < n) cp_async4(reinterpret_cast<float *>(dst) + q, job.row + s);
      }
    }
  }
}

// The selection of one row whose chunks this thread has in `buf`. Ends with
// every thread past its last use of the shared state.
template <int NT, int KPT>
__device__ __forceinline__ void rows_select(const RowJob &job, const float4 *buf, uint32_t k,
                                            RowsShared<NT> &sm) {
  constexpr int KV = KPT / 4;
  constexpr int kWarps = NT / 32;
  constexpr int kBinsPerLane = kTopkBins / NT;
  const int tid = threadIdx.x;
  const int lane = tid & 31, warp = tid >> 5;
  int *const out = job.out;
  const uint32_t n = job.n;
#pragma unroll
  for (int i = 0; i < kBinsPerLane; ++i) sm.hist[tid + i * NT] = 0;
  if (tid == 0) sm.nsmall = 0;

  // ---- 1. the row from this thread's buffer slots, validity, range ----
  const uint32_t h = static_cast<uint32_t>(reinterpret_cast<uintptr_t>(job.row) & 15u) / 4u;
  const uint32_t jmax = (h + n + 4u * NT - 1u) / (4u * NT);   // chunk rows holding a slot
  float v[KPT];
  uint32_t valid = 0;                    // bit i: v[i] holds a slot of the row
  float vlo = __int_as_float(0x7f800000), vhi = -__int_as_float(0x7f800000);
#pragma unroll
  for (int j = 0; j < KV; ++j) {
    v[4 * j] = v[4 * j + 1] = v[4 * j + 2] = v[4 * j + 3] = 0.f;
    if (static_cast<uint32_t>(j) < jmax) {
      const uint32_t e0 = 4u * static_cast<uint32_t>(j * NT + tid);
      const float4 x = buf[j * NT + tid];
      v[4 * j] = x.x;
      v[4 * j + 1] = x.y;
      v[4 * j + 2] = x.z;
      v[4 * j + 3] = x.w;
#pragma unroll
      for (int q = 0; q < 4; ++q)
        if (e0 + q - h < n) valid |= 1u << (4 * j + q);   // unsigned: wraps before the row
    }
  }
#pragma unroll
  for (int i = 0; i < KPT; ++i)
    if (static_cast<uint32_t>(i / 4) < jmax && (valid >> i & 1u)) {
      vlo = fminf(vlo, v[i]);
      vhi = fmaxf(vhi, v[i]);
    }
  {
    uint32_t klo = valid ? score_key(vlo) : 0xffffffffu, khi = valid ? score_key(vhi) : 0u;
#pragma unroll
    for (int off = 16; off > 0; off >>= 1) {
      klo = min(klo, __shfl_xor_sync(0xffffffffu, klo, off));
      khi = max(khi, __shfl_xor_sync(0xffffffffu, khi, off));
    }
    if (lane == 0) {
      sm.part_a[warp] = klo;
      sm.part_b[warp] = khi;
    }
  }
  __syncthreads();                                                      // (1)
  uint32_t kmin = 0xffffffffu, kmax = 0u;
#pragma unroll
  for (int w = 0; w < kWarps; ++w) {
    kmin = min(kmin, sm.part_a[w]);
    kmax = max(kmax, sm.part_b[w]);
  }

  // ---- 2. value-linear bins ----
  uint32_t live = valid;                 // the members of the bin being resolved
  uint32_t need = k;                     // of them, how many the set still takes
  uint32_t n_live = n;
  const float vmin = key_value(kmin), vmax = key_value(kmax);
  const float vscale = 2048.f / (vmax - vmin);
  const bool value_round = kmax != kmin && isfinite(vscale) && vscale > 0.f;
  int b1 = -1;
  if (value_round) {
#pragma unroll
    for (int i = 0; i < KPT; ++i)
      if (static_cast<uint32_t>(i / 4) < jmax && (valid >> i & 1u))
        atomicAdd(&sm.hist[value_bin(v[i], vmin, vscale)], 1u);
    __syncthreads();                                                    // (2)
    // warp w owns bins [w*32*kBinsPerLane, ..): chunks of 32 consecutive bins,
    // one a lane (no bank conflicts)
    const int wbin0 = warp * 32 * kBinsPerLane;
    uint32_t own = 0;
#pragma unroll
    for (int i = 0; i < kBinsPerLane; ++i) own += sm.hist[wbin0 + i * 32 + lane];
    const uint32_t wtot = warp_sum(own);
    if (lane == 0) sm.part_a[warp] = wtot;   // part_a's minima were read before (2)
    __syncthreads();                                                    // (3)
    uint32_t above_w = 0;
#pragma unroll
    for (int w = 0; w < kWarps; ++w) above_w += w > warp ? sm.part_a[w] : 0u;
    if (above_w < need && need <= above_w + wtot) {     // this warp holds the bin
      uint32_t acc = above_w;                           // bins above the chunk
#pragma unroll
      for (int i = kBinsPerLane - 1; i >= 0; --i) {
        const uint32_t c = sm.hist[wbin0 + i * 32 + lane];
        const uint32_t suf = warp_suffix_scan_u32(c, lane);   // this bin and those above it
        const uint32_t ctot = __shfl_sync(0xffffffffu, suf, 0);
        if (acc + ctot >= need) {
          // the bin: acc + suf >= need > acc + suf - c
          if (acc + suf >= need && acc + suf - c < need) {
            sm.sel_bin = wbin0 + i * 32 + lane;
            sm.sel_above = acc + suf - c;
          }
          break;
        }
        acc += ctot;
      }
    }
    __syncthreads();                                                    // (4)
    b1 = static_cast<int>(sm.sel_bin);
    need -= sm.sel_above;
    n_live = sm.hist[b1];
  }

  // ---- radix digits on the live keys (a crowded bin; rare) ----
  uint32_t tau = 0, need_eq = 0, n_eq = 0;
  bool ties_written = false;
  if (n_live > static_cast<uint32_t>(kRowsSmall)) {
    if (value_round) {
#pragma unroll
      for (int i = 0; i < KPT; ++i)
        if ((live >> i & 1u) && value_bin(v[i], vmin, vscale) != b1) live &= ~(1u << i);
    }
    uint32_t lo = 0xffffffffu, hi = 0u;
#pragma unroll
    for (int i = 0; i < KPT; ++i)
      if (live >> i & 1u) {
        const uint32_t key = score_key(v[i]);
        lo = min(lo, key);
        hi = max(hi, key);
      }
    block_minmax<NT>(lo, hi, sm);
    const uint32_t ckmin = sm.kmin;
    const uint32_t crange = sm.kmax - ckmin;
    int lo_bit = crange == 0 ? 0 : 32 - __clz(crange);
    uint32_t prefix = 0;
#pragma unroll 1
    while (lo_bit > 0 && n_live > static_cast<uint32_t>(kRowsSmall)) {
      const int dbits = lo_bit >= 11 ? 11 : lo_bit;
      const int shift = lo_bit - dbits;
      const uint32_t dmask = (1u << dbits) - 1u;
      for (int b = tid; b < (1 << dbits); b += NT) sm.hist[b] = 0;
      __syncthreads();
#pragma unroll
      for (int i = 0; i < KPT; ++i)
        if (live >> i & 1u) atomicAdd(&sm.hist[((score_key(v[i]) - ckmin) >> shift) & dmask], 1u);
      __syncthreads();
      select_bin<NT>(sm, sm.hist, need, 1 << dbits);
      const uint32_t b = sm.sel_bin;
      need -= sm.sel_above;
      n_live = sm.hist[b];
#pragma unroll
      for (int i = 0; i < KPT; ++i)
        if ((live >> i & 1u) && (((score_key(v[i]) - ckmin) >> shift) & dmask) != b)
          live &= ~(1u << i);
      prefix = (prefix << dbits) | b;
      lo_bit = shift;
      __syncthreads();                   // every thread has read hist[b]
    }
    if (n_live > static_cast<uint32_t>(kRowsSmall)) {
      // every digit resolved: the live keys are all equal, to tau
      tau = ckmin + prefix;
      need_eq = need;
      n_eq = n_live;
    }
    b1 = -1;                             // live now marks the members
  }

  // ---- 3. the last <= 32 live keys: one warp ranks them ----
  if (n_live <= static_cast<uint32_t>(kRowsSmall)) {
#pragma unroll
    for (int i = 0; i < KPT; ++i) {
      const bool member = static_cast<uint32_t>(i / 4) < jmax && (live >> i & 1u) &&
                          (b1 < 0 || value_bin(v[i], vmin, vscale) == b1);
      if (member) {
        const uint32_t at = atomicAdd(&sm.nsmall, 1u);
        if (at < static_cast<uint32_t>(kRowsSmall)) {
          sm.small_key[at] = score_key(v[i]);
          sm.small_slot[at] = 4u * static_cast<uint32_t>((i / 4) * NT + tid) + (i % 4) - h;
        }
      }
    }
    __syncthreads();                                                    // (5)
    if (warp == 0) {
      const uint32_t nl = min(sm.nsmall, static_cast<uint32_t>(kRowsSmall));
      const bool mine_ok = static_cast<uint32_t>(lane) < nl;
      const uint32_t mine = mine_ok ? sm.small_key[lane] : 0u;
      const uint32_t my_slot = mine_ok ? sm.small_slot[lane] : 0xffffffffu;
      uint32_t above = 0, equal = 0;
#pragma unroll
      for (int l = 0; l < 32; ++l) {
        const uint32_t other = __shfl_sync(0xffffffffu, mine, l);
        const bool ok = static_cast<uint32_t>(l) < nl;
        above += ok && other > mine;
        equal += ok && other == mine;
      }
      const bool is_tau = mine_ok && above < need && need <= above + equal;
      // some lane holds tau (1 <= need <= n_live); the guards below keep every
      // write inside the row's k outputs regardless
      const int who = max(0, __ffs(__ballot_sync(0xffffffffu, is_tau)) - 1);
      const uint32_t t_key = __shfl_sync(0xffffffffu, mine, who);
      const uint32_t t_need = min(k, need - __shfl_sync(0xffffffffu, above, who));
      // the ties are all here: take the t_need lowest slots of them
      const bool tie = mine_ok && mine == t_key;
      uint32_t rank = 0;
#pragma unroll
      for (int l = 0; l < 32; ++l) {
        const uint32_t other = __shfl_sync(0xffffffffu, mine, l);
        const uint32_t oslot = __shfl_sync(0xffffffffu, my_slot, l);
        rank += static_cast<uint32_t>(l) < nl && other == t_key && oslot < my_slot;
      }
      if (tie && rank < t_need) out[k - t_need + rank] = static_cast<int>(my_slot);
      if (lane == 0) {
        sm.tau = t_key;
        sm.need = t_need;
      }
    }
    __syncthreads();                                                    // (6)
    tau = sm.tau;
    need_eq = sm.need;
    ties_written = true;
  }

  // ---- 4. output: scores above tau (and all the ties, when all are taken) ----
  const bool ties_here = !ties_written && need_eq == n_eq;
  const float tau_v = key_value(tau);    // same order as the keys (-0 == +0)
  uint32_t sel = 0;
#pragma unroll
  for (int i = 0; i < KPT; ++i)
    if (static_cast<uint32_t>(i / 4) < jmax && (valid >> i & 1u) &&
        (v[i] > tau_v || (ties_here && v[i] == tau_v)))
      sel |= 1u << i;
  const uint32_t wcnt = warp_sum(__popc(sel));
  if (lane == 0) sm.part_b[warp] = wcnt;    // part_b's maxima were read before (2)
  __syncthreads();                                                      // (7)
  // the warp's outputs start after the earlier warps'; for each register
  // slot i in turn the warp's selected lanes write one contiguous run
  uint32_t at = 0;
#pragma unroll
  for (int w = 0; w < kWarps; ++w) at += w < warp ? sm.part_b[w] : 0u;
  const uint32_t lt = (1u << lane) - 1u;
#pragma unroll
  for (int i = 0; i < KPT; ++i) {
    if (static_cast<uint32_t>(i / 4) >= jmax) break;
    const uint32_t m = __ballot_sync(0xffffffffu, sel >> i & 1u);
    const uint32_t o = at + __popc(m & lt);
    if ((sel >> i & 1u) && o < k)
      out[o] = static_cast<int>(4u * static_cast<uint32_t>((i / 4) * NT + tid) + (i % 4) - h);
    at += __popc(m);
  }
  if (ties_written || ties_here) {
    __syncthreads();                   // the next row reuses the shared state
    return;
  }

  // ---- many ties, only some taken: rank them by slot, chunk row by chunk row ----
  const uint32_t n_gt = k - need_eq;
  uint32_t before = 0;
#pragma unroll
  for (int j = 0; j < KV; ++j) {
    uint32_t c = 0;
#pragma unroll
    for (int q = 0; q < 4; ++q) {
      const int i = 4 * j + q;
      c += (valid >> i & 1u) && v[i] == tau_v;
    }
    uint32_t row_total;
    uint32_t r = before + block_incl_scan<NT>(c, sm, &row_total) - c;
#pragma unroll
    for (int q = 0; q < 4; ++q) {
      const int i = 4 * j + q;
      if ((valid >> i & 1u) && v[i] == tau_v) {
        if (r < need_eq && n_gt + r < k)
          out[n_gt + r] = static_cast<int>(4u * static_cast<uint32_t>(j * NT + tid) + q - h);
        ++r;
      }
    }
    before += row_total;
  }
  __syncthreads();                     // the next row reuses the shared state
}

// One CTA per row. The row goes through this thread's own slots of a
// shared-memory buffer (per-thread asynchronous copies), then into registers.
template <int NT, int KPT>
__global__ void __launch_bounds__(NT) topk_rows_kernel(const TopkParams p) {
  static_assert(KPT % 4 == 0 && KPT <= 32, "KPT: float4 chunks, one mask bit each");
  static_assert(kTopkBins % NT == 0, "whole bins per thread");
  __shared__ RowsShared<NT> sm;
  extern __shared__ float4 rows_buf[];   // [KPT/4][NT]
  const int t = blockIdx.x;
  const int tid = threadIdx.x;
  const uint32_t k = static_cast<uint32_t>(p.k);
  // scores (and positions) come from earlier work on the stream
  grid_dep_wait();
  grid_dep_launch_dependents();

  const RowJob job = rows_job<NT, KPT>(p, t, tid & 31);
  if (job.kind == 1) {
    for (uint32_t i = tid; i < k; i += NT) job.out[i] = i < job.n ? static_cast<int>(i) : -1;
    return;
  }
  if (job.kind == 0) {                   // the host sends no row this long
    if (tid == 0) atomicCAS(p.err, 0u, 2u);   // DSA_ERR_UNSUPPORTED, never expected
    return;
  }
  rows_prefetch<NT, KPT>(job, rows_buf);
  cp_async_commit();
  cp_async_wait<0>();
  rows_select<NT, KPT>(job, rows_buf, k, sm);
}

}  // namespace dsa
