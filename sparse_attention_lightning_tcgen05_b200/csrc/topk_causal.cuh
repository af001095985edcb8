// topk_causal.cuh -- per-row top-k of packed causal (prefill) score rows in
// two passes over the row.
//
// The same selection as topk_kernel (the index_topk valid slots with the
// largest scores, ties at the threshold to the lowest slots; DeepSeek-V3.2
// Sparse Indexer Kernel API Reference, Notes: an unordered set). One CTA per
// row; every score becomes a monotone 32-bit key (score_key).
//   A. one read of the row from memory: the keys go to shared memory (rows
//      that fit the stage) and into a 2048-bin histogram of their top 11 bits
//      (sign, exponent, two mantissa bits);
//   the bin b holding the k-th largest key follows from one block scan;
//   B. one pass over the staged keys (or the row again, from L2): keys above
//      bin b are written out at once (warp-aggregated offsets), keys in bin b
//      become candidates (key and slot) in shared memory;
//   the candidates (a few percent of the row) then resolve the exact
//   threshold key tau with two more digits (bits 10..20, then 0..9), and the
//   ties at tau take the lowest slots (a binary search on the slot when only
//   some are taken).
// A threshold bin with more candidates than fit (long runs of equal scores)
// sends the row to topk_row_full, which handles any distribution.
#pragma once

#include <cstdint>

#include "topk_kernel.cuh"
#include "topk_rows.cuh"

namespace dsa {

constexpr int kCausalCand = 2048;        // candidates of the threshold bin kept in smem

template <int NT>
struct CausalTopkShared {
  uint32_t hist[kTopkBins];
  uint32_t ckey[kCausalCand];
  uint32_t cslot[kCausalCand];
  uint32_t warp_a[NT / 32];
  uint32_t warp_b[NT / 32];
  uint32_t sel_bin, sel_above;
  uint32_t nout, ncand;
  uint32_t small[32];
  uint32_t nsmall;
  int seq;
  long long seq_off;
  // followed by the staged keys (dynamic size)
};

// Append the selected ones of this thread's (up to 4) slots to a list: one
// atomic per warp on the list's cursor; each thread writes its own slots at
// consecutive positions. sel: bit q set = slot s0 + q selected. Full warp.
__device__ __forceinline__ void warp_append4(uint32_t sel, uint32_t s0, uint32_t *cursor,
                                             int *out, uint32_t out_cap) {
  const int lane = threadIdx.x & 31;
  const uint32_t c = __popc(sel);
  uint32_t incl = c;
#pragma unroll
  for (int off = 1; off < 32; off <<= 1) {
    const uint32_t v = __shfl_up_sync(0xffffffffu, incl, off);
    if (lane >= off) incl += v;
  }
  const uint32_t total = __shfl_sync(0xffffffffu, incl, 31);
  if (total == 0) return;
  uint32_t base = 0;
  if (lane == 31) base = atomicAdd(cursor, total);
  base = __shfl_sync(0xffffffffu, base, 31) + incl - c;
#pragma unroll
  for (int q = 0; q < 4; ++q)
    if (sel >> q & 1u) {
      if (base < out_cap) out[base] = static_cast<int>(s0 + q);
      ++base;
    }
}

// The same for candidates: key and slot pairs.
__device__ __forceinline__ void warp_append4_cand(uint32_t sel, uint32_t s0, const uint32_t *keys,
                                                  uint32_t *cursor, uint32_t *ckey,
                                                  uint32_t *cslot) {
  const int lane = threadIdx.x & 31;
  const uint32_t c = __popc(sel);
  uint32_t incl = c;
#pragma unroll
  for (int off = 1; off < 32; off <<= 1) {
    const uint32_t v = __shfl_up_sync(0xffffffffu, incl, off);
    if (lane >= off) incl += v;
  }
  const uint32_t total = __shfl_sync(0xffffffffu, incl, 31);
  if (total == 0) return;
  uint32_t base = 0;
  if (lane == 31) base = atomicAdd(cursor, total);
  base = __shfl_sync(0xffffffffu, base, 31) + incl - c;
#pragma unroll
  for (int q = 0; q < 4; ++q)
    if (sel >> q & 1u) {
      if (base < static_cast<uint32_t>(kCausalCand)) {
        ckey[base] = keys[q];
        cslot[base] = s0 + q;
      }
      ++base;
    }
}

template <int NT>
__global__ void __launch_bounds__(NT) topk_causal_kernel(const TopkParams p) {
  extern __shared__ __align__(16) uint8_t smem_raw[];
  CausalTopkShared<NT> &sm = *reinterpret_cast<CausalTopkShared<NT> *>(smem_raw);
  uint32_t *stage = reinterpret_cast<uint32_t *>(
      smem_raw + ((sizeof(CausalTopkShared<NT>) + 15) & ~size_t(15)));
  const int t = blockIdx.x;
  const int tid = threadIdx.x;
  const int lane = tid & 31;
  grid_dep_wait();                 // scores come from earlier work on the stream
  grid_dep_launch_dependents();
  if (*p.cu_bad) return;           // a cu_seqlens array that failed its check

  const float *row;
  int64_t nvalid;
  topk_row_geometry<NT>(p, t, sm, row, nvalid);
  int *out = p.topk + static_cast<int64_t>(t) * p.k;
  const uint32_t k = static_cast<uint32_t>(p.k);
  if (nvalid <= static_cast<int64_t>(k)) {
    for (uint32_t i = tid; i < k; i += NT) out[i] = i < nvalid ? static_cast<int>(i) : -1;
    return;
  }
  const uint32_t n = static_cast<uint32_t>(nvalid);
  // slots [0, head) come before the row's first 16-byte boundary; slot s is
  // staged at stage[s + o], so that the vector body lands on 16-byte rows
  const uint32_t head =
      min(n, static_cast<uint32_t>((16u - (reinterpret_cast<uintptr_t>(row) & 15u)) & 15u) / 4u);
  const uint32_t o = (4u - head) & 3u;
  const uint32_t nvec = (n - head) / 4;
  const uint32_t tail0 = head + 4 * nvec;
  const bool staged = n + 3 <= static_cast<uint32_t>(p.stage_cap);
  const float4 *v4 = reinterpret_cast<const float4 *>(row + head);

  for (int b = tid; b < kTopkBins; b += NT) sm.hist[b] = 0;
  if (tid == 0) {
    sm.nout = 0;
    sm.ncand = 0;
  }
  __syncthreads();

  // ---- A. keys, stage, top-11-bit histogram ----
  for (uint32_t s = tid; s < head; s += NT) {
    const uint32_t key = score_key(__ldg(row + s));
    if (staged) stage[s + o] = key;
    atomicAdd(&sm.hist[key >> 21], 1u);
  }
#pragma unroll 4
  for (uint32_t i = tid; i < nvec; i += NT) {
    const float4 v = __ldg(v4 + i);
    const uint4 kk = make_uint4(score_key(v.x), score_key(v.y), score_key(v.z), score_key(v.w));
    if (staged) *reinterpret_cast<uint4 *>(stage + head + o + 4 * i) = kk;
    atomicAdd(&sm.hist[kk.x >> 21], 1u);
    atomicAdd(&sm.hist[kk.y >> 21], 1u);
    atomicAdd(&sm.hist[kk.z >> 21], 1u);
    atomicAdd(&sm.hist[kk.w >> 21], 1u);
  }
  for (uint32_t s = tail0 + tid; s < n; s += NT) {
    const uint32_t key = score_key(__ldg(row + s));
    if (staged) stage[s + o] = key;
    atomicAdd(&sm.hist[key >> 21], 1u);
  }
  __syncthreads();
  select_bin<NT>(sm, sm.hist, k, kTopkBins);
  const uint32_t b1 = sm.sel_bin;
  const uint32_t above1 = sm.sel_above;       // keys in bins above b1: all taken
  const uint32_t m = sm.hist[b1];              // the threshold bin's keys
  uint32_t need = k - above1;                  // of them, how many the set takes
  __syncthreads();                             // hist is reused below

  if (m > static_cast<uint32_t>(kCausalCand)) {
    // a crowded threshold bin: the general selection (restages the row)
    topk_row_full<NT>(p, *reinterpret_cast<TopkShared<NT> *>(smem_raw),
                      reinterpret_cast<float *>(smem_raw + sizeof(TopkShared<NT>)), row, n, out);
    return;
  }

  // ---- B. keys above bin b1 out, bin b1 to the candidates ----
  // Every thread runs the same number of warp-collective rounds: the loop
  // bounds are rounded up to whole warps.
  {
    auto classify = [&](uint32_t s0, const uint32_t (&kk)[4], uint32_t valid) {
      uint32_t gt = 0, eq = 0;
#pragma unroll
      for (int q = 0; q < 4; ++q) {
        const uint32_t d = kk[q] >> 21;
        gt |= static_cast<uint32_t>((valid >> q & 1u) && d > b1) << q;
        eq |= static_cast<uint32_t>((valid >> q & 1u) && d == b1) << q;
      }
      warp_append4(gt, s0, &sm.nout, out, k);
      // members of the threshold bin are a few percent of the row: most
      // rounds have none in the whole warp
      if (__any_sync(0xffffffffu, eq != 0u))
        warp_append4_cand(eq, s0, kk, &sm.ncand, sm.ckey, sm.cslot);
    };
    // head and tail slots: one per thread, as a 1-slot group
    const uint32_t edge = head + (n - tail0);
    const uint32_t edge_rounds = (edge + NT - 1) / NT;
    for (uint32_t r = 0; r < edge_rounds; ++r) {
      const uint32_t e = r * NT + tid;
      uint32_t kk[4] = {0u, 0u, 0u, 0u};
      uint32_t s = 0, valid = 0;
      if (e < edge) {
        s = e < head ? e : tail0 + (e - head);
        kk[0] = staged ? stage[s + o] : score_key(__ldg(row + s));
        valid = 1u;
      }
      classify(s, kk, valid);
    }
    const uint32_t body_rounds = (nvec + NT - 1) / NT;
    for (uint32_t r = 0; r < body_rounds; ++r) {
      const uint32_t i = r * NT + tid;
      uint32_t kk[4] = {0u, 0u, 0u, 0u};
      uint32_t valid = 0;
      if (i < nvec) {
        if (staged) {
          const uint4 v = *reinterpret_cast<const uint4 *>(stage + head + o + 4 * i);
          kk[0] = v.x; kk[1] = v.y; kk[2] = v.z; kk[3] = v.w;
        } else {
          const float4 v = __ldg(v4 + i);
          kk[0] = score_key(v.x); kk[1] = score_key(v.y);
          kk[2] = score_key(v.z); kk[3] = score_key(v.w);
        }
        valid = 0xFu;
      }
      classify(head + 4 * i, kk, valid);
    }
  }
  for (int b = tid; b < kTopkBins; b += NT) sm.hist[b] = 0;
  __syncthreads();

  // ---- the candidates: digit 2 (key bits 10..20) ----
  for (uint32_t i = tid; i < m; i += NT) atomicAdd(&sm.hist[(sm.ckey[i] >> 10) & 2047u], 1u);
  __syncthreads();
  select_bin<NT>(sm, sm.hist, need, 2048);
  const uint32_t b2 = sm.sel_bin;
  need -= sm.sel_above;
  __syncthreads();
  for (int b = tid; b < 1024; b += NT) sm.hist[b] = 0;
  __syncthreads();
  // ---- digit 3 (key bits 0..9) of the candidates in bin b2 ----
  for (uint32_t i = tid; i < m; i += NT) {
    const uint32_t key = sm.ckey[i];
    if (((key >> 10) & 2047u) == b2) atomicAdd(&sm.hist[key & 1023u], 1u);
  }
  __syncthreads();
  select_bin<NT>(sm, sm.hist, need, 1024);
  const uint32_t b3 = sm.sel_bin;
  need -= sm.sel_above;                        // ties at tau to take (>= 1)
  const uint32_t n_eq = sm.hist[b3];
  const uint32_t tau = (b1 << 21) | (b2 << 10) | b3;
  __syncthreads();

  // ---- output: candidates above tau, and the ties ----
  // slot threshold for partial ties: the need-th lowest slot among the ties
  uint32_t slot_lim = 0xffffffffu;             // ties with slot < slot_lim are taken
  if (need < n_eq) {
    uint32_t lo = 0, hi = n;                   // count(slot < hi) >= need
    while (lo + 1 < hi) {
      const uint32_t mid = (lo + hi) / 2;
      uint32_t cnt = 0;
      for (uint32_t i = tid; i < m; i += NT) cnt += sm.ckey[i] == tau && sm.cslot[i] < mid;
      cnt = warp_sum(cnt);
      if (lane == 0) sm.warp_a[tid >> 5] = cnt;
      __syncthreads();
      uint32_t tot = 0;
#pragma unroll
      for (int w = 0; w < NT / 32; ++w) tot += sm.warp_a[w];
      __syncthreads();
      if (tot >= need) hi = mid; else lo = mid;
    }
    slot_lim = hi;                             // exactly `need` ties below hi
  }
  const uint32_t rounds = (m + NT - 1) / NT;
  for (uint32_t r = 0; r < rounds; ++r) {
    const uint32_t i = r * NT + tid;
    uint32_t sel = 0, s = 0;
    if (i < m) {
      const uint32_t key = sm.ckey[i];
      s = sm.cslot[i];
      sel = key > tau || (key == tau && s < slot_lim);
    }
    // one slot a thread: append as a 1-slot group
    warp_append4(sel, s, &sm.nout, out, k);
  }
}

}  // namespace dsa
