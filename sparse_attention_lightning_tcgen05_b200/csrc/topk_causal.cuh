// topk_causal.cuh -- per-row top-k of packed causal (prefill) score rows.
//
// The same selection as topk_kernel (the index_topk valid slots with the
// largest scores, ties at the threshold to the lowest slots; DeepSeek-V3.2
// Sparse Indexer Kernel API Reference, Notes: an unordered set). One CTA per
// row; every score is ordered by its monotone 32-bit key (score_key). Rows
// that fit the shared-memory stage take the two-pass selection, longer rows
// the sampled threshold; either falls back to topk_row_full (which handles
// any distribution) when its fast path cannot finish.
//
// Two-pass selection (staged rows):
//   A. one read of the row: the keys go to shared memory and into a
//      2048-bin histogram of their top 11 bits (sign, exponent, two mantissa
//      bits); the bin b holding the k-th largest key follows from one block
//      scan;
//   B. one pass over the staged keys: keys above bin b are written out at
//      once (warp-aggregated offsets), keys in bin b become candidates (key
//      and slot); the candidates (a few percent of the row) resolve the
//      exact threshold key tau with two more digits (bits 10..20, 0..9), the
//      ties at tau take the lowest slots (a binary search on the slot when
//      only some are taken). More than kTwoPassCand candidates: fallback.
//
// Sampled threshold (rows that do not fit the stage):
//   1. a sample: every sstride-th 16-byte chunk of the row (at least 1 in 8,
//      at most 1536 chunks); its keys' exact r-th largest (three radix
//      digits, 11, 11, 10 bits) is the threshold t_lo, r chosen so that about
//      k + max(k/2, 256) of the row's scores are expected at or above it (the
//      spread of that count is a few percent of it);
//   2. one pass over the row compares each score with t_lo (one float
//      compare); the scores at or above it become candidates (key and slot),
//      16 a thread per round with one warp scan;
//   3. among the candidates (at least k, at most kCausalCand), three radix
//      digits give the exact k-th key and the ties it takes. Fewer than k
//      candidates, or more than fit: fallback.
#pragma once

#include <cstdint>

#include "topk_kernel.cuh"
#include "topk_rows.cuh"

namespace dsa {

constexpr int kTwoPassCand = 2048;        // candidates of the threshold bin kept in smem

template <int NT>
struct TwoPassShared {
  uint32_t hist[kTopkBins];
  uint32_t ckey[kTwoPassCand];
  uint32_t cslot[kTwoPassCand];
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
      if (base < static_cast<uint32_t>(kTwoPassCand)) {
        ckey[base] = keys[q];
        cslot[base] = s0 + q;
      }
      ++base;
    }
}

constexpr int kCausalCand = 6144;        // candidates (and sample keys) in smem
constexpr int kCausalSampleChunks = 1536;

template <int NT>
struct SampledShared {
  uint32_t hist[kTopkBins];
  uint32_t ckey[kCausalCand];            // first the sample keys, then the candidates'
  uint32_t cslot[kCausalCand];
  uint32_t warp_a[NT / 32];
  uint32_t warp_b[NT / 32];
  uint32_t sel_bin, sel_above;
  uint32_t nout, ncand;
  int seq;
  long long seq_off;
};

// Exact need-th largest (1-based) of the keys list[0, m) by three radix
// digits (bits 21..31, 10..20, 0..9): returns the key and, in *need_out, how
// many keys equal to it the need largest take. Whole block; sm.hist is used.
template <int NT, typename SM>
__device__ uint32_t keys_select(SM &sm, const uint32_t *list, uint32_t m, uint32_t need,
                                uint32_t *need_out) {
  const int tid = threadIdx.x;
  for (int b = tid; b < kTopkBins; b += NT) sm.hist[b] = 0;
  __syncthreads();
  for (uint32_t i = tid; i < m; i += NT) atomicAdd(&sm.hist[list[i] >> 21], 1u);
  __syncthreads();
  select_bin<NT>(sm, sm.hist, need, kTopkBins);
  const uint32_t b1 = sm.sel_bin;
  need -= sm.sel_above;
  __syncthreads();
  for (int b = tid; b < kTopkBins; b += NT) sm.hist[b] = 0;
  __syncthreads();
  for (uint32_t i = tid; i < m; i += NT) {
    const uint32_t key = list[i];
    if ((key >> 21) == b1) atomicAdd(&sm.hist[(key >> 10) & 2047u], 1u);
  }
  __syncthreads();
  select_bin<NT>(sm, sm.hist, need, 2048);
  const uint32_t b2 = sm.sel_bin;
  need -= sm.sel_above;
  __syncthreads();
  for (int b = tid; b < 1024; b += NT) sm.hist[b] = 0;
  __syncthreads();
  const uint32_t top = (b1 << 11) | b2;
  for (uint32_t i = tid; i < m; i += NT) {
    const uint32_t key = list[i];
    if ((key >> 10) == top) atomicAdd(&sm.hist[key & 1023u], 1u);
  }
  __syncthreads();
  select_bin<NT>(sm, sm.hist, need, 1024);
  const uint32_t b3 = sm.sel_bin;
  need -= sm.sel_above;
  __syncthreads();
  *need_out = need;
  return (top << 10) | b3;
}

// A warp's positions in a list for `cnt` entries a thread: one warp scan and
// one shared atomic on the list's cursor per warp. Full warp.
__device__ __forceinline__ uint32_t warp_list_base(uint32_t cnt, uint32_t *cursor) {
  const int lane = threadIdx.x & 31;
  uint32_t incl = cnt;
#pragma unroll
  for (int off = 1; off < 32; off <<= 1) {
    const uint32_t v = __shfl_up_sync(0xffffffffu, incl, off);
    if (lane >= off) incl += v;
  }
  const uint32_t total = __shfl_sync(0xffffffffu, incl, 31);
  uint32_t base = 0;
  if (lane == 31 && total) base = atomicAdd(cursor, total);
  return __shfl_sync(0xffffffffu, base, 31) + incl - cnt;
}

// Block-wide sum of one value a thread (two barriers).
template <int NT, typename SM>
__device__ __forceinline__ uint32_t block_sum(SM &sm, uint32_t v) {
  v = warp_sum(v);
  if ((threadIdx.x & 31) == 0) sm.warp_a[threadIdx.x >> 5] = v;
  __syncthreads();
  uint32_t tot = 0;
#pragma unroll
  for (int w = 0; w < NT / 32; ++w) tot += sm.warp_a[w];
  __syncthreads();
  return tot;
}

// The two-pass selection of a staged row (n + 3 <= p.stage_cap).
template <int NT>
__device__ void topk_row_two_pass(const TopkParams &p, uint8_t *smem_raw, const float *row,
                                  uint32_t n, int *out) {
  TwoPassShared<NT> &sm = *reinterpret_cast<TwoPassShared<NT> *>(smem_raw);
  uint32_t *stage = reinterpret_cast<uint32_t *>(
      smem_raw + ((sizeof(TwoPassShared<NT>) + 15) & ~size_t(15)));
  const int tid = threadIdx.x;
  const int lane = tid & 31;
  const uint32_t k = static_cast<uint32_t>(p.k);
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

  if (m > static_cast<uint32_t>(kTwoPassCand)) {
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

// The sampled-threshold selection of a row of n > k scores.
template <int NT>
__device__ void topk_row_sampled(const TopkParams &p, uint8_t *smem_raw, const float *row,
                                 uint32_t n, int *out) {
  SampledShared<NT> &sm = *reinterpret_cast<SampledShared<NT> *>(smem_raw);
  const int tid = threadIdx.x;
  const uint32_t k = static_cast<uint32_t>(p.k);
  const uint32_t tgt = k + max(k / 2, 256u);          // expected candidates
  const bool take_all = n <= static_cast<uint32_t>(kCausalCand);
  bool fallback = !take_all && tgt > static_cast<uint32_t>(kCausalCand) * 2 / 3;
  // slots [0, head) come before the row's first 16-byte boundary
  const uint32_t head =
      min(n, static_cast<uint32_t>((16u - (reinterpret_cast<uintptr_t>(row) & 15u)) & 15u) / 4u);
  const uint32_t nvec = (n - head) / 4;
  const uint32_t tail0 = head + 4 * nvec;
  const float4 *v4 = reinterpret_cast<const float4 *>(row + head);
  float tlo = -__int_as_float(0x7f800000);

  if (!take_all && !fallback) {
    // ---- 1. the sample and its exact r-th largest key ----
    const uint32_t sstride = max(8u, (nvec + kCausalSampleChunks - 1) / kCausalSampleChunks);
    const uint32_t nsc = (nvec + sstride - 1) / sstride;
    const uint32_t nsamp = 4 * nsc;
    for (uint32_t s = tid; s < nsc; s += NT) {
      const float4 v = __ldg(v4 + static_cast<size_t>(s) * sstride);
      *reinterpret_cast<uint4 *>(&sm.ckey[4 * s]) =
          make_uint4(score_key(v.x), score_key(v.y), score_key(v.z), score_key(v.w));
    }
    __syncthreads();
    const uint32_t r = static_cast<uint32_t>(
        max(static_cast<uint64_t>(1), static_cast<uint64_t>(tgt) * nsamp / n));
    if (r >= nsamp) {
      fallback = true;
    } else {
      uint32_t unused;
      tlo = key_value(keys_select<NT>(sm, sm.ckey, nsamp, r, &unused));
    }
  }
  if (!fallback) {
    // ---- 2. the candidates: every score, or those at or above t_lo ----
    if (tid == 0) {
      sm.ncand = take_all ? n : 0u;
      sm.nout = 0;
    }
    __syncthreads();
    if (take_all) {
      for (uint32_t s = tid; s < n; s += NT) {
        sm.ckey[s] = score_key(__ldg(row + s));
        sm.cslot[s] = s;
      }
    } else {
      // the slots before the first and after the last whole chunk (< 8)
      const uint32_t edge = head + (n - tail0);
      if (tid < 32) {
        uint32_t s = 0, sel = 0;
        float v = 0.f;
        if (static_cast<uint32_t>(tid) < edge) {
          s = static_cast<uint32_t>(tid) < head ? tid : tail0 + (tid - head);
          v = __ldg(row + s);
          sel = v >= tlo;
        }
        const uint32_t base = warp_list_base(sel, &sm.ncand);
        if (sel && base < static_cast<uint32_t>(kCausalCand)) {
          sm.ckey[base] = score_key(v);
          sm.cslot[base] = s;
        }
      }
      // the chunks: round R gives thread tid the chunks R*4*NT + tid + j*NT
      const uint32_t rounds = (nvec + 4 * NT - 1) / (4 * NT);
      for (uint32_t R = 0; R < rounds; ++R) {
        const uint32_t c0 = R * 4 * NT + tid;
        float4 v[4];
#pragma unroll
        for (int j = 0; j < 4; ++j)
          v[j] = c0 + j * NT < nvec ? __ldg(v4 + c0 + j * NT) : make_float4(0.f, 0.f, 0.f, 0.f);
        uint32_t mask = 0;
#pragma unroll
        for (int j = 0; j < 4; ++j) {
          if (c0 + j * NT < nvec) {
            mask |= static_cast<uint32_t>(v[j].x >= tlo) << (4 * j);
            mask |= static_cast<uint32_t>(v[j].y >= tlo) << (4 * j + 1);
            mask |= static_cast<uint32_t>(v[j].z >= tlo) << (4 * j + 2);
            mask |= static_cast<uint32_t>(v[j].w >= tlo) << (4 * j + 3);
          }
        }
        uint32_t base = warp_list_base(__popc(mask), &sm.ncand);
#pragma unroll
        for (int b = 0; b < 16; ++b) {
          if (mask >> b & 1u) {
            if (base < static_cast<uint32_t>(kCausalCand)) {
              const float4 &w = v[b >> 2];
              const float x = (b & 3) == 0 ? w.x : (b & 3) == 1 ? w.y : (b & 3) == 2 ? w.z : w.w;
              sm.ckey[base] = score_key(x);
              sm.cslot[base] = head + 4 * (c0 + (b >> 2) * NT) + (b & 3);
            }
            ++base;
          }
        }
      }
    }
    __syncthreads();
    const uint32_t m = sm.ncand;
    fallback = m < k || m > static_cast<uint32_t>(kCausalCand);
    if (!fallback) {
      // ---- 3. the exact selection among the candidates ----
      uint32_t need;                                 // ties at tau to take
      const uint32_t tau = keys_select<NT>(sm, sm.ckey, m, k, &need);
      uint32_t mine = 0;
      for (uint32_t i = tid; i < m; i += NT) mine += sm.ckey[i] == tau;
      const uint32_t n_eq = block_sum<NT>(sm, mine);
      uint32_t slot_lim = 0xffffffffu;               // ties with slot < slot_lim are taken
      if (need < n_eq) {
        uint32_t lo = 0, hi = n;                     // count(slot < hi) >= need
        while (lo + 1 < hi) {
          const uint32_t mid = (lo + hi) / 2;
          uint32_t cnt = 0;
          for (uint32_t i = tid; i < m; i += NT) cnt += sm.ckey[i] == tau && sm.cslot[i] < mid;
          if (block_sum<NT>(sm, cnt) >= need) hi = mid; else lo = mid;
        }
        slot_lim = hi;
      }
      const uint32_t orounds = (m + NT - 1) / NT;
      for (uint32_t R = 0; R < orounds; ++R) {
        const uint32_t i = R * NT + tid;
        uint32_t sel = 0, s = 0;
        if (i < m) {
          const uint32_t key = sm.ckey[i];
          s = sm.cslot[i];
          sel = key > tau || (key == tau && s < slot_lim);
        }
        const uint32_t base = warp_list_base(sel, &sm.nout);
        if (sel && base < k) out[base] = static_cast<int>(s);
      }
      return;
    }
  }
  // a sample far from the row or a crowded threshold: the general selection
  __syncthreads();
  topk_row_full<NT>(p, *reinterpret_cast<TopkShared<NT> *>(smem_raw),
                    reinterpret_cast<float *>(smem_raw + sizeof(TopkShared<NT>)), row, n, out);
}

// CTAs an SM should hold (caps the registers a thread; build-time tunable)
#ifndef DSA_CAUSAL_TOPK_MIN_BLOCKS
#define DSA_CAUSAL_TOPK_MIN_BLOCKS 3
#endif

template <int NT>
__global__ void __launch_bounds__(NT, DSA_CAUSAL_TOPK_MIN_BLOCKS)
    topk_causal_kernel(const TopkParams p) {
  extern __shared__ __align__(16) uint8_t smem_raw[];
  const int t = blockIdx.x;
  const int tid = threadIdx.x;
  grid_dep_wait();                 // scores come from earlier work on the stream
  grid_dep_launch_dependents();
  if (*p.cu_bad) return;           // a cu_seqlens array that failed its check

  const float *row;
  int64_t nvalid;
  topk_row_geometry<NT>(p, t, *reinterpret_cast<TopkShared<NT> *>(smem_raw), row, nvalid);
  int *out = p.topk + static_cast<int64_t>(t) * p.k;
  const uint32_t k = static_cast<uint32_t>(p.k);
  if (nvalid <= static_cast<int64_t>(k)) {
    for (uint32_t i = tid; i < k; i += NT) out[i] = i < nvalid ? static_cast<int>(i) : -1;
    return;
  }
  const uint32_t n = static_cast<uint32_t>(nvalid);
  __syncthreads();                 // the geometry's shared words are reused
  if (n + 3 <= static_cast<uint32_t>(p.stage_cap))
    topk_row_two_pass<NT>(p, smem_raw, row, n, out);
  else
    topk_row_sampled<NT>(p, smem_raw, row, n, out);
}

}  // namespace dsa
