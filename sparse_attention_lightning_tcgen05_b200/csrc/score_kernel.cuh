// score_kernel.cuh -- lightning-indexer score kernel for sm_100a.
//
// Computes I[t,s] = sum_h w[t,h] * ReLU(q[t,h,:] . k[s,:]) for valid slots
// and the finite mask bound elsewhere (DeepSeek-V3.2 Sparse Indexer Kernel
// API Reference: scores over every cached slot, clamped to a finite bound).
//
// Shape of the contraction: q . k^T is the dense [T*H, D] x [D, S] product.
// The MMA puts KEY SLOTS on M (128 per tile) and query (token, head) pairs on
// N, so accumulator lane i of TMEM holds slot i and the head reduction of
// the epilogue is thread-local: no shuffles, and a warp's 32 lanes write 32
// consecutive scores of a row.
//
//   warp 0      : work scheduler + TMA producer (one elected thread)
//   warp 1      : TMEM allocator + MMA issuer (one elected thread)
//   warps 2..   : epilogue (TMEM -> ReLU, w-weighted head sum, mask, store)
//
// Work unit = (query block of up to tq_sub*NSUB tokens sharing one key
// cache, range of `chunk_tiles` key tiles). Units are handed out through a
// global atomic counter and a small shared-memory ring so that the three
// roles walk the same sequence. Per active key tile the MMA issues one
// accumulator per sub-block (NSUB); accumulators rotate through NACC TMEM
// buffers so the epilogue of one overlaps the MMA of the next. Key tiles past
// every token's last valid slot are never loaded: the epilogue writes the
// mask bound there directly.
#pragma once

#include <cstdint>

#include "sm100_ptx.cuh"

namespace dsa {

constexpr int kBlockM = 128;          // key slots per tile (MMA M)
constexpr int kHeadDim = 128;         // D
constexpr int kSchedSlots = 4;        // unit ring depth
constexpr float kMaskBound = -0x1.FEp127f;   // lowest finite bf16

enum : int { kModePositions = 0, kModeCausal = 1 };

struct ScoreParams {
  int mode;
  int T, H;
  int64_t S;                 // POSITIONS: slots per cache
  int shared_cache;          // POSITIONS: every token reads cache 0
  int num_seqs;              // CAUSAL
  const int *cu_seqlens;     // CAUSAL
  const int *positions;      // POSITIONS
  const float *w;            // [T, H]
  float *scores;
  int tq_sub;                // tokens per MMA sub-block
  int n_cols;                // MMA N per sub-block: round_up(tq_sub*H, 16)
  int chunk_tiles;           // key tiles per work unit
  unsigned int *sched_counter;   // next unit to hand out (0 at launch)
  unsigned int *done_counter;    // CTAs finished (0 at launch)
  unsigned int *err;
  unsigned int *err_info;
  uint64_t wait_limit_ns;
};

// Shared-memory plan, identical on host and device.
struct ScoreSmem {
  uint32_t k_stage_bytes, q_sub_bytes;
  uint32_t off_k, off_q, off_bar, off_misc, total;
  __host__ __device__ ScoreSmem(int stages, int qbuf, int nsub, int n_cols,
                                bool fp8) {
    // bf16: two 128-byte-wide halves along D; fp8: one 128-byte row.
    k_stage_bytes = fp8 ? kBlockM * 128 : kBlockM * 256;
    q_sub_bytes = fp8 ? n_cols * 128 : n_cols * 256;
    off_k = 0;
    off_q = off_k + stages * k_stage_bytes;
    off_bar = off_q + qbuf * nsub * q_sub_bytes;
    off_misc = off_bar + 64 * 8;            // up to 64 mbarriers
    total = off_misc + 128 + 1024;          // misc words + alignment slack
  }
};

struct Unit {
  int t0, ntok;        // tokens [t0, t0 + ntok)
  int z;               // key-cache index (3rd TMA coordinate)
  int y0;              // first key row of the sequence (2nd TMA coordinate)
  int64_t row_len;     // slots per score row
  int64_t out0;        // float offset of token t0's score row
  int lv0;             // CAUSAL: last valid slot of token t0
  int j0, j1;          // key tiles [j0, j1) of this unit
  int j_act;           // tiles [j0, j_act) need the MMA; [j_act, j1) are masked
};

__device__ __forceinline__ int last_valid_pos(const ScoreParams &p, int t) {
  int pos = __ldg(p.positions + t);
  int64_t lv = pos < 0 ? -1 : (pos >= p.S ? p.S - 1 : pos);
  return static_cast<int>(lv);
}

// Last valid slot of token t0 + i of unit U.
__device__ __forceinline__ int unit_last_valid(const ScoreParams &p,
                                               const Unit &U, int i) {
  return p.mode == kModeCausal ? U.lv0 + i : last_valid_pos(p, U.t0 + i);
}

// Decode work unit u. Returns false once u is past the last unit. Every
// role calls this with the same u and gets the same answer.
__device__ bool decode_unit(const ScoreParams &p, int tq_total, uint32_t u,
                            Unit &U) {
  const int ch = p.chunk_tiles;
  if (p.mode == kModePositions) {
    const int64_t ntiles = (p.S + kBlockM - 1) / kBlockM;
    const int64_t nch = (ntiles + ch - 1) / ch;
    const int64_t nqb = p.shared_cache ? (p.T + tq_total - 1) / tq_total : p.T;
    if (static_cast<int64_t>(u) >= nqb * nch) return false;
    const int64_t c = u / nqb, qb = u % nqb;     // chunk-major: early slots first
    U.t0 = static_cast<int>(qb * tq_total);
    U.ntok = min(tq_total, p.T - U.t0);
    U.z = p.shared_cache ? 0 : U.t0;
    U.y0 = 0;
    U.row_len = p.S;
    U.out0 = static_cast<int64_t>(U.t0) * p.S;
    U.lv0 = 0;
    U.j0 = static_cast<int>(c * ch);
    U.j1 = static_cast<int>(U.j0 + ch < ntiles ? U.j0 + ch : ntiles);
    int mx = -1;
    for (int i = 0; i < U.ntok; ++i) mx = max(mx, last_valid_pos(p, U.t0 + i));
    U.j_act = mx < 0 ? U.j0 : min(U.j1, mx / kBlockM + 1);
    U.j_act = max(U.j_act, U.j0);
    return true;
  }
  // CAUSAL: sequences in order; inside one, the longest query blocks first.
  int64_t uu = u, seqoff = 0;
  for (int i = 0; i < p.num_seqs; ++i) {
    const int a = __ldg(p.cu_seqlens + i), b = __ldg(p.cu_seqlens + i + 1);
    const int L = b - a;
    if (L <= 0) continue;
    const int64_t nqb = (L + tq_total - 1) / tq_total;
    const int64_t ntiles = (L + kBlockM - 1) / kBlockM;
    const int64_t nch = (ntiles + ch - 1) / ch;
    if (uu < nqb * nch) {
      const int64_t blk = nqb - 1 - uu / nch, c = uu % nch;
      const int tl0 = static_cast<int>(blk * tq_total);
      U.t0 = a + tl0;
      U.ntok = min(tq_total, L - tl0);
      U.z = 0;
      U.y0 = a;
      U.row_len = L;
      U.out0 = seqoff + static_cast<int64_t>(tl0) * L;
      U.lv0 = tl0;
      U.j0 = static_cast<int>(c * ch);
      U.j1 = static_cast<int>(U.j0 + ch < ntiles ? U.j0 + ch : ntiles);
      const int mx = tl0 + U.ntok - 1;
      U.j_act = max(U.j0, min(U.j1, mx / kBlockM + 1));
      return true;
    }
    uu -= nqb * nch;
    seqoff += static_cast<int64_t>(L) * L;
  }
  return false;
}

// Epilogue for one token with H == 64 (the tuned head count): the two
// 32-column TMEM loads hold heads 0..31 and 32..63 of this slot.
__device__ __forceinline__ float head_sum_h64(uint32_t taddr, const float *wrow) {
  float v[32];
  float acc = 0.f;
  const float4 *w4 = reinterpret_cast<const float4 *>(wrow);
#pragma unroll
  for (int half = 0; half < 2; ++half) {
    tmem_ld32_wait(taddr + half * 32, v);
#pragma unroll
    for (int i = 0; i < 8; ++i) {
      const float4 wv = __ldg(w4 + half * 8 + i);
      acc = fmaf(wv.x, fmaxf(v[4 * i + 0], 0.f), acc);
      acc = fmaf(wv.y, fmaxf(v[4 * i + 1], 0.f), acc);
      acc = fmaf(wv.z, fmaxf(v[4 * i + 2], 0.f), acc);
      acc = fmaf(wv.w, fmaxf(v[4 * i + 3], 0.f), acc);
    }
  }
  return acc;
}

// Role bookkeeping of a ring of mbarrier pairs.
struct Ring {
  uint32_t idx = 0, phase = 0;
  __device__ __forceinline__ void next(uint32_t n) {
    if (++idx == n) { idx = 0; phase ^= 1u; }
  }
};

// kH: 64 selects the tuned epilogue; 0 = any H (generic epilogue).
// kNSUB: MMA sub-blocks per key tile (each its own accumulator, same A).
// kNACC: TMEM accumulator buffers. kSTAGES: key-tile smem stages.
// kQBUF: query-block smem buffers. kEPI: epilogue warps (4 or 8).
template <int kH, int kNSUB, int kNACC, int kSTAGES, int kQBUF, int kEPI>
__global__ void __launch_bounds__((2 + kEPI) * 32, 1)
    score_bf16_kernel(const __grid_constant__ CUtensorMap tmap_k,
                      const __grid_constant__ CUtensorMap tmap_q,
                      const ScoreParams p) {
  static_assert(kEPI == 4 || kEPI == 8, "epilogue warps");
  static_assert(kH == 64 || kEPI == 4, "generic epilogue uses 4 warps");
  constexpr int kGroups = kEPI / 4;
  extern __shared__ uint8_t smem_raw[];
  uint8_t *smem = reinterpret_cast<uint8_t *>(
      (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  const ScoreSmem L(kSTAGES, kQBUF, kNSUB, p.n_cols, false);
  uint8_t *sk = smem + L.off_k;
  uint8_t *sq = smem + L.off_q;
  uint64_t *bars = reinterpret_cast<uint64_t *>(smem + L.off_bar);
  uint64_t *full_k = bars;                       // [kSTAGES]
  uint64_t *empty_k = full_k + kSTAGES;          // [kSTAGES]
  uint64_t *q_full = empty_k + kSTAGES;          // [kQBUF]
  uint64_t *q_empty = q_full + kQBUF;            // [kQBUF]
  uint64_t *acc_full = q_empty + kQBUF;          // [kNACC]
  uint64_t *acc_empty = acc_full + kNACC;        // [kNACC]
  uint64_t *sched_full = acc_empty + kNACC;      // [kSchedSlots]
  uint64_t *sched_empty = sched_full + kSchedSlots;
  uint32_t *misc = reinterpret_cast<uint32_t *>(smem + L.off_misc);
  uint32_t *tmem_base_slot = misc;               // written by tcgen05.alloc
  volatile int *abort_flag = reinterpret_cast<volatile int *>(misc + 1);
  uint32_t *sched_unit = misc + 4;               // [kSchedSlots]

  const int warp = threadIdx.x / 32;
  const int lane = threadIdx.x % 32;
  const int tq_total = p.tq_sub * kNSUB;
  const int n_cols = p.n_cols;
  const uint32_t tmem_cols_needed = kNACC * n_cols;
  uint32_t tmem_cols = 32;
  while (tmem_cols < tmem_cols_needed) tmem_cols <<= 1;

  if (threadIdx.x == 0) {
    for (int i = 0; i < kSTAGES; ++i) { mbar_init(full_k + i, 1); mbar_init(empty_k + i, 1); }
    for (int i = 0; i < kQBUF; ++i) { mbar_init(q_full + i, 1); mbar_init(q_empty + i, 1); }
    for (int i = 0; i < kNACC; ++i) { mbar_init(acc_full + i, 1); mbar_init(acc_empty + i, kEPI); }
    for (int i = 0; i < kSchedSlots; ++i) {
      mbar_init(sched_full + i, 1);
      mbar_init(sched_empty + i, 1 + kEPI);
    }
    *abort_flag = 0;
    fence_mbar_init();
    tma_prefetch_desc(&tmap_k);
    tma_prefetch_desc(&tmap_q);
  }
  if (warp == 1) {
    tmem_alloc(tmem_base_slot, tmem_cols);
    tmem_relinquish();
  }
  tc_fence_before_sync();
  __syncthreads();
  tc_fence_after_sync();
  const uint32_t tmem_base = *tmem_base_slot;
  const WaitCtl ctl{abort_flag, p.err, p.err_info, p.wait_limit_ns};

  if (warp == 0) {
    // ---------------- scheduler + TMA producer ----------------
    if (lane == 0) {
      Ring st, qb, sc;
      uint32_t k_issued = 0, q_issued = 0;   // bitmasks: stage / buffer used
      uint32_t k_last_phase = 0, q_last_phase = 0;
      for (;;) {
        const uint32_t u = atomicAdd(p.sched_counter, 1u);
        if (!mbar_wait(sched_empty + sc.idx, sc.phase ^ 1u, ctl, 1)) break;
        sched_unit[sc.idx] = u;
        mbar_arrive(sched_full + sc.idx);
        sc.next(kSchedSlots);
        Unit U;
        if (!decode_unit(p, tq_total, u, U)) break;
        if (U.j_act == U.j0) continue;
        const int nsub = (U.ntok + p.tq_sub - 1) / p.tq_sub;
        if (!mbar_wait(q_empty + qb.idx, qb.phase ^ 1u, ctl, 2)) break;
        mbar_arrive_expect_tx(q_full + qb.idx, nsub * L.q_sub_bytes);
        for (int s = 0; s < nsub; ++s) {
          uint8_t *dst = sq + (qb.idx * kNSUB + s) * L.q_sub_bytes;
          const int row = (U.t0 + s * p.tq_sub) * p.H;
          tma_load_2d(dst, &tmap_q, q_full + qb.idx, 0, row);
          tma_load_2d(dst + n_cols * 128, &tmap_q, q_full + qb.idx, 64, row);
        }
        q_issued |= 1u << qb.idx;
        q_last_phase = (q_last_phase & ~(1u << qb.idx)) | (qb.phase << qb.idx);
        qb.next(kQBUF);
        bool ok = true;
        for (int j = U.j0; j < U.j_act; ++j) {
          if (!mbar_wait(empty_k + st.idx, st.phase ^ 1u, ctl, 3)) { ok = false; break; }
          mbar_arrive_expect_tx(full_k + st.idx, L.k_stage_bytes);
          uint8_t *dst = sk + st.idx * L.k_stage_bytes;
          tma_load_3d(dst, &tmap_k, full_k + st.idx, 0, U.y0 + j * kBlockM, U.z);
          tma_load_3d(dst + kBlockM * 128, &tmap_k, full_k + st.idx, 64,
                      U.y0 + j * kBlockM, U.z);
          k_issued |= 1u << st.idx;
          k_last_phase = (k_last_phase & ~(1u << st.idx)) | (st.phase << st.idx);
          st.next(kSTAGES);
        }
        if (!ok) break;
      }
      // Let every copy this thread started land before the CTA can exit.
      for (int i = 0; i < kSTAGES; ++i)
        if (k_issued >> i & 1u) mbar_drain(full_k + i, k_last_phase >> i & 1u, p.wait_limit_ns);
      for (int i = 0; i < kQBUF; ++i)
        if (q_issued >> i & 1u) mbar_drain(q_full + i, q_last_phase >> i & 1u, p.wait_limit_ns);
    }
  } else if (warp == 1) {
    // ---------------- MMA issuer ----------------
    if (lane == 0) {
      const uint32_t idesc = idesc_bf16_f32(kBlockM, n_cols);
      Ring st, qb, ac, sc;
      uint64_t *last_commit = nullptr;
      uint32_t last_commit_phase = 0;
      for (;;) {
        if (!mbar_wait(sched_full + sc.idx, sc.phase, ctl, 11)) break;
        const uint32_t u = sched_unit[sc.idx];
        mbar_arrive(sched_empty + sc.idx);
        sc.next(kSchedSlots);
        Unit U;
        if (!decode_unit(p, tq_total, u, U)) break;
        if (U.j_act == U.j0) continue;
        const int nsub = (U.ntok + p.tq_sub - 1) / p.tq_sub;
        if (!mbar_wait(q_full + qb.idx, qb.phase, ctl, 12)) break;
        tc_fence_after_sync();
        const uint32_t q_base = smem_u32(sq + qb.idx * kNSUB * L.q_sub_bytes);
        bool ok = true;
        for (int j = U.j0; j < U.j_act && ok; ++j) {
          if (!mbar_wait(full_k + st.idx, st.phase, ctl, 13)) { ok = false; break; }
          tc_fence_after_sync();
          const uint32_t k_base = smem_u32(sk + st.idx * L.k_stage_bytes);
          for (int s = 0; s < nsub; ++s) {
            if (!mbar_wait(acc_empty + ac.idx, ac.phase ^ 1u, ctl, 14)) { ok = false; break; }
            tc_fence_after_sync();
            const uint32_t d_tmem = tmem_base + ac.idx * n_cols;
            const uint32_t qs = q_base + s * L.q_sub_bytes;
#pragma unroll
            for (int kk = 0; kk < kHeadDim / 16; ++kk) {
              const uint32_t half = kk / 4, koff = (kk % 4) * 32;
              const uint64_t ad = sdesc_kmajor_sw128(k_base + half * (kBlockM * 128) + koff);
              const uint64_t bd = sdesc_kmajor_sw128(qs + half * (n_cols * 128) + koff);
              mma_f16_ss(d_tmem, ad, bd, idesc, kk > 0 ? 1u : 0u);
            }
            mma_commit(acc_full + ac.idx);
            last_commit = acc_full + ac.idx;
            last_commit_phase = ac.phase;
            ac.next(kNACC);
          }
          if (!ok) break;
          mma_commit(empty_k + st.idx);      // stage free once these MMAs finish
          st.next(kSTAGES);
        }
        if (!ok) break;
        mma_commit(q_empty + qb.idx);
        qb.next(kQBUF);
      }
      // MMAs still in flight must finish before TMEM is released.
      if (last_commit) mbar_drain(last_commit, last_commit_phase, p.wait_limit_ns);
    }
  } else {
    // ---------------- epilogue ----------------
    const int epi = warp - 2;                  // 0 .. kEPI-1
    const int quad = warp & 3;                 // TMEM lane quadrant of this warp
    const int group = epi / 4;                 // token subset of this warp
    const uint32_t lane_addr = static_cast<uint32_t>(quad * 32) << 16;
    Ring ac, sc;
    for (;;) {
      if (!mbar_wait(sched_full + sc.idx, sc.phase, ctl, 21)) break;
      const uint32_t u = sched_unit[sc.idx];
      __syncwarp();
      if (lane == 0) mbar_arrive(sched_empty + sc.idx);
      sc.next(kSchedSlots);
      Unit U;
      if (!decode_unit(p, tq_total, u, U)) break;
      const int nsub = (U.ntok + p.tq_sub - 1) / p.tq_sub;
      bool ok = true;
      for (int j = U.j0; j < U.j1 && ok; ++j) {
        const int64_t slot = static_cast<int64_t>(j) * kBlockM + quad * 32 + lane;
        const bool in_row = slot < U.row_len;
        if (j >= U.j_act) {
          // every token of the unit is masked on this whole tile
          if (in_row)
            for (int i = group; i < U.ntok; i += kGroups)
              p.scores[U.out0 + i * U.row_len + slot] = kMaskBound;
          continue;
        }
        for (int s = 0; s < nsub; ++s) {
          if (!mbar_wait(acc_full + ac.idx, ac.phase, ctl, 22)) { ok = false; break; }
          tc_fence_after_sync();
          const uint32_t tbase = tmem_base + lane_addr + ac.idx * n_cols;
          const int i0 = s * p.tq_sub;
          const int ntok_s = min(p.tq_sub, U.ntok - i0);
          if constexpr (kH == 64) {
            for (int i = group; i < ntok_s; i += kGroups) {
              const int t = U.t0 + i0 + i;
              const float acc = head_sum_h64(tbase + i * 64, p.w + static_cast<int64_t>(t) * 64);
              const int lv = unit_last_valid(p, U, i0 + i);
              if (in_row)
                p.scores[U.out0 + (i0 + i) * U.row_len + slot] = slot <= lv ? acc : kMaskBound;
            }
          } else {
            // any H: walk the sub-block's columns in 16-wide chunks
            const int H = p.H, ncols = ntok_s * H;
            const float *wsub = p.w + static_cast<int64_t>(U.t0 + i0) * H;
            float acc = 0.f;
            int tok = 0, h = 0;
            for (int c0 = 0; c0 < ncols; c0 += 16) {
              float v[16];
              tmem_ld16_wait(tbase + c0, v);
#pragma unroll
              for (int c = 0; c < 16; ++c) {
                if (c0 + c < ncols) {
                  acc = fmaf(__ldg(wsub + c0 + c), fmaxf(v[c], 0.f), acc);
                  if (++h == H) {
                    const int lv = unit_last_valid(p, U, i0 + tok);
                    if (in_row)
                      p.scores[U.out0 + (i0 + tok) * U.row_len + slot] =
                          slot <= lv ? acc : kMaskBound;
                    acc = 0.f; h = 0; ++tok;
                  }
                }
              }
            }
          }
          tc_fence_before_sync();
          __syncwarp();
          if (lane == 0) mbar_arrive(acc_empty + ac.idx);
          ac.next(kNACC);
        }
      }
      if (!ok) break;
    }
  }

  tc_fence_before_sync();
  __syncthreads();
  tc_fence_after_sync();
  if (warp == 1) tmem_dealloc(tmem_base, tmem_cols);
  // The last CTA to finish leaves the scheduler counters at zero for the
  // next launch on this workspace (every fetch of this launch is done).
  if (threadIdx.x == 0) {
    __threadfence();
    if (atomicAdd(p.done_counter, 1u) == gridDim.x - 1) {
      atomicExch(p.sched_counter, 0u);
      atomicExch(p.done_counter, 0u);
      __threadfence();
    }
  }
}

}  // namespace dsa
