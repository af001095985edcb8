// sparse_mqa.cuh -- sparse multi-query attention over top-k key indices, the
// consumer of the lightning indexer, for sm_100a.
//
// For every query token t (batch b = t / S_per_batch) and head h:
//   l_j = sm_scale * q[t,h,:] . kv[b, idx[t,j], :]   for the kept entries j
//   out[t,h,:] = sum_j e^{l_j} kv[b, idx[t,j], :] / (sum_j e^{l_j} + e^{sinks[h]})
// An index of -1, or outside [0, K), masks its entry; a token with no kept
// entry gets out = 0. (NeMo AutoModel optimized_kernels, sparse_attention_torch
// and dense_attention_topk_torch: q [B,S,H,D], one kv head [B,K,D] that is both
// key and value, sinks [H], topk_idxs [B,S,K_top] with -1 masking an entry; the
// DeepSeek-V4 inference kernel write-up, sparse attention section: keys
// gathered by index, masked entries scored -inf, an online softmax whose
// denominator gains exp(sink - max) at the end.)
//
// One work item = one token and a contiguous range of its index row (all of
// it, or 1/nsplit of it when there are too few tokens to fill the GPU; a
// second kernel then merges the ranges). Persistent CTAs, one per SM, walk
// the items. Per tile of 128 index entries:
//   producer warp 5     : lane l gathers the tile's rows 4l .. 4l+3 with TMA
//                         tile::gather4 loads (four 128-byte row halves an
//                         instruction, two a lane) into a 128-byte-swizzled
//                         K-major tile; a masked entry reads a row past the
//                         tensor, which TMA fills with zeros; lane 0 publishes
//                         the tile's validity bits;
//   MMA warp 4          : S = Q K^T  (M = 128 head rows, N = 128 keys, K = D)
//                         into one of two TMEM score buffers, then
//                         O += P V    (M = 128 head rows, N = D, K = 128 keys)
//                         with V read MN-major from the same gathered tile;
//   softmax warps 0..3  : one thread per head row: the row's 128 logits from
//                         TMEM, the running max, P = 2^(x - max) as bf16 into
//                         shared memory, the running sum; O in TMEM is rescaled
//                         only when the max grows by more than 2^8 (P stays
//                         <= 256, exact in the final division either way).
// The epilogue divides O by (sum + 2^(sink - max)) and stores bf16 rows.
#pragma once

#include <cstdint>

#include <cuda_bf16.h>

#include "sm100_ptx.cuh"

namespace dsa {

constexpr int kMqaD = 128;               // head dim (the indexer's)
constexpr int kMqaTile = 128;            // index entries per tile
constexpr int kMqaStages = 3;            // gathered kv tiles in flight
constexpr int kMqaSoftmaxWarps = 4;
constexpr int kMqaProducerWarps = 1;        // four key rows a lane (TMA gathers)
constexpr int kMqaMmaWarp = 4;
constexpr int kMqaThreads = (kMqaSoftmaxWarps + 1 + kMqaProducerWarps) * 32;   // 192
constexpr float kMqaLazyRescale = 8.f;   // log2 units: rescale O when the max grows by more
constexpr float kLog2e = 1.4426950408889634f;

struct MqaParams {
  int T, H, S_per_batch;     // query tokens (B * S), heads, tokens per batch
  int64_t K;                 // kv rows per batch
  int K_top;                 // index entries per token
  int nsplit, chunk;         // ranges per token, entries per range (multiple of 128)
  const uint16_t *kv;        // [B, K, D] bf16
  const int *idx;            // [T, K_top]
  const float *sinks;        // [H]
  float scale_log2;          // sm_scale * log2(e)
  uint16_t *out;             // [T, H, D] bf16
  float *part_o;             // nsplit > 1: [T, nsplit, H, D] unnormalised
  float *part_ml;            // nsplit > 1: [T, nsplit, H, 2] (max in log2 units, sum)
  unsigned int *err;
  unsigned int *err_info;
  uint64_t wait_limit_ns;
  uint64_t drain_limit_ns;
};

struct MqaSmem {
  static constexpr uint32_t kTileBytes = kMqaTile * kMqaD * 2;   // two 128-byte-wide halves
  static constexpr uint32_t off_k = 0;
  static constexpr uint32_t off_q = off_k + kMqaStages * kTileBytes;
  static constexpr uint32_t off_p = off_q + kTileBytes;
  static constexpr uint32_t off_mask = off_p + 2 * kTileBytes;
  static constexpr uint32_t off_bar = off_mask + kMqaStages * 16;
  static constexpr uint32_t off_misc = off_bar + 32 * 8;
  static constexpr uint32_t total = off_misc + 64 + 1024;        // + alignment slack
};

// Byte offset of 16-byte chunk c (0..15 along the 128 columns) of row r in a
// [128 x 128] bf16 tile stored as two [128 x 64] halves with the 128-byte
// swizzle (chunk c of a half at (c ^ (r & 7)) within the row).
__device__ __forceinline__ uint32_t mqa_sw128(int r, int c) {
  return static_cast<uint32_t>((c >> 3) * 16384 + r * 128 + (((c & 7) ^ (r & 7)) << 4));
}

// Item n: token t, and its index entries [k0, k1).
__device__ __forceinline__ void mqa_item(const MqaParams &p, int n, int &t, int &k0, int &k1,
                                         int &ntiles) {
  t = n / p.nsplit;
  const int c = n - t * p.nsplit;
  k0 = c * p.chunk;
  k1 = min(p.K_top, k0 + p.chunk);
  ntiles = k1 > k0 ? (k1 - k0 + kMqaTile - 1) / kMqaTile : 1;   // >= 1: uniform protocol
}

__global__ void __launch_bounds__(kMqaThreads, 1)
    sparse_mqa_kernel(const __grid_constant__ CUtensorMap tmap_q,
                      const __grid_constant__ CUtensorMap tmap_kv, const MqaParams p) {
  extern __shared__ uint8_t smem_raw[];
  // 1024-byte aligned, by pointer arithmetic on the shared array, so that
  // the compiler keeps every access through it in the shared address space
  uint8_t *smem = smem_raw + ((1024u - (smem_u32(smem_raw) & 1023u)) & 1023u);
  uint8_t *sk = smem + MqaSmem::off_k;
  uint8_t *sq = smem + MqaSmem::off_q;
  uint8_t *sp = smem + MqaSmem::off_p;
  uint32_t *smask = reinterpret_cast<uint32_t *>(smem + MqaSmem::off_mask);
  uint64_t *bars = reinterpret_cast<uint64_t *>(smem + MqaSmem::off_bar);
  uint64_t *full = bars;                       // [stages] TMA bytes (lane 0 expects them)
  uint64_t *empty = full + kMqaStages;         // [stages] MMA commit after P V
  uint64_t *q_full = empty + kMqaStages;       // TMA bytes
  uint64_t *q_empty = q_full + 1;              // MMA commit after the item's last Q K^T
  uint64_t *s_full = q_empty + 1;              // [2] MMA commit
  uint64_t *s_empty = s_full + 2;              // [2] softmax warps (4)
  uint64_t *p_full = s_empty + 2;              // [2] softmax warps (4)
  uint64_t *pv_done = p_full + 2;              // [2] MMA commit
  uint64_t *o_free = pv_done + 2;              // softmax warps (4): O read by the epilogue
  uint32_t *misc = reinterpret_cast<uint32_t *>(smem + MqaSmem::off_misc);
  uint32_t *tmem_slot = misc;
  volatile int *abort_flag = reinterpret_cast<volatile int *>(misc + 1);

  const int tid = threadIdx.x;
  const int warp = tid >> 5, lane = tid & 31;
  const int H = p.H;

  if (warp == kMqaMmaWarp) {
    tmem_alloc(tmem_slot, 512);
    tmem_relinquish();
  }
  if (tid == 0) {
    for (int i = 0; i < kMqaStages; ++i) {
      mbar_init(full + i, 1);
      mbar_init(empty + i, 1);
    }
    mbar_init(q_full, 1);
    mbar_init(q_empty, 1);
    for (int i = 0; i < 2; ++i) {
      mbar_init(s_full + i, 1);
      mbar_init(s_empty + i, kMqaSoftmaxWarps);
      mbar_init(p_full + i, kMqaSoftmaxWarps);
      mbar_init(pv_done + i, 1);
    }
    mbar_init(o_free, kMqaSoftmaxWarps);
    *abort_flag = 0;
    fence_mbar_init();
    tma_prefetch_desc(&tmap_q);
    tma_prefetch_desc(&tmap_kv);
  }
  if (warp > kMqaMmaWarp) {
    // head rows H..127 of the query tile stay zero (TMA fills rows 0..H-1)
    for (int r = tid - (kMqaMmaWarp + 1) * 32; r < 128; r += kMqaProducerWarps * 32)
      if (r >= H)
        for (int c = 0; c < 16; ++c) *reinterpret_cast<uint4 *>(sq + mqa_sw128(r, c)) = uint4{};
    fence_proxy_async_smem();
  }
  grid_dep_wait();                 // q, kv, idx may come from earlier work on the stream
  grid_dep_launch_dependents();
  tc_fence_before_sync();
  __syncthreads();
  tc_fence_after_sync();
  const uint32_t tmem = *tmem_slot;
  const WaitCtl ctl{abort_flag, p.err, p.err_info, p.wait_limit_ns};
  const int nitems = p.T * p.nsplit;

  if (warp > kMqaMmaWarp) {
    // ---------------- producer: gather the selected kv rows ----------------
    const int pt = tid - (kMqaMmaWarp + 1) * 32;       // lane: tile rows 4pt .. 4pt+3
    const int32_t oob_row = static_cast<int32_t>(static_cast<int64_t>(p.T / p.S_per_batch) * p.K);
    uint32_t g = 0, qn = 0;
    bool q_issued = false, k_issued = false;
    uint32_t q_phase = 0, k_last_phase = 0;
    uint32_t k_issued_mask = 0;
    bool ok = true;
    for (int n = blockIdx.x; n < nitems && ok; n += gridDim.x, ++qn) {
      int t, k0, k1, nt;
      mqa_item(p, n, t, k0, k1, nt);
      if (pt == 0) {
        if (!mbar_wait(q_empty, (qn & 1u) ^ 1u, ctl, 40)) { ok = false; }
        if (ok) {
          mbar_arrive_expect_tx(q_full, static_cast<uint32_t>(2 * H * 128));
          tma_load_2d(sq, &tmap_q, q_full, 0, t * H);
          tma_load_2d(sq + 16384, &tmap_q, q_full, 64, t * H);
          q_issued = true;
          q_phase = qn & 1u;
        }
      }
      ok = __shfl_sync(0xffffffffu, ok, 0) && !*abort_flag;
      if (!ok) break;
      const int64_t rb = static_cast<int64_t>(t / p.S_per_batch) * p.K;   // batch's first row
      const int *irow = p.idx + static_cast<int64_t>(t) * p.K_top;
      for (int j = 0; j < nt; ++j, ++g) {
        const uint32_t st = g % kMqaStages;
        if (!mbar_wait(empty + st, ((g / kMqaStages) & 1u) ^ 1u, ctl, 41)) { ok = false; break; }
        int32_t y[4];
        uint32_t nib = 0;                               // validity of rows 4pt .. 4pt+3
#pragma unroll
        for (int q = 0; q < 4; ++q) {
          const int key = k0 + j * kMqaTile + 4 * pt + q;
          const int row = key < k1 ? __ldg(irow + key) : -1;
          const bool valid = row >= 0 && row < p.K;
          y[q] = valid ? static_cast<int32_t>(rb + row) : oob_row;
          nib |= static_cast<uint32_t>(valid) << q;
        }
        // validity words: slot 4l + q of the tile is bit (4l + q) % 32 of word l / 8
        uint32_t word = nib << (4 * (pt & 7));
#pragma unroll
        for (int off = 1; off < 8; off <<= 1) word |= __shfl_xor_sync(0xffffffffu, word, off);
        if ((pt & 7) == 0) smask[st * 4 + pt / 8] = word;
        __syncwarp();
        if (pt == 0) mbar_arrive_expect_tx(full + st, MqaSmem::kTileBytes);
        __syncwarp();
        uint8_t *dst = sk + st * MqaSmem::kTileBytes + 4 * pt * 128;
        tma_gather4(dst, &tmap_kv, full + st, 0, y[0], y[1], y[2], y[3]);
        tma_gather4(dst + 16384, &tmap_kv, full + st, 64, y[0], y[1], y[2], y[3]);
        k_issued = true;
        k_issued_mask |= 1u << st;
        k_last_phase = (k_last_phase & ~(1u << st)) | (((g / kMqaStages) & 1u) << st);
      }
    }
    // every copy started here lands before the CTA can exit
    if (pt == 0 && q_issued) mbar_drain(q_full, q_phase, p.drain_limit_ns);
    if (pt == 0 && k_issued)
      for (int i = 0; i < kMqaStages; ++i)
        if (k_issued_mask >> i & 1u) mbar_drain(full + i, k_last_phase >> i & 1u, p.drain_limit_ns);
    __syncwarp();
  } else if (warp == kMqaMmaWarp) {
    // ---------------- MMA issuer ----------------
    const uint32_t idesc_s = idesc_bf16_f32(128, 128);
    const uint32_t idesc_o = idesc_bf16_f32_bmn(128, kMqaD);
    const uint64_t q_desc = sdesc_kmajor_sw128(smem_u32(sq));
    uint64_t *last_commit = nullptr;
    uint32_t last_phase = 0;
    uint32_t g = 0, qn = 0;
    bool ok = true;
    // O += P V for global tile gp (first: the item's first tile, O starts over)
    auto issue_pv = [&](uint32_t gp, bool first, uint32_t item) -> bool {
      const uint32_t pb = gp & 1u;
      if (!mbar_wait(p_full + pb, (gp >> 1) & 1u, ctl, 42)) return false;
      if (first && item > 0 && !mbar_wait(o_free, (item - 1) & 1u, ctl, 43)) return false;
      tc_fence_after_sync();
      if (lane == 0) {
        const uint32_t st = gp % kMqaStages;
        const uint64_t p_desc = sdesc_kmajor_sw128(smem_u32(sp + pb * MqaSmem::kTileBytes));
        const uint32_t v_base = smem_u32(sk + st * MqaSmem::kTileBytes);
#pragma unroll
        for (int kk = 0; kk < kMqaTile / 16; ++kk) {
          const uint32_t half = kk / 4, koff = (kk % 4) * 2;
          const uint64_t adesc = p_desc + half * (16384 >> 4) + koff;
          // V: 16 keys = two 8-row atoms further along K; D halves 16 KB apart
          const uint64_t bdesc = sdesc_mnmajor_sw128(v_base + kk * 2048, 16384, 1024);
          mma_f16_ss(tmem + 256, adesc, bdesc, idesc_o, (first && kk == 0) ? 0u : 1u);
        }
        mma_commit(pv_done + pb);
        mma_commit(empty + st);
        last_commit = pv_done + pb;
        last_phase = (gp >> 1) & 1u;
      }
      __syncwarp();
      return true;
    };
    for (int n = blockIdx.x; n < nitems && ok; n += gridDim.x, ++qn) {
      int t, k0, k1, nt;
      mqa_item(p, n, t, k0, k1, nt);
      if (!mbar_wait(q_full, qn & 1u, ctl, 44)) break;
      tc_fence_after_sync();
      for (int j = 0; j < nt; ++j) {
        const uint32_t gj = g + j;
        const uint32_t st = gj % kMqaStages, sb = gj & 1u;
        if (!mbar_wait(full + st, (gj / kMqaStages) & 1u, ctl, 45) ||
            !mbar_wait(s_empty + sb, ((gj >> 1) & 1u) ^ 1u, ctl, 46)) {
          ok = false;
          break;
        }
        tc_fence_after_sync();
        if (lane == 0) {
          const uint64_t k_desc = sdesc_kmajor_sw128(smem_u32(sk + st * MqaSmem::kTileBytes));
#pragma unroll
          for (int kk = 0; kk < kMqaD / 16; ++kk) {
            const uint32_t half = kk / 4, koff = (kk % 4) * 2;
            mma_f16_ss(tmem + sb * 128, q_desc + half * (16384 >> 4) + koff,
                       k_desc + half * (16384 >> 4) + koff, idesc_s, kk > 0 ? 1u : 0u);
          }
          mma_commit(s_full + sb);
          if (j == nt - 1) mma_commit(q_empty);     // Q free once these MMAs finish
          last_commit = s_full + sb;
          last_phase = (gj >> 1) & 1u;
        }
        __syncwarp();
        if (j >= 1 && !issue_pv(gj - 1, j == 1, qn)) { ok = false; break; }
      }
      if (!ok || !issue_pv(g + nt - 1, nt == 1, qn)) break;
      g += nt;
    }
    if (lane == 0 && last_commit) mbar_drain(last_commit, last_phase, p.drain_limit_ns);
    __syncwarp();
  } else {
    // ---------------- softmax and epilogue: thread = head row ----------------
    const int h = tid;                               // TMEM lane = head row
    const uint32_t lane_base = static_cast<uint32_t>(warp * 32) << 16;
    const float sink2 = h < H ? __ldg(p.sinks + h) * kLog2e : 0.f;
    const float neg_inf = -__int_as_float(0x7f800000);
    uint32_t g = 0, qn = 0;
    bool ok = true;
    for (int n = blockIdx.x; n < nitems && ok; n += gridDim.x, ++qn) {
      int t, k0, k1, nt;
      mqa_item(p, n, t, k0, k1, nt);
      float m_run = neg_inf, l_run = 0.f;
      for (int j = 0; j < nt; ++j, ++g) {
        const uint32_t sb = g & 1u, st = g % kMqaStages;
        if (!mbar_wait(s_full + sb, (g >> 1) & 1u, ctl, 47)) { ok = false; break; }
        tc_fence_after_sync();
        float s[128];
#pragma unroll
        for (int q4 = 0; q4 < 4; ++q4) {
          float (&v)[32] = *reinterpret_cast<float (*)[32]>(&s[32 * q4]);
          tmem_ld32_async(tmem + lane_base + sb * 128 + 32 * q4, v);
        }
#pragma unroll
        for (int q4 = 0; q4 < 4; ++q4)
          tmem_wait_ld32(*reinterpret_cast<float (*)[32]>(&s[32 * q4]));
        tc_fence_before_sync();
        __syncwarp();
        if (lane == 0) mbar_arrive(s_empty + sb);
        // the tile's validity bits (published with the gathered rows)
        if (!mbar_wait(full + st, (g / kMqaStages) & 1u, ctl, 48)) { ok = false; break; }
        uint32_t mw[4];
#pragma unroll
        for (int i = 0; i < 4; ++i) mw[i] = smask[st * 4 + i];
        float mt = neg_inf;
#pragma unroll
        for (int c = 0; c < 128; ++c) {
          const float x = (mw[c >> 5] >> (c & 31)) & 1u ? s[c] * p.scale_log2 : neg_inf;
          s[c] = x;
          mt = fmaxf(mt, x);
        }
        const float m_new = fmaxf(m_run, mt);
        const bool need = j > 0 && m_run != neg_inf && m_new > m_run + kMqaLazyRescale;
        if (__any_sync(0xffffffffu, need)) {
          // O holds sums up to the previous tile: wait for its P V, rescale
          const uint32_t gp = g - 1;
          if (!mbar_wait(pv_done + (gp & 1u), (gp >> 1) & 1u, ctl, 49)) { ok = false; break; }
          tc_fence_after_sync();
          const float alpha = m_run == neg_inf ? 0.f : ex2_approx(m_run - m_new);
#pragma unroll
          for (int q4 = 0; q4 < 4; ++q4) {
            float o[32];
            tmem_ld32_wait(tmem + lane_base + 256 + 32 * q4, o);
#pragma unroll
            for (int i = 0; i < 32; ++i) o[i] *= alpha;
            tmem_st32(tmem + lane_base + 256 + 32 * q4, o);
          }
          tmem_wait_st();
          l_run *= alpha;
          m_run = m_new;
        } else if (m_run == neg_inf) {
          m_run = m_new;
        }
        // P buffer g&1 is free once the P V of tile g-2 has finished
        if (g >= 2 && !mbar_wait(pv_done + (g & 1u), ((g - 2) >> 1) & 1u, ctl, 50)) {
          ok = false;
          break;
        }
        uint8_t *prow = sp + (g & 1u) * MqaSmem::kTileBytes;
        float lsum = 0.f;
#pragma unroll
        for (int c8 = 0; c8 < 16; ++c8) {
          uint32_t w[4];
#pragma unroll
          for (int i = 0; i < 4; ++i) {
            const float a = m_run == neg_inf ? 0.f : ex2_approx(s[8 * c8 + 2 * i] - m_run);
            const float b2 = m_run == neg_inf ? 0.f : ex2_approx(s[8 * c8 + 2 * i + 1] - m_run);
            lsum += a + b2;
            const __nv_bfloat162 pr = __floats2bfloat162_rn(a, b2);
            w[i] = *reinterpret_cast<const uint32_t *>(&pr);
          }
          *reinterpret_cast<uint4 *>(prow + mqa_sw128(h, c8)) = make_uint4(w[0], w[1], w[2], w[3]);
        }
        l_run += lsum;
        fence_proxy_async_smem();       // P is read by the MMA (async proxy)
        tc_fence_before_sync();
        __syncwarp();
        if (lane == 0) mbar_arrive(p_full + (g & 1u));
      }
      if (!ok) break;
      // ---- epilogue: O / (sum + 2^(sink - max)) ----
      const uint32_t gl = g - 1;
      if (!mbar_wait(pv_done + (gl & 1u), (gl >> 1) & 1u, ctl, 51)) break;
      tc_fence_after_sync();
      const int c_split = n - t * p.nsplit;
      const bool write = h < H;
      const int64_t row = static_cast<int64_t>(t) * H + h;
      float inv = 0.f;
      if (p.nsplit == 1 && l_run > 0.f) inv = 1.f / (l_run + ex2_approx(sink2 - m_run));
#pragma unroll
      for (int q4 = 0; q4 < 4; ++q4) {
        float o[32];
        __syncwarp();                 // the TMEM load is warp-collective
        tmem_ld32_wait(tmem + lane_base + 256 + 32 * q4, o);
        if (!write) {
          // rows past H hold no head
        } else if (p.nsplit == 1) {
          uint4 *dst = reinterpret_cast<uint4 *>(p.out + row * kMqaD + 32 * q4);
#pragma unroll
          for (int c8 = 0; c8 < 4; ++c8) {
            uint32_t w[4];
#pragma unroll
            for (int i = 0; i < 4; ++i) {
              const __nv_bfloat162 pr =
                  __floats2bfloat162_rn(o[8 * c8 + 2 * i] * inv, o[8 * c8 + 2 * i + 1] * inv);
              w[i] = *reinterpret_cast<const uint32_t *>(&pr);
            }
            dst[c8] = make_uint4(w[0], w[1], w[2], w[3]);
          }
        } else {
          float4 *dst = reinterpret_cast<float4 *>(
              p.part_o + ((static_cast<int64_t>(t) * p.nsplit + c_split) * H + h) * kMqaD +
              32 * q4);
#pragma unroll
          for (int i = 0; i < 8; ++i)
            dst[i] = make_float4(o[4 * i], o[4 * i + 1], o[4 * i + 2], o[4 * i + 3]);
        }
      }
      if (write && p.nsplit > 1) {
        float2 *ml = reinterpret_cast<float2 *>(p.part_ml) +
                     (static_cast<int64_t>(t) * p.nsplit + c_split) * H + h;
        *ml = make_float2(m_run, l_run);
      }
      tc_fence_before_sync();
      __syncwarp();
      if (lane == 0) mbar_arrive(o_free);
    }
  }

  tc_fence_before_sync();
  __syncthreads();
  tc_fence_after_sync();
  if (warp == kMqaMmaWarp) tmem_dealloc(tmem, 512);
}

// Merge of the nsplit ranges of each token: with M the largest range max,
//   out = sum_c 2^(m_c - M) O_c / (sum_c 2^(m_c - M) l_c + 2^(sink - M)),
// and out = 0 when no range kept an entry. One warp per (token, head): lane
// l merges columns 4l .. 4l+3; the ranges' (max, sum) pairs are read by the
// first nsplit lanes and shared by shuffles.
__global__ void __launch_bounds__(256) sparse_mqa_combine_kernel(const MqaParams p) {
  grid_dep_wait();
  grid_dep_launch_dependents();
  const int lane = threadIdx.x & 31;
  const int64_t wid = (static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x) >> 5;
  if (wid >= static_cast<int64_t>(p.T) * p.H) return;
  const int t = static_cast<int>(wid / p.H), h = static_cast<int>(wid % p.H);
  const float neg_inf = -__int_as_float(0x7f800000);
  const float2 *ml = reinterpret_cast<const float2 *>(p.part_ml) +
                     static_cast<int64_t>(t) * p.nsplit * p.H + h;
  float4 acc = make_float4(0.f, 0.f, 0.f, 0.f);
  float L = 0.f, M = neg_inf;
  for (int c0 = 0; c0 < p.nsplit; c0 += 32) {      // the ranges' maxima
    const int c = c0 + lane;
    const float m = c < p.nsplit ? ml[static_cast<int64_t>(c) * p.H].x : neg_inf;
    M = fmaxf(M, m);
  }
#pragma unroll
  for (int off = 16; off > 0; off >>= 1) M = fmaxf(M, __shfl_xor_sync(0xffffffffu, M, off));
  if (M != neg_inf) {
    for (int c0 = 0; c0 < p.nsplit; c0 += 32) {
      const int c = c0 + lane;
      float w = 0.f, l = 0.f;
      if (c < p.nsplit) {
        const float2 v = ml[static_cast<int64_t>(c) * p.H];
        w = v.x == neg_inf ? 0.f : ex2_approx(v.x - M);
        l = v.y;
      }
      L += w * l;
      const int n = min(32, p.nsplit - c0);
      for (int j = 0; j < n; ++j) {
        const float wj = __shfl_sync(0xffffffffu, w, j);
        const float4 o = reinterpret_cast<const float4 *>(
            p.part_o + ((static_cast<int64_t>(t) * p.nsplit + c0 + j) * p.H + h) * kMqaD)[lane];
        acc.x += wj * o.x;
        acc.y += wj * o.y;
        acc.z += wj * o.z;
        acc.w += wj * o.w;
      }
    }
  }
#pragma unroll
  for (int off = 16; off > 0; off >>= 1) L += __shfl_xor_sync(0xffffffffu, L, off);
  const float inv = L > 0.f ? 1.f / (L + ex2_approx(__ldg(p.sinks + h) * kLog2e - M)) : 0.f;
  const __nv_bfloat162 a = __floats2bfloat162_rn(acc.x * inv, acc.y * inv);
  const __nv_bfloat162 b = __floats2bfloat162_rn(acc.z * inv, acc.w * inv);
  uint2 w2;
  w2.x = *reinterpret_cast<const uint32_t *>(&a);
  w2.y = *reinterpret_cast<const uint32_t *>(&b);
  reinterpret_cast<uint2 *>(p.out + (static_cast<int64_t>(t) * p.H + h) * kMqaD)[lane] = w2;
}

}  // namespace dsa
