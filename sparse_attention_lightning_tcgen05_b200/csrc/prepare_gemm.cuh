// prepare_gemm.cuh -- the indexer's front end for sm_100a: the query, key and
// head-weight projections with their epilogues fused.
//
// Per query token t (DeepSeek-V3.2 Sparse Indexer Kernel API Reference,
// Parameters: qr, wq_b, hidden_states, wk, k_norm_weight / k_norm_bias,
// weights_proj, cos / sin, key_cache written in place at positions; tokamax
// Supported Ops, deepseek_rope: interleaved RoPE):
//   q[t, h, :] = rope(qr[t] . wq_b[h*D .. h*D+D-1, :]^T)            bf16
//   k[t, :]    = rope(layernorm(x[t] . wk^T))  -> key cache row      bf16
//   w[t, :]    = w_scale * (x[t] . weights_proj^T)                   fp32
// rope rotates the interleaved pairs (2i, 2i+1) of the leading rope_dim
// features by the angle of cos/sin[t, i]; the Hadamard rotation is left out
// (the bf16 score path's reading: it cancels in q . k).
//
// One GEMM kernel, C[tokens, features] = A[tokens, K] . B[features, K]^T, bf16
// in, fp32 accumulators in TMEM, both operands K-major and fed by TMA:
//   mode Q : A = qr, B = wq_b; a feature tile is one head (128 columns);
//   mode KW: A = x, B = wk (128 rows) stacked over weights_proj (H rows) in
//            one tile of 128 + H columns.
// Work items (token tile of 128, feature tile, K range) run on persistent
// CTAs: warp 0 issues the TMA loads, warp 1 owns TMEM and issues the MMAs
// into two accumulator slots, warps 2..5 (one per TMEM lane quadrant, one
// thread per token row) run the epilogue. When a GEMM has too few tiles to
// fill the GPU (decode batches) its K range is split: each split writes fp32
// partial rows and a second kernel sums them and runs the same epilogue.
#pragma once

#include <cstdint>

#include <cuda_bf16.h>

#include "sm100_ptx.cuh"

namespace dsa {

enum : int { kPrepQ = 0, kPrepKW = 1 };

constexpr int kPrepD = 128;          // head dim
constexpr int kPrepBK = 64;          // K per stage (one 128-byte swizzle row of bf16)
constexpr int kPrepStages = 4;
constexpr int kPrepThreads = 192;    // producer, MMA, 4 epilogue warps

struct PrepParams {
  int mode;
  int T;                     // tokens (rows of A)
  int ksteps;                // K / 64
  int m_tiles, n_tiles, nsplit, per;   // tiles, K splits, K steps per split
  int BN, n1;                // columns per tile; columns of it from the first B map
  int N_total;               // columns of C (partial rows)
  int H, rope_dim;
  float eps, w_scale;
  const float *cos, *sin;    // [T, rope_dim / 2]
  const float *gain, *bias;  // [D]
  uint16_t *q_out;           // [T, H, D] bf16
  float *w_out;              // [T, H]
  uint16_t *k_cache;         // key rows at k_cache + t*k_seq_stride + pos*D
  int64_t k_seq_stride;
  int64_t S;                 // slots per cache: positions outside [0, S) write nothing
  const int *positions;      // NULL: token t at position t
  float *part;               // nsplit > 1: [nsplit, T, N_total]
  unsigned int *err;
  unsigned int *err_info;
  uint64_t wait_limit_ns;
  uint64_t drain_limit_ns;
};

struct PrepSmem {
  static constexpr uint32_t kABytes = 128 * kPrepBK * 2;        // 16 KB
  static constexpr uint32_t kBBytes = 256 * kPrepBK * 2;        // room for 256 rows
  static constexpr uint32_t off_a = 0;
  static constexpr uint32_t off_b = off_a + kPrepStages * kABytes;
  static constexpr uint32_t off_bar = off_b + kPrepStages * kBBytes;
  static constexpr uint32_t off_misc = off_bar + 16 * 8;
  static constexpr uint32_t total = off_misc + 64 + 1024;
};

__device__ __forceinline__ void prep_item(const PrepParams &p, int n, int &mt, int &nt, int &k0,
                                          int &k1) {
  const int sp = n % p.nsplit;
  const int tile = n / p.nsplit;
  nt = tile % p.n_tiles;
  mt = tile / p.n_tiles;
  k0 = sp * p.per;
  k1 = min(p.ksteps, k0 + p.per);
}

// ---- epilogue arithmetic on one row (shared by the fused and split paths) ----

// Interleaved RoPE on the pairs of columns [c0, c0 + n) of a row chunk v
// (c0 even): the pair (2i, 2i+1) turns by the angle of cos/sin[i].
template <int N>
__device__ __forceinline__ void rope_chunk(float (&v)[N], int c0, int rope_dim, const float *cosr,
                                           const float *sinr) {
#pragma unroll
  for (int j = 0; j < N; j += 2) {
    const int c = c0 + j;
    if (c < rope_dim) {
      const float cs = __ldg(cosr + c / 2), sn = __ldg(sinr + c / 2);
      const float a = v[j], b = v[j + 1];
      v[j] = a * cs - b * sn;
      v[j + 1] = a * sn + b * cs;
    }
  }
}

__device__ __forceinline__ uint32_t pack_bf16x2(float a, float b) {
  const __nv_bfloat162 h = __floats2bfloat162_rn(a, b);
  return *reinterpret_cast<const uint32_t *>(&h);
}

// Where token t's key row goes (nullptr: its position is outside the cache).
__device__ __forceinline__ uint16_t *prep_key_row(const PrepParams &p, int t) {
  const int64_t pos = p.positions ? __ldg(p.positions + t) : t;
  if (pos < 0 || pos >= p.S) return nullptr;
  return p.k_cache + static_cast<int64_t>(t) * p.k_seq_stride + pos * kPrepD;
}

__global__ void __launch_bounds__(kPrepThreads, 1)
    prep_gemm_kernel(const __grid_constant__ CUtensorMap tmap_a,
                     const __grid_constant__ CUtensorMap tmap_b1,
                     const __grid_constant__ CUtensorMap tmap_b2, const PrepParams p) {
  extern __shared__ uint8_t smem_raw[];
  // 1024-byte aligned, by pointer arithmetic on the shared array, so that
  // the compiler keeps every access through it in the shared address space
  uint8_t *smem = smem_raw + ((1024u - (smem_u32(smem_raw) & 1023u)) & 1023u);
  uint8_t *sa = smem + PrepSmem::off_a;
  uint8_t *sb = smem + PrepSmem::off_b;
  uint64_t *bars = reinterpret_cast<uint64_t *>(smem + PrepSmem::off_bar);
  uint64_t *full = bars;                       // [stages] TMA bytes
  uint64_t *empty = full + kPrepStages;        // [stages] MMA commit
  uint64_t *acc_full = empty + kPrepStages;    // [2] MMA commit
  uint64_t *acc_empty = acc_full + 2;          // [2] epilogue warps (4)
  uint32_t *misc = reinterpret_cast<uint32_t *>(smem + PrepSmem::off_misc);
  volatile int *abort_flag = reinterpret_cast<volatile int *>(misc + 1);
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int BN = p.BN;

  if (warp == 1) {
    tmem_alloc(misc, 512);
    tmem_relinquish();
  }
  if (threadIdx.x == 0) {
    for (int i = 0; i < kPrepStages; ++i) {
      mbar_init(full + i, 1);
      mbar_init(empty + i, 1);
    }
    for (int i = 0; i < 2; ++i) {
      mbar_init(acc_full + i, 1);
      mbar_init(acc_empty + i, 4);
    }
    *abort_flag = 0;
    fence_mbar_init();
    tma_prefetch_desc(&tmap_a);
    tma_prefetch_desc(&tmap_b1);
    if (p.mode == kPrepKW) tma_prefetch_desc(&tmap_b2);
  }
  grid_dep_wait();
  grid_dep_launch_dependents();
  tc_fence_before_sync();
  __syncthreads();
  tc_fence_after_sync();
  const uint32_t tmem = *misc;
  const WaitCtl ctl{abort_flag, p.err, p.err_info, p.wait_limit_ns};
  const int nitems = p.m_tiles * p.n_tiles * p.nsplit;

  if (warp == 0) {
    // ---------------- TMA producer ----------------
    if (lane == 0) {
      uint32_t g = 0;
      uint32_t issued = 0, last_phase = 0;
      const uint32_t tx = PrepSmem::kABytes + static_cast<uint32_t>(BN) * kPrepBK * 2;
      bool ok = true;
      for (int n = blockIdx.x; n < nitems && ok; n += gridDim.x) {
        int mt, nt, k0, k1;
        prep_item(p, n, mt, nt, k0, k1);
        for (int ks = k0; ks < k1; ++ks, ++g) {
          const uint32_t st = g % kPrepStages;
          if (!mbar_wait(empty + st, ((g / kPrepStages) & 1u) ^ 1u, ctl, 60)) { ok = false; break; }
          mbar_arrive_expect_tx(full + st, tx);
          tma_load_2d(sa + st * PrepSmem::kABytes, &tmap_a, full + st, ks * kPrepBK, mt * 128);
          uint8_t *b = sb + st * PrepSmem::kBBytes;
          tma_load_2d(b, &tmap_b1, full + st, ks * kPrepBK, nt * p.n1);
          if (p.mode == kPrepKW)
            tma_load_2d(b + p.n1 * 128, &tmap_b2, full + st, ks * kPrepBK, 0);
          issued |= 1u << st;
          last_phase = (last_phase & ~(1u << st)) | (((g / kPrepStages) & 1u) << st);
        }
      }
      for (int i = 0; i < kPrepStages; ++i)
        if (issued >> i & 1u) mbar_drain(full + i, last_phase >> i & 1u, p.drain_limit_ns);
    }
  } else if (warp == 1) {
    // ---------------- MMA issuer ----------------
    const uint32_t idesc = idesc_bf16_f32(128, static_cast<uint32_t>(BN));
    uint64_t *last = nullptr;
    uint32_t last_phase = 0;
    uint32_t g = 0, it = 0;
    bool ok = true;
    for (int n = blockIdx.x; n < nitems && ok; n += gridDim.x, ++it) {
      int mt, nt, k0, k1;
      prep_item(p, n, mt, nt, k0, k1);
      const uint32_t ab = it & 1u;
      if (!mbar_wait(acc_empty + ab, ((it >> 1) & 1u) ^ 1u, ctl, 61)) break;
      tc_fence_after_sync();
      for (int ks = k0; ks < k1; ++ks, ++g) {
        const uint32_t st = g % kPrepStages;
        if (!mbar_wait(full + st, (g / kPrepStages) & 1u, ctl, 62)) { ok = false; break; }
        tc_fence_after_sync();
        if (lane == 0) {
          const uint64_t ad = sdesc_kmajor_sw128(smem_u32(sa + st * PrepSmem::kABytes));
          const uint64_t bd = sdesc_kmajor_sw128(smem_u32(sb + st * PrepSmem::kBBytes));
#pragma unroll
          for (int kk = 0; kk < kPrepBK / 16; ++kk)
            mma_f16_ss(tmem + ab * 256, ad + kk * 2, bd + kk * 2, idesc,
                       (ks > k0 || kk > 0) ? 1u : 0u);
          mma_commit(empty + st);
        }
        __syncwarp();
      }
      if (!ok) break;
      if (lane == 0) {
        mma_commit(acc_full + ab);
        last = acc_full + ab;
        last_phase = (it >> 1) & 1u;
      }
      __syncwarp();
    }
    if (lane == 0 && last) mbar_drain(last, last_phase, p.drain_limit_ns);
    __syncwarp();
  } else {
    // ---------------- epilogue: one thread per token row ----------------
    const int quad = warp & 3;
    const uint32_t lane_addr = static_cast<uint32_t>(quad * 32) << 16;
    uint32_t it = 0;
    for (int n = blockIdx.x; n < nitems; n += gridDim.x, ++it) {
      int mt, nt, k0, k1;
      prep_item(p, n, mt, nt, k0, k1);
      const uint32_t ab = it & 1u;
      if (!mbar_wait(acc_full + ab, (it >> 1) & 1u, ctl, 63)) break;
      tc_fence_after_sync();
      const int t = mt * 128 + quad * 32 + lane;
      const bool row_ok = t < p.T;
      const uint32_t tb = tmem + lane_addr + ab * 256;
      if (p.nsplit > 1) {
        // partial row of this K range
        const int sp = n % p.nsplit;
        float *dst = p.part + (static_cast<int64_t>(sp) * p.T + t) * p.N_total + nt * BN;
        for (int c0 = 0; c0 < BN; c0 += 32) {
          float v[32];
          __syncwarp();
          tmem_ld32_wait(tb + c0, v);
          if (row_ok) {
            float4 *d4 = reinterpret_cast<float4 *>(dst + c0);
            const int nv = min(32, BN - c0) / 4;
#pragma unroll
            for (int i = 0; i < 8; ++i)
              if (i < nv) d4[i] = make_float4(v[4 * i], v[4 * i + 1], v[4 * i + 2], v[4 * i + 3]);
          }
        }
      } else if (p.mode == kPrepQ) {
        const float *cosr = p.cos + static_cast<int64_t>(t < p.T ? t : 0) * (p.rope_dim / 2);
        const float *sinr = p.sin + static_cast<int64_t>(t < p.T ? t : 0) * (p.rope_dim / 2);
        uint4 *dst = reinterpret_cast<uint4 *>(p.q_out + (static_cast<int64_t>(t) * p.H + nt) *
                                                             kPrepD);
#pragma unroll
        for (int c0 = 0; c0 < kPrepD; c0 += 32) {
          float v[32];
          __syncwarp();
          tmem_ld32_wait(tb + c0, v);
          if (row_ok) {
            rope_chunk(v, c0, p.rope_dim, cosr, sinr);
#pragma unroll
            for (int i = 0; i < 4; ++i)
              dst[c0 / 8 + i] = make_uint4(pack_bf16x2(v[8 * i], v[8 * i + 1]),
                                           pack_bf16x2(v[8 * i + 2], v[8 * i + 3]),
                                           pack_bf16x2(v[8 * i + 4], v[8 * i + 5]),
                                           pack_bf16x2(v[8 * i + 6], v[8 * i + 7]));
          }
        }
      } else {
        // the key: LayerNorm over the 128 features, RoPE, into the cache
        float a0[32], a1[32], a2[32], a3[32];
        __syncwarp();
        tmem_ld32_async(tb, a0);
        tmem_ld32_async(tb + 32, a1);
        tmem_ld32_async(tb + 64, a2);
        tmem_ld32_async(tb + 96, a3);
        tmem_wait_ld32(a0);
        tmem_wait_ld32(a1);
        tmem_wait_ld32(a2);
        tmem_wait_ld32(a3);
        float mean = 0.f;
#pragma unroll
        for (int c = 0; c < 32; ++c) mean += (a0[c] + a1[c]) + (a2[c] + a3[c]);
        mean *= 1.f / kPrepD;
        float var = 0.f;
#pragma unroll
        for (int c = 0; c < 32; ++c) {
          a0[c] -= mean;
          a1[c] -= mean;
          a2[c] -= mean;
          a3[c] -= mean;
          var += (a0[c] * a0[c] + a1[c] * a1[c]) + (a2[c] * a2[c] + a3[c] * a3[c]);
        }
        const float rstd = rsqrtf(var * (1.f / kPrepD) + p.eps);
        uint16_t *krow = row_ok ? prep_key_row(p, t) : nullptr;
        if (krow) {
          const float *cosr = p.cos + static_cast<int64_t>(t) * (p.rope_dim / 2);
          const float *sinr = p.sin + static_cast<int64_t>(t) * (p.rope_dim / 2);
          uint4 *dst = reinterpret_cast<uint4 *>(krow);
          auto finish = [&](float (&a)[32], int c0) {
#pragma unroll
            for (int c = 0; c < 32; ++c)
              a[c] = a[c] * rstd * __ldg(p.gain + c0 + c) + __ldg(p.bias + c0 + c);
            rope_chunk(a, c0, p.rope_dim, cosr, sinr);
#pragma unroll
            for (int i = 0; i < 4; ++i)
              dst[c0 / 8 + i] = make_uint4(pack_bf16x2(a[8 * i], a[8 * i + 1]),
                                           pack_bf16x2(a[8 * i + 2], a[8 * i + 3]),
                                           pack_bf16x2(a[8 * i + 4], a[8 * i + 5]),
                                           pack_bf16x2(a[8 * i + 6], a[8 * i + 7]));
          };
          finish(a0, 0);
          finish(a1, 32);
          finish(a2, 64);
          finish(a3, 96);
        }
        // the head weights: columns 128 .. 128 + H
        for (int c0 = 0; c0 < p.H; c0 += 32) {
          float v[32];
          __syncwarp();
          tmem_ld32_wait(tb + kPrepD + c0, v);
          if (row_ok) {
            float *wrow = p.w_out + static_cast<int64_t>(t) * p.H + c0;
            const int nv = min(32, p.H - c0);
#pragma unroll
            for (int i = 0; i < 32; ++i)
              if (i < nv) wrow[i] = v[i] * p.w_scale;
          }
        }
      }
      tc_fence_before_sync();
      __syncwarp();
      if (lane == 0) mbar_arrive(acc_empty + ab);
    }
  }

  tc_fence_before_sync();
  __syncthreads();
  tc_fence_after_sync();
  if (warp == 1) tmem_dealloc(tmem, 512);
}

// Sum of the K splits and the epilogue. One CTA per (token, feature tile);
// column c of the tile belongs to threads c + g * BNp (g < groups, BNp = BN
// rounded up to a warp): group g sums the splits g, g + groups, ... with four
// loads in flight, and group 0 adds the groups' sums. Then, for the columns:
//   mode Q : RoPE (the pair partner is the neighbouring lane), bf16 q;
//   mode KW: LayerNorm over the key's 128 columns (block reduction), RoPE,
//            the bf16 key row into the cache; the H head weights scaled.
__global__ void __launch_bounds__(1024) prep_reduce_kernel(const PrepParams p, int groups) {
  __shared__ float part_sum[1024];
  __shared__ float red[2][4];
  grid_dep_wait();
  grid_dep_launch_dependents();
  const int BNp = (p.BN + 31) & ~31;
  const int g = threadIdx.x / BNp, c = threadIdx.x % BNp;
  const int t = blockIdx.x / p.n_tiles, nt = blockIdx.x % p.n_tiles;
  float v = 0.f;
  if (c < p.BN && g < groups) {
    const float *src = p.part + static_cast<int64_t>(t) * p.N_total + nt * p.BN + c;
    const int64_t step = static_cast<int64_t>(p.T) * p.N_total;
    float s0 = 0.f, s1 = 0.f, s2 = 0.f, s3 = 0.f;
    int sp = g;
    for (; sp + 3 * groups < p.nsplit; sp += 4 * groups) {
      s0 += src[sp * step];
      s1 += src[(sp + groups) * step];
      s2 += src[(sp + 2 * groups) * step];
      s3 += src[(sp + 3 * groups) * step];
    }
    for (; sp < p.nsplit; sp += groups) s0 += src[sp * step];
    v = (s0 + s1) + (s2 + s3);
  }
  part_sum[threadIdx.x] = v;
  __syncthreads();
  if (g != 0) return;
  for (int k = 1; k < groups; ++k) v += part_sum[k * BNp + c];
  const float *cosr = p.cos + static_cast<int64_t>(t) * (p.rope_dim / 2);
  const float *sinr = p.sin + static_cast<int64_t>(t) * (p.rope_dim / 2);
  const int warp = c >> 5, lane = c & 31;
  // RoPE of the column pair (c & ~1, c | 1): the partner is the next lane over
  auto rope1 = [&](float x) {
    const float other = __shfl_xor_sync(0xffffffffu, x, 1);
    if (c >= p.rope_dim) return x;
    const float cs = __ldg(cosr + c / 2), sn = __ldg(sinr + c / 2);
    return (c & 1) ? other * sn + x * cs : x * cs - other * sn;
  };
  if (p.mode == kPrepQ) {                      // 128 columns, four full warps
    const float y = rope1(v);
    const __nv_bfloat16 b = __float2bfloat16_rn(y);
    p.q_out[(static_cast<int64_t>(t) * p.H + nt) * kPrepD + c] =
        *reinterpret_cast<const uint16_t *>(&b);
    return;
  }
  if (warp < kPrepD / 32) {                    // the key: warps 0..3
    float s = v;
#pragma unroll
    for (int off = 16; off > 0; off >>= 1) s += __shfl_xor_sync(0xffffffffu, s, off);
    if (lane == 0) red[0][warp] = s;
  }
  __syncthreads();
  const float mean = (red[0][0] + red[0][1] + red[0][2] + red[0][3]) * (1.f / kPrepD);
  if (warp < kPrepD / 32) {
    const float d = v - mean;
    float q = d * d;
#pragma unroll
    for (int off = 16; off > 0; off >>= 1) q += __shfl_xor_sync(0xffffffffu, q, off);
    if (lane == 0) red[1][warp] = q;
  }
  __syncthreads();
  if (warp < kPrepD / 32) {
    const float var = (red[1][0] + red[1][1] + red[1][2] + red[1][3]) * (1.f / kPrepD);
    const float y = rope1((v - mean) * rsqrtf(var + p.eps) * __ldg(p.gain + c) + __ldg(p.bias + c));
    uint16_t *krow = prep_key_row(p, t);
    if (krow) {
      const __nv_bfloat16 b = __float2bfloat16_rn(y);
      krow[c] = *reinterpret_cast<const uint16_t *>(&b);
    }
  } else if (c < kPrepD + p.H) {
    p.w_out[static_cast<int64_t>(t) * p.H + (c - kPrepD)] = v * p.w_scale;
  }
}

}  // namespace dsa
