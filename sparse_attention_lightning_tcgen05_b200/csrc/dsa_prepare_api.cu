// dsa_prepare_api.cu -- C ABI of the front end (operation, layouts and error
// rules in include/dsa_prepare.h): argument checks, the K splits, the TMA
// tensor maps and the launches of the two projection GEMMs.
#include <cuda.h>
#include <cuda_runtime.h>

#include <algorithm>
#include <cmath>
#include <cstdint>

#include "dsa_launch.h"
#include "dsa_prepare.h"
#include "prepare_gemm.cuh"

namespace dsa_host {
namespace {

constexpr uint64_t kPrepWaitLimitNs = 4000000000ull;
constexpr uint64_t kPrepDrainLimitNs = 4000000000ull;
constexpr int kSizingSms = 148;   // K splits are sized for a B200, from the descriptor alone

dsa_status_t check_prep_desc(const dsa_prepare_desc_t *d) {
  if (!d) return DSA_ERR_INVALID_ARG;
  if (d->T < 1 || d->H < 1 || d->hidden < 1 || d->q_lora_rank < 1 || d->S < 1)
    return DSA_ERR_INVALID_ARG;
  if (d->rope_dim < 0 || d->rope_dim % 2 != 0 || d->rope_dim > d->D) return DSA_ERR_INVALID_ARG;
  if (!(d->k_norm_eps >= 0.f) || !std::isfinite(d->k_norm_eps) || !std::isfinite(d->w_scale))
    return DSA_ERR_INVALID_ARG;
  if (d->k_seq_stride < 0 || (d->k_seq_stride != 0 &&
                              (d->k_seq_stride % 128 != 0 || d->k_seq_stride < d->S * 128)))
    return DSA_ERR_INVALID_ARG;
  if (d->D != 128) return DSA_ERR_UNSUPPORTED;
  if (d->H % 16 != 0 || d->H > 128) return DSA_ERR_UNSUPPORTED;
  if (d->hidden % 64 != 0 || d->q_lora_rank % 64 != 0) return DSA_ERR_UNSUPPORTED;
  if (static_cast<int64_t>(d->T) * d->H * 128 > INT32_MAX) return DSA_ERR_UNSUPPORTED;
  return DSA_OK;
}

struct Split {
  int m_tiles, n_tiles, ksteps, nsplit, per;
};

// K splits: the count that minimises (waves of items over the SMs) x (K steps
// an item runs + the fixed cost of an item, about 3 K steps), at most 32
// splits (the reduction sums them).
Split plan(int T, int n_tiles, int K) {
  Split s{};
  s.m_tiles = (T + 127) / 128;
  s.n_tiles = n_tiles;
  s.ksteps = K / dsa::kPrepBK;
  const int64_t tiles = static_cast<int64_t>(s.m_tiles) * n_tiles;
  int64_t best = -1;
  s.nsplit = 1;
  s.per = s.ksteps;
  for (int want = 1; want <= std::min(32, s.ksteps); ++want) {
    const int per = (s.ksteps + want - 1) / want;
    const int ns = (s.ksteps + per - 1) / per;
    const int64_t waves = (tiles * ns + kSizingSms - 1) / kSizingSms;
    const int64_t cost = waves * (per + 3);
    if (best < 0 || cost < best) {
      best = cost;
      s.nsplit = ns;
      s.per = per;
    }
  }
  return s;
}

size_t partial_bytes(const Split &s, int T, int n_total) {
  return s.nsplit > 1 ? static_cast<size_t>(s.nsplit) * T * n_total * 4 : 0;
}

size_t workspace_bytes_for(const dsa_prepare_desc_t *d) {
  const Split q = plan(d->T, d->H, d->q_lora_rank);
  const Split kw = plan(d->T, 1, d->hidden);
  return kWorkspaceHeader + std::max(partial_bytes(q, d->T, d->H * 128),
                                     partial_bytes(kw, d->T, 128 + d->H));
}

dsa_status_t map_rows(CUtensorMap *m, const void *base, int64_t rows, int64_t K, int box_rows) {
  const cuuint64_t dims[2] = {static_cast<cuuint64_t>(K), static_cast<cuuint64_t>(rows)};
  const cuuint64_t strides[1] = {static_cast<cuuint64_t>(K) * 2};
  const cuuint32_t box[2] = {static_cast<cuuint32_t>(dsa::kPrepBK),
                             static_cast<cuuint32_t>(box_rows)};
  return make_map(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, base, dims, strides, box);
}

dsa_status_t launch_gemm(DeviceInfo *dev, const CUtensorMap &a, const CUtensorMap &b1,
                         const CUtensorMap &b2, const dsa::PrepParams &p, cudaStream_t s) {
  const int items = p.m_tiles * p.n_tiles * p.nsplit;
  const int grid = std::min(items, dev->num_sms);
  if (launch_pdl(dsa::prep_gemm_kernel, grid, dsa::kPrepThreads,
                 static_cast<size_t>(dsa::PrepSmem::total), s, 0, a, b1, b2, p) != cudaSuccess)
    return DSA_ERR_CUDA;
  if (p.nsplit > 1) {
    // one CTA per (token, feature tile); up to 4 thread groups a column share
    // the splits
    const int bnp = (p.BN + 31) & ~31;
    const int groups = std::max(1, std::min({4, (p.nsplit + 7) / 8, 1024 / bnp}));
    if (launch_pdl(dsa::prep_reduce_kernel, p.T * p.n_tiles, groups * bnp, 0, s, 0, p,
                   groups) != cudaSuccess)
      return DSA_ERR_CUDA;
  }
  return DSA_OK;
}

}  // namespace
}  // namespace dsa_host

using namespace dsa_host;

extern "C" {

dsa_status_t dsa_indexer_prepare_workspace_size(const dsa_prepare_desc_t *desc, size_t *bytes) {
  if (!bytes) return DSA_ERR_INVALID_ARG;
  const dsa_status_t st = check_prep_desc(desc);
  if (st != DSA_OK) return st;
  *bytes = workspace_bytes_for(desc);
  return DSA_OK;
}

dsa_status_t dsa_indexer_prepare(const dsa_prepare_desc_t *desc, const void *x, const void *qr,
                                 const void *wq_b, const void *wk, const void *weights_proj,
                                 const float *k_norm_weight, const float *k_norm_bias,
                                 const float *cos, const float *sin, const int32_t *positions,
                                 void *q_out, float *w_out, void *key_cache, void *workspace,
                                 size_t workspace_bytes, dsa_stream_t stream) {
  dsa_status_t st = check_prep_desc(desc);
  if (st != DSA_OK) return st;
  if (!x || !qr || !wq_b || !wk || !weights_proj || !k_norm_weight || !k_norm_bias || !q_out ||
      !w_out || !key_cache)
    return DSA_ERR_INVALID_ARG;
  if (desc->rope_dim > 0 && (!cos || !sin)) return DSA_ERR_INVALID_ARG;
  for (const void *ptr : {x, qr, wq_b, wk, weights_proj, static_cast<const void *>(q_out),
                          static_cast<const void *>(key_cache)})
    if (!aligned(ptr, 16)) return DSA_ERR_INVALID_ARG;
  if (!aligned(w_out, 4) || !aligned(k_norm_weight, 4) || !aligned(k_norm_bias, 4) ||
      (positions && !aligned(positions, 4)))
    return DSA_ERR_INVALID_ARG;
  if (!workspace || !aligned(workspace, 256) || workspace_bytes < workspace_bytes_for(desc))
    return DSA_ERR_WORKSPACE;
  DeviceInfo *dev = nullptr;
  st = device_info(&dev);
  if (st != DSA_OK) return st;
  st = ensure_smem_attr(dev, kAttrPrepare, dsa::prep_gemm_kernel, static_cast<int>(dsa::PrepSmem::total));
  if (st != DSA_OK) return st;

  const int T = desc->T, H = desc->H;
  CUtensorMap ta_q, tb_q, ta_x, tb_k, tb_w;
  if ((st = map_rows(&ta_q, qr, T, desc->q_lora_rank, 128)) != DSA_OK) return st;
  if ((st = map_rows(&tb_q, wq_b, static_cast<int64_t>(H) * 128, desc->q_lora_rank, 128)) !=
      DSA_OK)
    return st;
  if ((st = map_rows(&ta_x, x, T, desc->hidden, 128)) != DSA_OK) return st;
  if ((st = map_rows(&tb_k, wk, 128, desc->hidden, 128)) != DSA_OK) return st;
  if ((st = map_rows(&tb_w, weights_proj, H, desc->hidden, H)) != DSA_OK) return st;

  uint8_t *ws = static_cast<uint8_t *>(workspace);
  dsa::PrepParams p{};
  p.T = T;
  p.H = H;
  p.rope_dim = desc->rope_dim;
  p.eps = desc->k_norm_eps;
  p.w_scale = desc->w_scale;
  p.cos = cos;
  p.sin = sin;
  p.gain = k_norm_weight;
  p.bias = k_norm_bias;
  p.q_out = static_cast<uint16_t *>(q_out);
  p.w_out = w_out;
  p.k_cache = static_cast<uint16_t *>(key_cache);
  p.k_seq_stride = desc->k_seq_stride;
  p.S = desc->S;
  p.positions = positions;
  p.part = reinterpret_cast<float *>(ws + kWorkspaceHeader);
  p.err = reinterpret_cast<unsigned int *>(ws);
  p.err_info = reinterpret_cast<unsigned int *>(ws) + 1;
  p.wait_limit_ns = desc->wait_limit_ns ? desc->wait_limit_ns : kPrepWaitLimitNs;
  p.drain_limit_ns = kPrepDrainLimitNs;
  cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);

  // queries: one head a feature tile
  const Split q = plan(T, H, desc->q_lora_rank);
  dsa::PrepParams pq = p;
  pq.mode = dsa::kPrepQ;
  pq.m_tiles = q.m_tiles;
  pq.n_tiles = q.n_tiles;
  pq.ksteps = q.ksteps;
  pq.nsplit = q.nsplit;
  pq.per = q.per;
  pq.BN = 128;
  pq.n1 = 128;
  pq.N_total = H * 128;
  st = launch_gemm(dev, ta_q, tb_q, tb_q, pq, s);
  if (st != DSA_OK) return st;
  // keys and head weights: wk's 128 rows over weights_proj's H rows
  const Split kw = plan(T, 1, desc->hidden);
  dsa::PrepParams pk = p;
  pk.mode = dsa::kPrepKW;
  pk.m_tiles = kw.m_tiles;
  pk.n_tiles = 1;
  pk.ksteps = kw.ksteps;
  pk.nsplit = kw.nsplit;
  pk.per = kw.per;
  pk.BN = 128 + H;
  pk.n1 = 128;
  pk.N_total = 128 + H;
  st = launch_gemm(dev, ta_x, tb_k, tb_w, pk, s);
  if (st != DSA_OK) return st;
  return DSA_OK;
}

}  // extern "C"
