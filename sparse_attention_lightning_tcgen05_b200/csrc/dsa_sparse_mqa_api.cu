// dsa_sparse_mqa_api.cu -- C ABI of the sparse-MQA consumer (the operation,
// layouts and error rules are stated in include/dsa_sparse_mqa.h): argument
// checks, the split of each token's index row, the query tensor map and the
// launches.
#include <cuda.h>
#include <cuda_runtime.h>

#include <algorithm>
#include <cmath>
#include <cstdint>

#include "dsa_launch.h"
#include "dsa_sparse_mqa.h"
#include "sparse_mqa.cuh"

namespace dsa_host {
namespace {

constexpr uint64_t kMqaWaitLimitNs = 4000000000ull;
constexpr uint64_t kMqaDrainLimitNs = 4000000000ull;
// The split of index rows is sized for the 148 SMs of a B200, so that the
// workspace size depends on the descriptor alone.
constexpr int kSizingSms = 148;

dsa_status_t check_mqa_desc(const dsa_sparse_mqa_desc_t *d) {
  if (!d) return DSA_ERR_INVALID_ARG;
  if (d->B < 1 || d->S < 1 || d->H < 1 || d->K < 1 || d->K_top < 1) return DSA_ERR_INVALID_ARG;
  if (!std::isfinite(d->sm_scale)) return DSA_ERR_INVALID_ARG;
  if (d->D != 128) return DSA_ERR_UNSUPPORTED;
  if (d->H > 128) return DSA_ERR_UNSUPPORTED;
  if (static_cast<int64_t>(d->B) * d->S * d->H > INT32_MAX - 256) return DSA_ERR_UNSUPPORTED;
  // kv rows are addressed as 32-bit TMA coordinates over all batches
  if (static_cast<int64_t>(d->B) * d->K >= INT32_MAX) return DSA_ERR_UNSUPPORTED;
  return DSA_OK;
}

// Ranges per token and index entries per range (a multiple of 128): one
// range when the tokens alone fill the GPU, else enough ranges for about
// one item per SM, each of at least one tile.
void mqa_split(const dsa_sparse_mqa_desc_t *d, int &nsplit, int &chunk) {
  const int64_t T = static_cast<int64_t>(d->B) * d->S;
  const int tiles = (d->K_top + dsa::kMqaTile - 1) / dsa::kMqaTile;
  int want = 1;
  if (T < kSizingSms) want = static_cast<int>((kSizingSms + T - 1) / T);
  want = std::max(1, std::min(want, tiles));
  const int per = (tiles + want - 1) / want;
  chunk = per * dsa::kMqaTile;
  nsplit = (d->K_top + chunk - 1) / chunk;
}

size_t partial_bytes(const dsa_sparse_mqa_desc_t *d, int nsplit) {
  if (nsplit <= 1) return 0;
  const size_t T = static_cast<size_t>(d->B) * d->S;
  return T * nsplit * d->H * (dsa::kMqaD + 2) * 4;
}

}  // namespace
}  // namespace dsa_host

using namespace dsa_host;

extern "C" {

dsa_status_t dsa_sparse_mqa_workspace_size(const dsa_sparse_mqa_desc_t *desc, size_t *bytes) {
  if (!bytes) return DSA_ERR_INVALID_ARG;
  const dsa_status_t st = check_mqa_desc(desc);
  if (st != DSA_OK) return st;
  int nsplit = 1, chunk = 0;
  mqa_split(desc, nsplit, chunk);
  *bytes = kWorkspaceHeader + partial_bytes(desc, nsplit);
  return DSA_OK;
}

dsa_status_t dsa_sparse_mqa_forward(const dsa_sparse_mqa_desc_t *desc, const void *q,
                                    const void *kv, const float *sinks, const int32_t *topk,
                                    void *out, void *workspace, size_t workspace_bytes,
                                    dsa_stream_t stream) {
  dsa_status_t st = check_mqa_desc(desc);
  if (st != DSA_OK) return st;
  if (!q || !kv || !sinks || !topk || !out) return DSA_ERR_INVALID_ARG;
  if (!aligned(q, 16) || !aligned(kv, 16) || !aligned(out, 16) || !aligned(sinks, 4) ||
      !aligned(topk, 4))
    return DSA_ERR_INVALID_ARG;
  int nsplit = 1, chunk = 0;
  mqa_split(desc, nsplit, chunk);
  const size_t part = partial_bytes(desc, nsplit);
  if (!workspace || !aligned(workspace, 256) || workspace_bytes < kWorkspaceHeader + part)
    return DSA_ERR_WORKSPACE;
  DeviceInfo *dev = nullptr;
  st = device_info(&dev);
  if (st != DSA_OK) return st;
  const int smem = static_cast<int>(dsa::MqaSmem::total);
  st = ensure_smem_attr(dev, kAttrSparseMqa, dsa::sparse_mqa_kernel, smem);
  if (st != DSA_OK) return st;

  const int T = desc->B * desc->S;
  CUtensorMap tq;
  {
    const cuuint64_t dims[2] = {128, static_cast<cuuint64_t>(T) * desc->H};
    const cuuint64_t strides[1] = {256};
    const cuuint32_t box[2] = {64, static_cast<cuuint32_t>(desc->H)};
    st = make_map(&tq, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, q, dims, strides, box);
    if (st != DSA_OK) return st;
  }
  // the kv rows of all batches, one row a box (tile::gather4 loads four)
  CUtensorMap tkv;
  {
    const cuuint64_t dims[2] = {128, static_cast<cuuint64_t>(desc->B) * desc->K};
    const cuuint64_t strides[1] = {256};
    const cuuint32_t box[2] = {64, 1};
    st = make_map(&tkv, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, kv, dims, strides, box);
    if (st != DSA_OK) return st;
  }
  uint8_t *ws = static_cast<uint8_t *>(workspace);
  dsa::MqaParams p{};
  p.T = T;
  p.H = desc->H;
  p.S_per_batch = desc->S;
  p.K = desc->K;
  p.K_top = desc->K_top;
  p.nsplit = nsplit;
  p.chunk = chunk;
  p.kv = static_cast<const uint16_t *>(kv);
  p.idx = topk;
  p.sinks = sinks;
  p.scale_log2 = desc->sm_scale * dsa::kLog2e;
  p.out = static_cast<uint16_t *>(out);
  if (nsplit > 1) {
    p.part_o = reinterpret_cast<float *>(ws + kWorkspaceHeader);
    p.part_ml = p.part_o + static_cast<size_t>(T) * nsplit * desc->H * dsa::kMqaD;
  }
  p.err = reinterpret_cast<unsigned int *>(ws);
  p.err_info = reinterpret_cast<unsigned int *>(ws) + 1;
  p.wait_limit_ns = desc->wait_limit_ns ? desc->wait_limit_ns : kMqaWaitLimitNs;
  p.drain_limit_ns = kMqaDrainLimitNs;
  const int64_t items = static_cast<int64_t>(T) * nsplit;
  const int grid = static_cast<int>(std::min<int64_t>(items, dev->num_sms));
  cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
  if (launch_pdl(dsa::sparse_mqa_kernel, grid, dsa::kMqaThreads, static_cast<size_t>(smem), s, 0,
                 tq, tkv, p) != cudaSuccess)
    return DSA_ERR_CUDA;
  if (nsplit > 1) {
    const int64_t warps = static_cast<int64_t>(T) * desc->H;   // one per (token, head)
    const int blocks = static_cast<int>((warps * 32 + 255) / 256);
    if (launch_pdl(dsa::sparse_mqa_combine_kernel, blocks, 256, 0, s, 0, p) != cudaSuccess)
      return DSA_ERR_CUDA;
  }
  return DSA_OK;
}

}  // extern "C"
