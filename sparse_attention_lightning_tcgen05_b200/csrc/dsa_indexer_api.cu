// dsa_indexer_api.cu -- C ABI of libdsa_indexer: argument checks, TMA tensor
// maps, kernel choice and launches. The operations, layouts and error rules
// are stated in include/dsa_indexer.h.
#include <cuda.h>
#include <cuda_runtime.h>
#include <cudaTypedefs.h>

#include <algorithm>
#include <cstdint>
#include <cstring>
#include <mutex>
#include <utility>

#include "dsa_indexer.h"
#include "dsa_launch.h"
#include "cu_check.cuh"
#include "score_kernel.cuh"
#include "topk_causal.cuh"
#include "topk_cluster.cuh"
#include "topk_rows.cuh"
#include "topk_kernel.cuh"

namespace dsa_host {

using dsa::ScoreParams;
using dsa::ScoreSmem;
using dsa::TopkParams;

constexpr uint64_t kWaitLimitNs = 4000000000ull;   // default limit of any single wait
constexpr uint64_t kDrainLimitNs = 4000000000ull;  // drains of in-flight copies / MMAs
constexpr int kMaxDevices = 64;
constexpr uint32_t kMaxSmemPerBlock = 232448;      // 227 KB opt-in limit of sm_100

// Packed causal top-k: threads per row, and the scores a row may stage in
// shared memory (rows that fit take the two-pass selection, longer rows the
// sampled threshold). Build-time tunables.
#ifndef DSA_CAUSAL_TOPK_THREADS
#define DSA_CAUSAL_TOPK_THREADS 512
#endif
#ifndef DSA_CAUSAL_TOPK_STAGE
#define DSA_CAUSAL_TOPK_STAGE 12288
#endif
constexpr int kCausalTopkThreads = DSA_CAUSAL_TOPK_THREADS;
constexpr int kCausalTopkStage = DSA_CAUSAL_TOPK_STAGE;

// Words of the workspace header.
// err/err_info: first device-side failure since the last get_error (sticky).
// cu_bad: written by the cu_seqlens check of every CAUSAL call, read by that
// call's score and top-k kernels.
struct WsHeader {
  unsigned int err;
  unsigned int err_info;
  unsigned int cu_bad;
  unsigned int reserved[61];
};
static_assert(sizeof(WsHeader) == kWorkspaceHeader, "header size");

// ---- per-device state -----------------------------------------------------------

std::mutex g_mu;
DeviceInfo g_dev[kMaxDevices];
PFN_cuTensorMapEncodeTiled_v12000 g_encode = nullptr;

dsa_status_t device_info(DeviceInfo **out) {
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices)
    return DSA_ERR_CUDA;
  std::lock_guard<std::mutex> lk(g_mu);
  DeviceInfo &d = g_dev[dev];
  if (!d.probed) {
    int major = 0, minor = 0, sms = 0;
    if (cudaDeviceGetAttribute(&major, cudaDevAttrComputeCapabilityMajor, dev) != cudaSuccess ||
        cudaDeviceGetAttribute(&minor, cudaDevAttrComputeCapabilityMinor, dev) != cudaSuccess ||
        cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess)
      return DSA_ERR_CUDA;
    d.probed = true;
    d.ok = (major == 10 && minor == 0);
    d.num_sms = sms;
  }
  if (!d.ok) return DSA_ERR_DEVICE;
  if (!g_encode) {
    void *fn = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &fn, cudaEnableDefault, &q) !=
            cudaSuccess ||
        q != cudaDriverEntryPointSuccess || fn == nullptr)
      return DSA_ERR_CUDA;
    g_encode = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(fn);
  }
  *out = &d;
  return DSA_OK;
}

// Raise the dynamic shared-memory limit of kernel `bit` once per device.
dsa_status_t ensure_smem_attr_raw(DeviceInfo *d, uint32_t bit, const void *kernel, int bytes) {
  std::lock_guard<std::mutex> lk(g_mu);
  if (d->attr_done >> bit & 1u) return DSA_OK;
  if (cudaFuncSetAttribute(kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, bytes) !=
      cudaSuccess)
    return DSA_ERR_CUDA;
  d->attr_done |= 1u << bit;
  return DSA_OK;
}

// ---- argument checks -----------------------------------------------------------------

dsa_status_t check_desc(const dsa_indexer_desc_t *d) {
  if (!d) return DSA_ERR_INVALID_ARG;
  if (d->T < 1 || d->H < 1 || d->index_topk < 1) return DSA_ERR_INVALID_ARG;
  if (d->flags & ~(DSA_FLAG_SCORES_IN_WORKSPACE | DSA_FLAG_SELFTEST_STALL))
    return DSA_ERR_INVALID_ARG;
  if (d->dtype != DSA_KV_BF16 && d->dtype != DSA_KV_FP8_E4M3_E8M0_B32) return DSA_ERR_INVALID_ARG;
  if (d->mask != DSA_MASK_POSITIONS && d->mask != DSA_MASK_CAUSAL &&
      d->mask != DSA_MASK_COMPRESSED)
    return DSA_ERR_INVALID_ARG;
  if (d->D != 128) return DSA_ERR_UNSUPPORTED;
  if (d->H > 256) return DSA_ERR_UNSUPPORTED;
  if (static_cast<int64_t>(d->T) * d->H > INT32_MAX - 256) return DSA_ERR_UNSUPPORTED;
  if (d->block_table) {
    // a paged cache: one page pool, a block-table row per token
    if (d->mask != DSA_MASK_POSITIONS || d->k_seq_stride != 0) return DSA_ERR_INVALID_ARG;
    if (d->page_size < 16 || d->page_size > 65536 || (d->page_size & (d->page_size - 1)) != 0)
      return DSA_ERR_INVALID_ARG;
    if (d->pages_per_seq < 1 || d->num_pages < 1) return DSA_ERR_INVALID_ARG;
    if (d->S < 1 || d->S > static_cast<int64_t>(d->pages_per_seq) * d->page_size)
      return DSA_ERR_INVALID_ARG;
    if (!aligned(d->block_table, 4)) return DSA_ERR_INVALID_ARG;
  }
  if (d->mask == DSA_MASK_POSITIONS) {
    if (d->S < 1) return DSA_ERR_INVALID_ARG;
    if (d->S > INT32_MAX - 256) return DSA_ERR_UNSUPPORTED;
    if (d->k_seq_stride != 0) {
      if (d->k_seq_stride < d->S * d->D || d->k_seq_stride % d->D != 0) return DSA_ERR_INVALID_ARG;
    }
  } else if (d->mask == DSA_MASK_COMPRESSED) {
    if (d->S < 1 || d->k_seq_stride != 0) return DSA_ERR_INVALID_ARG;
    if (d->compress_ratio < 1 || d->query_start < 0) return DSA_ERR_INVALID_ARG;
    if (d->S > INT32_MAX - 256) return DSA_ERR_UNSUPPORTED;
    // absolute positions, like decode positions, are 32-bit
    if (d->query_start > static_cast<int64_t>(INT32_MAX) - d->T) return DSA_ERR_UNSUPPORTED;
  } else {
    if (d->num_seqs < 1 || !d->cu_seqlens) return DSA_ERR_INVALID_ARG;
  }
  if (d->dtype == DSA_KV_FP8_E4M3_E8M0_B32) {
    if (d->H > 128) return DSA_ERR_UNSUPPORTED;
    // scale rows of consecutive caches must start on 16-byte boundaries
    if (d->mask == DSA_MASK_POSITIONS && d->k_seq_stride % 512 != 0) return DSA_ERR_INVALID_ARG;
  }
  return DSA_OK;
}

// The compressed rule of a COMPRESSED descriptor (flag 0 otherwise).
void set_compressed_rule(const dsa_indexer_desc_t *d, int &flag, dsa::CompressedRule &c) {
  flag = d->mask == DSA_MASK_COMPRESSED;
  c.base = flag ? static_cast<int32_t>(d->query_start + 1) : 1;
  c.div = dsa::div_magic(flag ? static_cast<uint32_t>(d->compress_ratio) : 1u);
}

dsa_status_t check_workspace(const void *ws, size_t bytes) {
  if (!ws || !aligned(ws, 256) || bytes < kWorkspaceHeader) return DSA_ERR_WORKSPACE;
  return DSA_OK;
}

// Floats of all score rows (host): T*S, or for CAUSAL sum_i L_i^2 from the
// host copy of cu_seqlens, which is checked like the device array is.
dsa_status_t score_elems(const dsa_indexer_desc_t *d, int64_t *n) {
  if (d->mask != DSA_MASK_CAUSAL) {
    *n = static_cast<int64_t>(d->T) * d->S;
    return DSA_OK;
  }
  const int32_t *cu = d->cu_seqlens_host;
  if (!cu || cu[0] != 0 || cu[d->num_seqs] != d->T) return DSA_ERR_INVALID_ARG;
  int64_t total = 0;
  for (int i = 0; i < d->num_seqs; ++i) {
    if (cu[i + 1] < cu[i]) return DSA_ERR_INVALID_ARG;
    const int64_t L = cu[i + 1] - cu[i];
    total += L * L;
  }
  *n = total;
  return DSA_OK;
}

// The score rows of a top-k-only call: right after the workspace header.
// Returns the floats the workspace holds for them (-1 when the caller's
// buffer is used and its size is unknown).
int64_t workspace_scores(void *ws, size_t ws_bytes, float **scores) {
  if (*scores != nullptr) return -1;
  *scores = reinterpret_cast<float *>(static_cast<uint8_t *>(ws) + kWorkspaceHeader);
  return static_cast<int64_t>((ws_bytes - kWorkspaceHeader) / 4);
}



// ---- tensor maps -------------------------------------------------------------------------

dsa_status_t make_map(CUtensorMap *m, CUtensorMapDataType dt, cuuint32_t rank, const void *base,
                      const cuuint64_t *dims, const cuuint64_t *strides_bytes,
                      const cuuint32_t *box, CUtensorMapSwizzle swz) {
  cuuint32_t estr[3] = {1, 1, 1};
  CUresult r = g_encode(m, dt, rank, const_cast<void *>(base), dims, strides_bytes, box, estr,
                        CU_TENSOR_MAP_INTERLEAVE_NONE, swz,
                        CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                        CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  return r == CUDA_SUCCESS ? DSA_OK : DSA_ERR_INVALID_ARG;
}

// One kernel choice: template instance and its geometry.
using ScoreKernelFn = void (*)(const CUtensorMap, const CUtensorMap, const CUtensorMap,
                               const CUtensorMap, const ScoreParams);
struct ScoreLaunch {
  ScoreKernelFn kernel;
  uint32_t attr_bit;
  int stages, qbuf, nsub, epi, tiles, issuers;   // as the template arguments
  int tq_sub, n_cols;
  int max_cols;   // widest query block this instance ever runs (smem attribute)
  bool fp8;
  // producer, MMA, epilogue warps, (fp8) scale warp, second issuer
  int threads() const { return (2 + epi + (fp8 ? 1 : 0) + (issuers - 1)) * 32; }
};



int round16(int x) { return (x + 15) / 16 * 16; }

// Largest power of two <= x (x >= 1).
int pow2_floor(int x) {
  int p = 1;
  while (p * 2 <= x) p *= 2;
  return p;
}

// Kernel instances. Decode with one cache per token (H = 64): two key tiles
// per pipeline item. Prefill / a shared cache (H = 64): 8 tokens per query
// block as two N = 256 sub-blocks. Any other H: the generic epilogue. Each
// instance is compiled for one mask mode.
constexpr int kPos = dsa::kModePositions, kCau = dsa::kModeCausal, kCmp = dsa::kModeCompressed;

// COMPRESSED: the shared-cache instances, compiled with the compressed rule.
ScoreLaunch choose_score_compressed(const dsa_indexer_desc_t *d) {
  const int H = d->H;
  if (d->dtype == DSA_KV_BF16) {
    if (H == 64)
      return {dsa::score_kernel<64, 2, 1, 2, 2, 1, 8, false, 1, kCmp>, 12, 2, 1, 2, 8, 1, 1, 4,
              256, 256, false};
    const int tq = pow2_floor(std::min(128, 256 / H));
    return {dsa::score_kernel<0, 1, 1, 2, 4, 1, 4, false, 1, kCmp>, 13, 4, 1, 1, 4, 1, 1, tq,
            round16(tq * H), 256, false};
  }
  if (H == 64)
    return {dsa::score_kernel<64, 2, 1, 2, 4, 1, 8, true, 1, kCmp>, 14, 4, 1, 2, 8, 1, 1, 2, 128,
            128, true};
  const int tq = pow2_floor(std::min(128, 128 / H));
  return {dsa::score_kernel<0, 1, 1, 2, 4, 1, 4, true, 1, kCmp>, 15, 4, 1, 1, 4, 1, 1, tq,
          round16(tq * H), 128, true};
}

ScoreLaunch choose_score(const dsa_indexer_desc_t *d) {
  if (d->mask == DSA_MASK_COMPRESSED) return choose_score_compressed(d);
  const bool causal = d->mask == DSA_MASK_CAUSAL;
  const bool per_token_cache = !causal && (d->k_seq_stride != 0 || d->block_table);
  const int H = d->H;
  if (d->dtype == DSA_KV_BF16) {
    if (per_token_cache) {
      if (H == 64)
        return {dsa::score_kernel<64, 1, 2, 3, 2, 2, 8, false, 2, kPos>, 0, 2, 2, 1, 8, 2, 2, 1, 64,
                64, false};
      return {dsa::score_kernel<0, 1, 1, 2, 4, 1, 4, false, 1, kPos>, 1, 4, 1, 1, 4, 1, 1, 1,
              round16(H), 256, false};
    }
    if (H == 64)
      return causal ? ScoreLaunch{dsa::score_kernel<64, 2, 1, 2, 2, 1, 8, false, 1, kCau>, 2, 2, 1,
                                  2, 8, 1, 1, 4, 256, 256, false}
                    : ScoreLaunch{dsa::score_kernel<64, 2, 1, 2, 2, 1, 8, false, 1, kPos>, 6, 2, 1,
                                  2, 8, 1, 1, 4, 256, 256, false};
    const int tq = pow2_floor(std::min(128, 256 / H));
    return causal ? ScoreLaunch{dsa::score_kernel<0, 1, 1, 2, 4, 1, 4, false, 1, kCau>, 7, 4, 1, 1,
                                4, 1, 1, tq, round16(tq * H), 256, false}
                  : ScoreLaunch{dsa::score_kernel<0, 1, 1, 2, 4, 1, 4, false, 1, kPos>, 1, 4, 1, 1,
                                4, 1, 1, tq, round16(tq * H), 256, false};
  }
  if (per_token_cache) {
    if (H == 64)
      return {dsa::score_kernel<64, 1, 2, 3, 5, 2, 8, true, 2, kPos>, 3, 5, 2, 1, 8, 2, 2, 1, 64,
              64, true};
    return {dsa::score_kernel<0, 1, 1, 2, 4, 1, 4, true, 1, kPos>, 4, 4, 1, 1, 4, 1, 1, 1,
            round16(H), 128, true};
  }
  if (H == 64)
    return causal ? ScoreLaunch{dsa::score_kernel<64, 2, 1, 2, 4, 1, 8, true, 1, kCau>, 5, 4, 1, 2,
                                8, 1, 1, 2, 128, 128, true}
                  : ScoreLaunch{dsa::score_kernel<64, 2, 1, 2, 4, 1, 8, true, 1, kPos>, 10, 4, 1,
                                2, 8, 1, 1, 2, 128, 128, true};
  const int tq = pow2_floor(std::min(128, 128 / H));
  return causal ? ScoreLaunch{dsa::score_kernel<0, 1, 1, 2, 4, 1, 4, true, 1, kCau>, 11, 4, 1, 1, 4,
                              1, 1, tq, round16(tq * H), 128, true}
                : ScoreLaunch{dsa::score_kernel<0, 1, 1, 2, 4, 1, 4, true, 1, kPos>, 4, 4, 1, 1, 4,
                              1, 1, tq, round16(tq * H), 128, true};
}

// CAUSAL: check cu_seqlens on the device (one CTA) before the kernels that
// read it; they skip their work when it fails. cap_elems >= 0 also bounds the
// score rows (they live in a workspace of that many floats).
dsa_status_t launch_cu_check(const dsa_indexer_desc_t *d, WsHeader *ws, int64_t cap_elems,
                             cudaStream_t stream) {
  if (launch_pdl(dsa::cu_seqlens_check_kernel<256>, 1, 256, 0, stream, 0, d->cu_seqlens,
                 d->num_seqs, d->T, static_cast<long long>(cap_elems), &ws->cu_bad,
                 &ws->err) != cudaSuccess)
    return DSA_ERR_CUDA;
  return DSA_OK;
}

dsa_status_t launch_score(const dsa_indexer_desc_t *d, const void *q, const uint8_t *q_scale,
                          const float *w, const void *k, const uint8_t *k_scale,
                          const int32_t *positions, float *scores, WsHeader *ws,
                          int64_t cap_elems, cudaStream_t stream) {
  DeviceInfo *dev = nullptr;
  dsa_status_t st = device_info(&dev);
  if (st != DSA_OK) return st;
  if (d->mask == DSA_MASK_CAUSAL) {
    st = launch_cu_check(d, ws, cap_elems, stream);
    if (st != DSA_OK) return st;
  }
  const ScoreLaunch L = choose_score(d);
  const ScoreSmem plan(L.stages, L.qbuf, L.nsub, L.n_cols, L.fp8, L.epi, L.tiles);
  // the attribute is set once per kernel: use the widest query block it runs
  const ScoreSmem widest(L.stages, L.qbuf, L.nsub, L.max_cols, L.fp8, L.epi, L.tiles);
  if (widest.total > kMaxSmemPerBlock || plan.total > widest.total) return DSA_ERR_UNSUPPORTED;
  st = ensure_smem_attr(dev, L.attr_bit, L.kernel, static_cast<int>(widest.total));
  if (st != DSA_OK) return st;

  const bool causal = d->mask == DSA_MASK_CAUSAL;
  const bool paged = d->block_table != nullptr;
  const bool shared = causal || (d->k_seq_stride == 0 && !paged);
  const cuuint64_t rows = causal ? static_cast<cuuint64_t>(d->T) : static_cast<cuuint64_t>(d->S);
  const cuuint64_t caches = shared ? 1 : static_cast<cuuint64_t>(d->T);
  const cuuint64_t elt = L.fp8 ? 1 : 2;
  const cuuint64_t stride_elems = shared ? rows * 128 : static_cast<cuuint64_t>(d->k_seq_stride);
  const cuuint64_t qrows = static_cast<cuuint64_t>(d->T) * d->H;
  CUtensorMap tk, tq, tksf, tqsf;
  std::memset(&tksf, 0, sizeof tksf);
  std::memset(&tqsf, 0, sizeof tqsf);
  if (paged) {
    // the page pool: [num_pages, page_size, D]; a 128-slot key tile is one
    // box (pages of >= 128 slots) or 128/page_size boxes of one page each
    const cuuint64_t ps = static_cast<cuuint64_t>(d->page_size);
    const cuuint64_t dims[3] = {128, ps, static_cast<cuuint64_t>(d->num_pages)};
    const cuuint64_t strides[2] = {128 * elt, ps * 128 * elt};
    const cuuint32_t box[3] = {static_cast<cuuint32_t>(128 / elt),
                               static_cast<cuuint32_t>(std::min<cuuint64_t>(ps, dsa::kBlockM)), 1};
    st = make_map(&tk, L.fp8 ? CU_TENSOR_MAP_DATA_TYPE_UINT8 : CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3,
                  k, dims, strides, box);
    if (st != DSA_OK) return st;
    if (L.fp8) {
      // the scale pool [num_pages, page_size] of 32-bit words (4 e8m0 bytes
      // a slot), one box per page box of the data
      const cuuint64_t sdims[2] = {ps, static_cast<cuuint64_t>(d->num_pages)};
      const cuuint64_t sstrides[1] = {ps * 4};
      const cuuint32_t sbox[2] = {static_cast<cuuint32_t>(std::min<cuuint64_t>(ps, dsa::kBlockM)),
                                  1};
      st = make_map(&tksf, CU_TENSOR_MAP_DATA_TYPE_UINT32, 2, k_scale, sdims, sstrides, sbox,
                    CU_TENSOR_MAP_SWIZZLE_NONE);
      if (st != DSA_OK) return st;
    }
  } else {
    const cuuint64_t dims[3] = {128, rows, caches};
    const cuuint64_t strides[2] = {128 * elt, stride_elems * elt};
    const cuuint32_t box[3] = {static_cast<cuuint32_t>(128 / elt), dsa::kBlockM, 1};
    st = make_map(&tk, L.fp8 ? CU_TENSOR_MAP_DATA_TYPE_UINT8 : CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3,
                  k, dims, strides, box);
    if (st != DSA_OK) return st;
  }
  {
    const cuuint64_t dims[2] = {128, qrows};
    const cuuint64_t strides[1] = {128 * elt};
    const cuuint32_t box[2] = {static_cast<cuuint32_t>(128 / elt),
                               static_cast<cuuint32_t>(L.n_cols)};
    st = make_map(&tq, L.fp8 ? CU_TENSOR_MAP_DATA_TYPE_UINT8 : CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2,
                  q, dims, strides, box);
    if (st != DSA_OK) return st;
  }
  if (L.fp8 && !paged) {
    // scale bytes of one slot (4 blocks of 32 along D) read as one 32-bit word
    // (one cache: the second dimension is never stepped; its stride only
    // has to be a legal multiple of 16 bytes)
    const cuuint64_t dims[2] = {rows, caches};
    const cuuint64_t strides[1] = {shared ? (rows * 4 + 15) / 16 * 16 : stride_elems / 32};
    const cuuint32_t box[2] = {dsa::kBlockM + dsa::kSfPad, 1};
    st = make_map(&tksf, CU_TENSOR_MAP_DATA_TYPE_UINT32, 2, k_scale, dims, strides, box,
                  CU_TENSOR_MAP_SWIZZLE_NONE);
    if (st != DSA_OK) return st;
  }
  if (L.fp8) {
    const cuuint64_t qdims[2] = {qrows, 1};
    const cuuint64_t qstrides[1] = {(qrows * 4 + 15) / 16 * 16};   // never stepped
    const cuuint32_t qbox[2] = {static_cast<cuuint32_t>(L.n_cols + dsa::kSfPad), 1};
    st = make_map(&tqsf, CU_TENSOR_MAP_DATA_TYPE_UINT32, 2, q_scale, qdims, qstrides, qbox,
                  CU_TENSOR_MAP_SWIZZLE_NONE);
    if (st != DSA_OK) return st;
  }

  ScoreParams p{};
  p.mode = causal ? dsa::kModeCausal : dsa::kModePositions;
  p.T = d->T;
  p.H = d->H;
  p.S = d->S;
  p.shared_cache = shared;
  // a cache per token: each key tile is read by one token only
  p.k_once = !causal && !shared;
  p.block_table = d->block_table;
  p.pages_per_seq = paged ? d->pages_per_seq : 0;
  p.num_pages = paged ? d->num_pages : 0;
  p.page_shift = paged ? __builtin_ctz(static_cast<unsigned>(d->page_size)) : 0;
  p.num_seqs = d->num_seqs;
  p.cu_seqlens = d->cu_seqlens;
  // COMPRESSED runs as POSITIONS over one shared cache, with no positions
  // array: the kernels derive each row's last valid slot from the ratio.
  p.positions = positions;
  set_compressed_rule(d, p.compressed, p.comp);
  p.w = w;
  p.scores = scores;
  p.tq_sub = L.tq_sub;
  p.n_cols = L.n_cols;
  p.err = &ws->err;
  p.err_info = &ws->err_info;
  p.cu_bad = &ws->cu_bad;
  p.wait_limit_ns = d->wait_limit_ns ? d->wait_limit_ns : kWaitLimitNs;
  p.drain_limit_ns = kDrainLimitNs;
  p.selftest_stall = (d->flags & DSA_FLAG_SELFTEST_STALL) ? 1 : 0;
  // With one query buffer the next block's query cannot load while the
  // current block's MMAs run: a block start costs about 3/4 of a key tile
  // (measured on an 8192-token prefill), so the split between CTAs counts
  // it. Double-buffered queries hide it.
  p.blk_w = L.qbuf == 1 ? 6 : 0;

  int grid = dev->num_sms;
  if (!causal) {
    const int64_t ntiles = (d->S + dsa::kBlockM - 1) / dsa::kBlockM;
    const int tqt = L.tq_sub * L.nsub;
    const int64_t nqb = p.shared_cache ? (d->T + tqt - 1) / tqt : d->T;
    if (nqb * ntiles < grid) grid = static_cast<int>(nqb * ntiles);
  }
  if (launch_pdl(L.kernel, grid, L.threads(), plan.total, stream, 0, tk, tq, tksf, tqsf, p) !=
      cudaSuccess)
    return DSA_ERR_CUDA;
  return DSA_OK;
}

// The row top-k: one CTA per row, a buffer of NT*KPT floats.
template <int NT, int KPT>
dsa_status_t launch_topk_rows(DeviceInfo *dev, int which, int T, const TopkParams &p,
                              cudaStream_t stream) {
  auto kernel = dsa::topk_rows_kernel<NT, KPT>;
  const int smem = NT * KPT * 4;
  dsa_status_t st = ensure_smem_attr(dev, which ? kAttrTopkRows16 : kAttrTopkRows8, kernel, smem);
  if (st != DSA_OK) return st;
  if (launch_pdl(kernel, T, NT, smem, stream, 0, p) != cudaSuccess) return DSA_ERR_CUDA;
  return DSA_OK;
}

dsa_status_t launch_topk(const dsa_indexer_desc_t *d, const float *scores,
                         const int32_t *positions, int32_t *topk, WsHeader *ws, bool check_cu,
                         int64_t cap_elems, cudaStream_t stream) {
  DeviceInfo *dev = nullptr;
  dsa_status_t st = device_info(&dev);
  if (st != DSA_OK) return st;
  if (check_cu && d->mask == DSA_MASK_CAUSAL) {
    st = launch_cu_check(d, ws, cap_elems, stream);
    if (st != DSA_OK) return st;
  }
  TopkParams p{};
  p.cu_bad = &ws->cu_bad;
  p.err = &ws->err;
  p.mode = d->mask == DSA_MASK_CAUSAL ? dsa::kModeCausal : dsa::kModePositions;
  p.T = d->T;
  p.S = d->S;
  p.num_seqs = d->num_seqs;
  p.cu_seqlens = d->cu_seqlens;
  p.positions = positions;
  set_compressed_rule(d, p.compressed, p.comp);
  p.scores = scores;
  p.topk = topk;
  p.k = d->index_topk;
  // Decode-style rows of at most 4096 slots (pooled keys, short caches): one
  // CTA a row, the row held in registers. A row's buffer starts at the
  // 16-byte boundary at or before it, up to 3 floats early (none when the
  // score buffer is 16-byte aligned and S a multiple of 4), so an instance
  // holding NT*KPT floats takes rows of up to NT*KPT - 3 slots (NT*KPT when
  // every row is aligned). Longer decode rows are few and long: a cluster of
  // C CTAs per row (up to 8, about 4096 slots each), the row staged across
  // their shared memories. Prefill rows are many: 512 threads a row and a
  // smaller stage, so that several rows run on each SM.
  const int64_t lead = (aligned(scores, 16) && d->S % 4 == 0) ? 0 : 3;
  if (p.mode == dsa::kModePositions && d->S + lead <= 4096) {
    const dsa_status_t rs = d->S + lead <= 2048
                                ? launch_topk_rows<256, 8>(dev, 0, d->T, p, stream)
                                : launch_topk_rows<256, 16>(dev, 1, d->T, p, stream);
    if (rs != DSA_OK) return rs;
    return DSA_OK;
  }
  if (p.mode == dsa::kModePositions) {
    using Sh = dsa::ClusterTopkShared<512>;
    const int C = static_cast<int>(std::min<int64_t>(dsa::kClusterMaxRanks,
                                                     std::max<int64_t>(1, (d->S + 4095) / 4096)));
    if (static_cast<int64_t>(d->T) * C > INT32_MAX) return DSA_ERR_UNSUPPORTED;
    const int64_t room = (kMaxSmemPerBlock - sizeof(Sh) - 1024) / 4;
    p.stage_cap = static_cast<int>(std::min<int64_t>((d->S + C - 1) / C, room));
    const int smem = static_cast<int>(sizeof(Sh) + 4 * static_cast<size_t>(p.stage_cap));
    st = ensure_smem_attr(dev, kAttrTopkCluster, dsa::topk_cluster_kernel<512>, static_cast<int>(kMaxSmemPerBlock));
    if (st != DSA_OK) return st;
    if (launch_pdl(dsa::topk_cluster_kernel<512>, d->T * C, 512, smem, stream, C, p) !=
        cudaSuccess)
      return DSA_ERR_CUDA;
  } else {
    // packed causal rows: the two-pass kernel (its shared memory also holds
    // the general selection's layout, which a crowded threshold bin falls
    // back to)
    constexpr int NT = kCausalTopkThreads;
    p.stage_cap = kCausalTopkStage;
    // the largest of the three layouts: the two-pass selection's and the
    // general one's (each with the stage), the sampled threshold's
    const size_t stage = 4 * static_cast<size_t>(p.stage_cap);
    const int smem = static_cast<int>(
        std::max({((sizeof(dsa::TwoPassShared<NT>) + 15) & ~size_t(15)) + stage,
                  sizeof(dsa::TopkShared<NT>) + stage, sizeof(dsa::SampledShared<NT>)}));
    st = ensure_smem_attr(dev, kAttrTopkCausal, dsa::topk_causal_kernel<NT>,
                          static_cast<int>(kMaxSmemPerBlock));
    if (st != DSA_OK) return st;
    if (launch_pdl(dsa::topk_causal_kernel<NT>, d->T, NT, smem, stream, 0, p) != cudaSuccess)
      return DSA_ERR_CUDA;
  }
  return DSA_OK;
}

dsa_status_t check_inputs(const dsa_indexer_desc_t *d, const void *q, const uint8_t *q_scale,
                          const float *w, const void *k, const uint8_t *k_scale,
                          const int32_t *positions, const float *scores) {
  if (!q || !w || !k || !scores) return DSA_ERR_INVALID_ARG;
  if (!aligned(q, 16) || !aligned(k, 16) || !aligned(w, 16) || !aligned(scores, 4))
    return DSA_ERR_INVALID_ARG;
  if (d->mask == DSA_MASK_POSITIONS && !positions) return DSA_ERR_INVALID_ARG;
  if (d->mask == DSA_MASK_COMPRESSED && positions) return DSA_ERR_INVALID_ARG;
  if (d->dtype == DSA_KV_FP8_E4M3_E8M0_B32 && (!q_scale || !k_scale)) return DSA_ERR_INVALID_ARG;
  return DSA_OK;
}

}  // namespace dsa_host

using namespace dsa_host;

extern "C" {

dsa_status_t dsa_indexer_workspace_size(const dsa_indexer_desc_t *desc, size_t *bytes) {
  if (!bytes) return DSA_ERR_INVALID_ARG;
  dsa_status_t st = check_desc(desc);
  if (st != DSA_OK) return st;
  size_t n = kWorkspaceHeader;
  if (desc->flags & DSA_FLAG_SCORES_IN_WORKSPACE) {
    int64_t elems = 0;
    st = score_elems(desc, &elems);
    if (st != DSA_OK) return st;
    n += static_cast<size_t>(elems) * 4;
  }
  *bytes = n;
  return DSA_OK;
}

dsa_status_t dsa_indexer_score(const dsa_indexer_desc_t *desc, const void *q,
                               const uint8_t *q_scale, const float *w, const void *k,
                               const uint8_t *k_scale, const int32_t *positions,
                               float *scores, void *workspace, size_t workspace_bytes,
                               dsa_stream_t stream) {
  dsa_status_t st = check_desc(desc);
  if (st == DSA_OK) st = check_inputs(desc, q, q_scale, w, k, k_scale, positions, scores);
  if (st == DSA_OK) st = check_workspace(workspace, workspace_bytes);
  if (st != DSA_OK) return st;
  cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
  return launch_score(desc, q, q_scale, w, k, k_scale, positions, scores,
                      static_cast<WsHeader *>(workspace), -1, s);
}

dsa_status_t dsa_indexer_topk(const dsa_indexer_desc_t *desc, const float *scores,
                              const int32_t *positions, int32_t *topk, void *workspace,
                              size_t workspace_bytes, dsa_stream_t stream) {
  dsa_status_t st = check_desc(desc);
  if (st != DSA_OK) return st;
  if (!scores || !topk || !aligned(scores, 4) || !aligned(topk, 4)) return DSA_ERR_INVALID_ARG;
  if (desc->mask == DSA_MASK_POSITIONS && !positions) return DSA_ERR_INVALID_ARG;
  if (desc->mask == DSA_MASK_COMPRESSED && positions) return DSA_ERR_INVALID_ARG;
  st = check_workspace(workspace, workspace_bytes);
  if (st != DSA_OK) return st;
  cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
  return launch_topk(desc, scores, positions, topk, static_cast<WsHeader *>(workspace), true,
                     -1, s);
}

dsa_status_t dsa_indexer_forward(const dsa_indexer_desc_t *desc, const void *q,
                                 const uint8_t *q_scale, const float *w, const void *k,
                                 const uint8_t *k_scale, const int32_t *positions,
                                 float *scores, int32_t *topk, void *workspace,
                                 size_t workspace_bytes, dsa_stream_t stream) {
  dsa_status_t st = check_desc(desc);
  if (st != DSA_OK) return st;
  st = check_workspace(workspace, workspace_bytes);
  if (st != DSA_OK) return st;
  // top-k only: the score rows go to the workspace, which must hold them
  int64_t cap = -1;
  if (!scores) {
    if (!(desc->flags & DSA_FLAG_SCORES_IN_WORKSPACE)) return DSA_ERR_INVALID_ARG;
    int64_t elems = 0;
    st = score_elems(desc, &elems);
    if (st != DSA_OK) return st;
    cap = workspace_scores(workspace, workspace_bytes, &scores);
    if (cap < elems) return DSA_ERR_WORKSPACE;
  }
  st = check_inputs(desc, q, q_scale, w, k, k_scale, positions, scores);
  if (st == DSA_OK && (!topk || !aligned(topk, 4))) st = DSA_ERR_INVALID_ARG;
  if (st != DSA_OK) return st;
  cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
  WsHeader *ws = static_cast<WsHeader *>(workspace);
  st = launch_score(desc, q, q_scale, w, k, k_scale, positions, scores, ws, cap, s);
  if (st != DSA_OK) return st;
  return launch_topk(desc, scores, positions, topk, ws, false, cap, s);
}

dsa_status_t dsa_indexer_get_error(const void *workspace, dsa_stream_t stream,
                                   dsa_status_t *device_status) {
  if (!workspace || !device_status || !aligned(workspace, 256)) return DSA_ERR_INVALID_ARG;
  cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
  unsigned int err = 0;
  if (cudaMemcpyAsync(&err, workspace, sizeof err, cudaMemcpyDeviceToHost, s) != cudaSuccess ||
      cudaStreamSynchronize(s) != cudaSuccess)
    return DSA_ERR_CUDA;
  // read and clear: the next report starts from a clean status
  if (err != 0 && (cudaMemsetAsync(const_cast<void *>(workspace), 0, 2 * sizeof err, s) !=
                       cudaSuccess ||
                   cudaStreamSynchronize(s) != cudaSuccess))
    return DSA_ERR_CUDA;
  *device_status = err == 0 ? DSA_OK : static_cast<dsa_status_t>(err);
  return DSA_OK;
}

const char *dsa_status_string(dsa_status_t status) {
  switch (status) {
    case DSA_OK: return "DSA_OK";
    case DSA_ERR_INVALID_ARG: return "DSA_ERR_INVALID_ARG";
    case DSA_ERR_UNSUPPORTED: return "DSA_ERR_UNSUPPORTED";
    case DSA_ERR_WORKSPACE: return "DSA_ERR_WORKSPACE";
    case DSA_ERR_CUDA: return "DSA_ERR_CUDA";
    case DSA_ERR_TIMEOUT: return "DSA_ERR_TIMEOUT";
    case DSA_ERR_DEVICE: return "DSA_ERR_DEVICE";
  }
  return "DSA_ERR_UNKNOWN";
}

}  // extern "C"
