// dsa_indexer_noalloc.cu -- dsa_indexer_forward_noalloc: the forward pass
// for callers that cannot hand the library a workspace.
//
// Some hosts of this code cannot call cudaMalloc (or any allocator) at the
// point where they run the indexer: an inference-engine plugin that is given
// only its input and output buffers, a runtime that owns a fixed device
// memory pool and forbids allocations after start-up, or a path that must not
// allocate because allocation can synchronise the device. This entry point
// runs the same score and top-k kernels as dsa_indexer_forward, but the
// scratch words those kernels need (the device-side error word and site) live
// in a fixed array compiled into the library instead of a caller workspace.
//
// The array is a file-scope __device__ variable of kNoAllocScratchBytes: every
// GPU that loads the library holds it until the process exits. Host code never
// uses its name as an address; the device address is looked up once per
// device with cudaGetSymbolAddress, on the first call made with that device
// current, so that first call should come before any stream capture. The
// address is kept for the life of the process: a cudaDeviceReset after the
// first call (which unloads the library's module) is not supported. All calls
// share the array: calls that overlap on the GPU (different streams, or
// different host threads on one device) race on it and must be serialised by
// the caller. Each call clears the scratch on its stream before the kernels
// run. Device-side timeouts of this entry point are not reported (the kernels
// still stop cleanly); use dsa_indexer_forward with a workspace to read them.
#include <cuda_runtime.h>

#include <cstdint>
#include <mutex>

#include "dsa_indexer.h"
#include "dsa_launch.h"

namespace {

constexpr size_t kNoAllocScratchBytes = 4096;
constexpr int kMaxDevices = 64;

static __device__ __align__(256) unsigned char g_noalloc_scratch[kNoAllocScratchBytes];

std::mutex g_mu;
void *g_scratch_ptr[kMaxDevices] = {};

// Device address of g_noalloc_scratch on the current device (looked up once
// per device, with that device current).
dsa_status_t scratch_address(void **out) {
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) return DSA_ERR_CUDA;
  std::lock_guard<std::mutex> lk(g_mu);
  if (g_scratch_ptr[dev] == nullptr) {
    void *p = nullptr;
    if (cudaGetSymbolAddress(&p, g_noalloc_scratch) != cudaSuccess || p == nullptr)
      return DSA_ERR_CUDA;
    g_scratch_ptr[dev] = p;
  }
  *out = g_scratch_ptr[dev];
  return DSA_OK;
}

}  // namespace

extern "C" dsa_status_t dsa_indexer_forward_noalloc(
    const dsa_indexer_desc_t *desc, const void *q, const uint8_t *q_scale, const float *w,
    const void *k, const uint8_t *k_scale, const int32_t *positions, float *scores,
    int32_t *topk, dsa_stream_t stream) {
  dsa_status_t st = dsa_host::check_desc(desc);
  if (st == DSA_OK)
    st = dsa_host::check_inputs(desc, q, q_scale, w, k, k_scale, positions, scores);
  if (st == DSA_OK && (!topk || (reinterpret_cast<uintptr_t>(topk) & 3u) != 0))
    st = DSA_ERR_INVALID_ARG;
  if (st != DSA_OK) return st;
  size_t need = 0;
  st = dsa_indexer_workspace_size(desc, &need);
  if (st != DSA_OK) return st;
  if (need > kNoAllocScratchBytes) return DSA_ERR_WORKSPACE;   // beyond the fixed scratch
  void *scratch = nullptr;
  st = scratch_address(&scratch);
  if (st != DSA_OK) return st;
  cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
  if (cudaMemsetAsync(scratch, 0, need, s) != cudaSuccess) return DSA_ERR_CUDA;
  dsa_host::WsHeader *ws = static_cast<dsa_host::WsHeader *>(scratch);
  st = dsa_host::launch_score(desc, q, q_scale, w, k, k_scale, positions, scores, ws, -1, s);
  if (st != DSA_OK) return st;
  return dsa_host::launch_topk(desc, scores, positions, topk, ws, false, -1, s);
}
