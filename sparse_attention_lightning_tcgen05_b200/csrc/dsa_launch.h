// dsa_launch.h -- host-side helpers shared by the C entry points: argument
// checks and the launches of the score and top-k kernels (definitions in
// dsa_indexer_api.cu).
#pragma once

#include <cuda.h>
#include <cuda_runtime.h>

#include <cstddef>
#include <cstdint>
#include <utility>

#include "dsa_indexer.h"

namespace dsa_host {

constexpr size_t kWorkspaceHeader = 256;   // bytes of workspace every call needs

// Bits of DeviceInfo::attr_done: one per kernel whose dynamic shared-memory
// limit is raised (the score kernel's instances take 0 .. 15). Every kernel
// needs its own bit: a shared one would skip another kernel's attribute.
enum : uint32_t {
  kAttrTopkRows8 = 16,
  kAttrTopkRows16 = 17,
  kAttrTopkCluster = 18,
  kAttrTopkCausal = 19,
  kAttrSparseMqa = 20,
  kAttrPrepare = 21,
};

// What the library knows about a device (probed once per device).
struct DeviceInfo {
  bool probed = false;
  bool ok = false;
  int num_sms = 0;
  uint32_t attr_done = 0;   // bit per kernel whose smem attribute is set
};

// The current device's info (sm_100 check, SM count, tensor-map encoder).
dsa_status_t device_info(DeviceInfo **out);
// Raise a kernel's dynamic shared-memory limit once per device (bit: which).
dsa_status_t ensure_smem_attr_raw(DeviceInfo *d, uint32_t bit, const void *kernel, int bytes);
template <typename K>
dsa_status_t ensure_smem_attr(DeviceInfo *d, uint32_t bit, K kernel, int bytes) {
  return ensure_smem_attr_raw(d, bit, reinterpret_cast<const void *>(kernel), bytes);
}
// A tiled TMA tensor map (DSA_ERR_INVALID_ARG when the driver rejects it).
dsa_status_t make_map(CUtensorMap *m, CUtensorMapDataType dt, cuuint32_t rank, const void *base,
                      const cuuint64_t *dims, const cuuint64_t *strides_bytes,
                      const cuuint32_t *box,
                      CUtensorMapSwizzle swz = CU_TENSOR_MAP_SWIZZLE_128B);

inline bool aligned(const void *p, uintptr_t a) {
  return (reinterpret_cast<uintptr_t>(p) & (a - 1)) == 0;
}

// Launch with programmatic stream serialisation: the kernel may start while
// the previous kernel on the stream is finishing; each kernel calls
// griddepcontrol.wait before it touches memory that earlier work wrote.
// `cluster` > 0 launches thread-block clusters of that many CTAs along x.
template <typename... KArgs, typename... Args>
cudaError_t launch_pdl(void (*kernel)(KArgs...), int grid, int threads, size_t smem,
                       cudaStream_t stream, int cluster, Args &&...args) {
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(static_cast<unsigned>(grid));
  cfg.blockDim = dim3(static_cast<unsigned>(threads));
  cfg.dynamicSmemBytes = smem;
  cfg.stream = stream;
  cudaLaunchAttribute attr[2];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  if (cluster > 0) {
    attr[1].id = cudaLaunchAttributeClusterDimension;
    attr[1].val.clusterDim.x = static_cast<unsigned>(cluster);
    attr[1].val.clusterDim.y = 1;
    attr[1].val.clusterDim.z = 1;
    cfg.numAttrs = 2;
  }
  const cudaError_t e = cudaLaunchKernelEx(&cfg, kernel, std::forward<Args>(args)...);
  // a launch this library failed is reported through its status: consume the
  // error so that it is not mistaken for a later call's
  if (e != cudaSuccess) (void)cudaGetLastError();
  return e;
}

struct WsHeader;

dsa_status_t check_desc(const dsa_indexer_desc_t *d);
dsa_status_t check_inputs(const dsa_indexer_desc_t *d, const void *q, const uint8_t *q_scale,
                          const float *w, const void *k, const uint8_t *k_scale,
                          const int32_t *positions, const float *scores);
// cap_elems: floats the score buffer is known to hold (a top-k-only call's
// workspace), or -1 when the caller's buffer is used. launch_score runs the
// CAUSAL cu_seqlens check first; launch_topk runs it when check_cu is set
// (a top-k call of its own).
dsa_status_t launch_score(const dsa_indexer_desc_t *d, const void *q, const uint8_t *q_scale,
                          const float *w, const void *k, const uint8_t *k_scale,
                          const int32_t *positions, float *scores, WsHeader *ws,
                          int64_t cap_elems, cudaStream_t stream);
dsa_status_t launch_topk(const dsa_indexer_desc_t *d, const float *scores,
                         const int32_t *positions, int32_t *topk, WsHeader *ws, bool check_cu,
                         int64_t cap_elems, cudaStream_t stream);

}  // namespace dsa_host
