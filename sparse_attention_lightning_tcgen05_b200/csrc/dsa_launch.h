// dsa_launch.h -- host-side helpers shared by the C entry points: argument
// checks and the launches of the score and top-k kernels (definitions in
// dsa_indexer_api.cu).
#pragma once

#include <cuda_runtime.h>

#include <cstddef>
#include <cstdint>

#include "dsa_indexer.h"

namespace dsa_host {

constexpr size_t kWorkspaceHeader = 256;   // bytes of workspace every call needs

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
