/*
 * dsa_sparse_mqa.h -- C ABI of the lightning indexer's consumer in
 * libdsa_indexer: sparse multi-query attention over the top-k key indices,
 * with per-head attention sinks, for NVIDIA B200 (sm_100a).
 *
 * For every query token (b, s) and head h, with t = b*S + s:
 *     l_j = sm_scale * q[b,s,h,:] . kv[b, idx_j, :]     for every kept entry
 *                                                        idx_j of topk[b,s,:]
 *     out[b,s,h,:] = sum_j e^{l_j} kv[b, idx_j, :]
 *                    / (sum_j e^{l_j} + e^{sinks[h]})
 * An entry that is -1, negative or >= K is masked (it takes no part); a
 * token with no kept entry gets out = 0. The single kv head is both key and
 * value (multi-query attention over one latent head).
 *
 * Where the operation is defined (page titles and sections):
 *  - NeMo AutoModel optimized_kernels, sparse_attention_torch ("sparse MQA")
 *    and dense_attention_topk_torch: q [B, S, H, D], single-head kv
 *    [B, K, D], per-head sink logits sinks [H], key indices topk_idxs
 *    [B, S, K_top] where -1 masks an entry, sm_scale.
 *  - The DeepSeek-V4 NVFP4 inference kernel write-up, sparse attention
 *    section: keys gathered by index, an out-of-range entry padded to -1
 *    and scored -inf, an online softmax whose denominator gains
 *    exp(attn_sink - max) at the end.
 *
 * Conventions are those of dsa_indexer.h: device pointers unless stated
 * otherwise, no allocation, host-side argument checks before any launch,
 * bounded device-side waits whose failures are recorded in the workspace
 * and read with dsa_indexer_get_error (the workspace header is the same).
 */
#ifndef DSA_SPARSE_MQA_H
#define DSA_SPARSE_MQA_H

#include "dsa_indexer.h"

#ifdef __cplusplus
extern "C" {
#endif

typedef struct {
  int32_t B;               /* batches, >= 1                                     */
  int32_t S;               /* query tokens per batch, >= 1 (B*S*H < 2^31)       */
  int32_t H;               /* heads, 1 <= H <= 128                               */
  int32_t D;               /* head dim; must be 128                             */
  int64_t K;               /* kv rows per batch, >= 1                           */
  int32_t K_top;           /* index entries per token, >= 1                     */
  float sm_scale;          /* logit scale (finite)                              */
  uint64_t wait_limit_ns;  /* device-side wait limit; 0 = the default, 4 s      */
} dsa_sparse_mqa_desc_t;

/*
 * Layouts (row-major, innermost index last, no padding):
 *  q     [B, S, H, D]   bf16                                  (16-byte aligned)
 *  kv    [B, K, D]      bf16                                  (16-byte aligned)
 *  sinks [H]            fp32
 *  topk  [B, S, K_top]  int32 (e.g. dsa_indexer_forward's index sets)
 *  out   [B, S, H, D]   bf16                                  (16-byte aligned)
 */

/* Bytes of workspace a call needs (host only): the 256-byte header, plus,
 * when there are too few query tokens to fill the GPU and every token's
 * index row is split into ranges, the ranges' partial results
 * (fp32, 4 * B*S * ranges * H * (D + 2) bytes). 256-byte aligned, zero-filled
 * once before first use, reused freely by calls ordered on one stream. */
dsa_status_t dsa_sparse_mqa_workspace_size(const dsa_sparse_mqa_desc_t *desc,
                                           size_t *bytes);

/* out = sparse MQA of q over the kv rows topk selects. Asynchronous on
 * `stream`. Device-side timeouts: dsa_indexer_get_error(workspace). */
dsa_status_t dsa_sparse_mqa_forward(const dsa_sparse_mqa_desc_t *desc,
                                    const void *q, const void *kv,
                                    const float *sinks, const int32_t *topk,
                                    void *out, void *workspace,
                                    size_t workspace_bytes, dsa_stream_t stream);

#ifdef __cplusplus
}
#endif

#endif /* DSA_SPARSE_MQA_H */
