/*
 * dsa_prepare.h -- C ABI of the lightning indexer's front end in
 * libdsa_indexer, for NVIDIA B200 (sm_100a): the query, key and head-weight
 * projections that produce the indexer's inputs, with the key written into
 * the key cache.
 *
 * Per query token t:
 *     q[t, h, :] = rope(qr[t, :] . wq_b[h*D .. h*D + D - 1, :]^T, t)
 *     k          = rope(layernorm(x[t, :] . wk^T), t)   written to the cache
 *     w[t, :]    = w_scale * (x[t, :] . weights_proj^T)
 * rope(v, t) turns every interleaved pair (v[2i], v[2i+1]), i < rope_dim/2,
 * by the angle whose cosine and sine are cos[t, i], sin[t, i]:
 *     (v[2i] cos - v[2i+1] sin,  v[2i] sin + v[2i+1] cos);
 * features from rope_dim on are unchanged. layernorm(v) = (v - mean) /
 * sqrt(var + eps) * k_norm_weight + k_norm_bias over the D features (biased
 * variance). q and k are then what dsa_indexer_score reads.
 *
 * Where the operation is defined (page titles and sections):
 *  - DeepSeek-V3.2 Sparse Indexer Kernel API Reference,
 *    deepseek_v32_sparse_indexer, Parameters: hidden_states [n_tokens,
 *    hidden]; qr [n_tokens, q_lora_rank] = q_norm(wq_a(x)) from the MLA
 *    block; wq_b, the query projection; wk [hidden, head_dim];
 *    k_norm_weight / k_norm_bias, fp32 LayerNorm gain and bias of the key;
 *    weights_proj [hidden, n_heads]; cos / sin [n_tokens, rope_dim // 2];
 *    key_cache written in place at each token's current position;
 *    rope_dim, the leading feature span RoPE rotates.
 *  - tokamax Supported Ops, deepseek_rope: DeepSeek's RoPE is interleaved.
 *  - Sparse Attention Indexer MX BF16Score Kernel API Reference, Notes: the
 *    bf16 score path leaves out the Hadamard rotation (q_H . k_H = q . k)
 *    and the MX quantisation it serves; so does this front end.
 * Readings where the pages are silent: weights are stored [out_features,
 * in_features] with the contraction contiguous (wq_b [H*D, q_lora_rank],
 * wk [D, hidden], weights_proj [H, hidden]); wq_b's output features are head
 * major; all projections are bf16 with fp32 accumulation; the head weights
 * carry one scalar factor w_scale (fold the softmax scale into it).
 *
 * Conventions are those of dsa_indexer.h (device pointers, no allocation,
 * host-side checks before any launch, bounded device waits recorded in the
 * workspace and read with dsa_indexer_get_error).
 */
#ifndef DSA_PREPARE_H
#define DSA_PREPARE_H

#include "dsa_indexer.h"

#ifdef __cplusplus
extern "C" {
#endif

typedef struct {
  int32_t T;               /* query tokens, >= 1                                */
  int32_t H;               /* indexer heads: a multiple of 16 in [16, 128]      */
  int32_t D;               /* head dim; must be 128                            */
  int32_t hidden;          /* model hidden width: a multiple of 64, >= 64       */
  int32_t q_lora_rank;     /* query LoRA rank: a multiple of 64, >= 64          */
  int32_t rope_dim;        /* leading features RoPE turns: even, 0 .. D         */
  float k_norm_eps;        /* LayerNorm epsilon, >= 0                          */
  float w_scale;           /* factor of the head weights                       */
  int64_t S;               /* slots per key cache: a position outside [0, S)
                              writes no key                                    */
  int64_t k_seq_stride;    /* elements between consecutive tokens' caches, or 0
                              when every token writes one shared cache          */
  uint64_t wait_limit_ns;  /* device-side wait limit; 0 = the default, 4 s      */
} dsa_prepare_desc_t;

/*
 * Layouts (row-major, innermost index last; the 16-byte alignment rules of
 * TMA apply to x, qr and the three weights):
 *  x            [T, hidden]          bf16                  (16-byte aligned)
 *  qr           [T, q_lora_rank]     bf16                  (16-byte aligned)
 *  wq_b         [H*D, q_lora_rank]   bf16                  (16-byte aligned)
 *  wk           [D, hidden]          bf16                  (16-byte aligned)
 *  weights_proj [H, hidden]          bf16                  (16-byte aligned)
 *  k_norm_weight, k_norm_bias [D]    fp32
 *  cos, sin     [T, rope_dim/2]      fp32 (may be NULL when rope_dim = 0)
 *  positions    [T] int32, or NULL: token t's key goes to slot t
 *  q_out        [T, H, D]            bf16                  (16-byte aligned)
 *  w_out        [T, H]               fp32
 *  key_cache    token t's key row at element t*k_seq_stride + pos*D, bf16
 *                                                          (16-byte aligned)
 */

/* Bytes of workspace a call needs (host only): the 256-byte header, plus the
 * fp32 partial rows of a projection whose K range is split over the SMs (too
 * few tokens to fill the GPU). 256-byte aligned, zero-filled once. */
dsa_status_t dsa_indexer_prepare_workspace_size(const dsa_prepare_desc_t *desc,
                                                size_t *bytes);

/* The three projections and their epilogues, asynchronous on `stream`. */
dsa_status_t dsa_indexer_prepare(const dsa_prepare_desc_t *desc, const void *x,
                                 const void *qr, const void *wq_b, const void *wk,
                                 const void *weights_proj,
                                 const float *k_norm_weight,
                                 const float *k_norm_bias, const float *cos,
                                 const float *sin, const int32_t *positions,
                                 void *q_out, float *w_out, void *key_cache,
                                 void *workspace, size_t workspace_bytes,
                                 dsa_stream_t stream);

#ifdef __cplusplus
}
#endif

#endif /* DSA_PREPARE_H */
