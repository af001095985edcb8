/*
 * dsa_indexer.h -- C ABI of libdsa_indexer, the DeepSeek Sparse Attention
 * lightning indexer (scores + top-k) for NVIDIA B200 (sm_100a).
 *
 * For every query token t and every key slot s of its key cache:
 *     I[t,s] = sum_h w[t,h] * ReLU(q[t,h,:] . k[s,:])      if valid(t,s)
 *     I[t,s] = DSA_MASK_BOUND                               otherwise
 * and, per token, an unordered set of index_topk slot positions holding the
 * largest valid scores (-1 where the row has fewer valid slots than
 * index_topk).
 *
 * Where the operation is defined (page titles and sections):
 *  - DeepSeek-V3.2 Sparse Indexer Kernel API Reference, deepseek_v32_sparse_
 *    indexer: "score every cached key slot against the current query and
 *    select the highest scoring ones"; parameters key_cache [n_tokens,
 *    max_seq_len, head_dim] (one cache per sequence), positions [n_tokens]
 *    int32 (absolute position of each sequence's current token),
 *    index_topk; returns [n_tokens, max_seq_len] fp32 scores with slots the
 *    token cannot attend to clamped to the mask bound, and [n_tokens,
 *    index_topk] int32 positions; Notes: the top-k output is an unordered
 *    set; the mask bound is finite rather than -inf because a bf16 consumer
 *    reads it; Dimensions: head_dim must equal 128.
 *  - Sparse Attention Indexer MX BF16Score Kernel API Reference: phase "all"
 *    scores the S queries of a sequence against its own keys (queries ==
 *    keys); scores [B*S, end_pos] f32; top-k positions are 0-based in
 *    [0, end_pos); block-32 e8m0 scales (qr_scale_hbm, wq_b_scale, wk_scale)
 *    for the MX (fp8-e4m3) format; Notes: the bf16 score path drops the
 *    Hadamard rotation because it is a no-op for q . k.
 *  - NeMo AutoModel optimized_kernels, sparse_attention_torch: a key index of
 *    -1 masks an entry.
 *  - tokamax Supported Ops, lightning_indexer: the scores run over a paged
 *    KV cache. This library reads it as one pool of pages and a block table
 *    with one row per query token (see block_table below).
 *  - NeMo AutoModel optimized_kernels, dsv4_indexer_scores and
 *    indexer_scores_torch: the DSV4 "C4" indexer scores queries against a
 *    pooled (compressed) key cache, given compress_ratio and query_start.
 *    The page gives the arguments, not the causal rule in pooled space; this
 *    library reads it as: pooled slot j holds raw tokens [j*r, (j+1)*r) and
 *    is valid for the query at absolute position query_start + t once all of
 *    them have been seen, (j+1)*r <= query_start + t + 1. The softmax_scale
 *    argument is a scalar factor of every score: fold it into w.
 *
 * Conventions common to every call:
 *  - Pointers are DEVICE pointers unless stated otherwise. The caller owns
 *    every buffer and the stream. The library allocates no memory, keeps no
 *    per-call state between calls, and never synchronises the stream (except
 *    dsa_indexer_get_error).
 *  - Argument checks run on the host before any launch; a failed check
 *    returns DSA_ERR_INVALID_ARG / DSA_ERR_UNSUPPORTED / DSA_ERR_WORKSPACE and
 *    launches nothing. A failed launch returns DSA_ERR_CUDA.
 *  - Kernels never trap. A device-side wait that runs past its time limit
 *    (desc->wait_limit_ns, default 4 s) makes the kernel stop, record
 *    DSA_ERR_TIMEOUT in the workspace and exit cleanly after the copies and
 *    MMAs it has in flight have landed (those drains have a bound of their
 *    own, 4 s, whatever the wait limit); read it with dsa_indexer_get_error.
 *  - CAUSAL: cu_seqlens is checked on the device before any score or top-k
 *    is written (cu[0] = 0, non-decreasing, cu[num_seqs] = T). A bad array
 *    makes the kernels of that call write nothing and records
 *    DSA_ERR_INVALID_ARG in the workspace (dsa_indexer_get_error).
 *  - A workspace belongs to one in-flight call at a time: two calls on
 *    different streams must not share one.
 */
#ifndef DSA_INDEXER_H
#define DSA_INDEXER_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef struct CUstream_st *dsa_stream_t;   /* == cudaStream_t; NULL = legacy default */

typedef enum {
  DSA_OK = 0,
  DSA_ERR_INVALID_ARG = 1,   /* a null pointer, a bad size, misaligned buffer */
  DSA_ERR_UNSUPPORTED = 2,   /* valid but not implemented (e.g. D != 128)    */
  DSA_ERR_WORKSPACE = 3,     /* workspace missing, misaligned or too small    */
  DSA_ERR_CUDA = 4,          /* a CUDA runtime call or a launch failed        */
  DSA_ERR_TIMEOUT = 5,       /* a device-side wait ran past its limit         */
  DSA_ERR_DEVICE = 6         /* the current device is not sm_100 (B200)       */
} dsa_status_t;

typedef enum {
  DSA_KV_BF16 = 0,               /* q, k bf16                                   */
  DSA_KV_FP8_E4M3_E8M0_B32 = 1   /* q, k fp8-e4m3 with one e8m0 scale byte per
                                    32 consecutive elements along D             */
} dsa_kv_dtype_t;

typedef enum {
  DSA_MASK_POSITIONS = 0,  /* decode: token t reads cache t (or the one shared
                              cache); slot s valid iff s <= positions[t];
                              every score row has S entries                    */
  DSA_MASK_CAUSAL = 1,     /* packed prefill: sequences back to back as given
                              by cu_seqlens; token t of sequence i scores the
                              L_i keys of its own sequence; slot s valid iff
                              s <= t - cu_seqlens[i]                           */
  DSA_MASK_COMPRESSED = 2  /* C4 indexer: every token scores the one pooled
                              cache of S slots, each pooling compress_ratio
                              raw tokens; token t sits at absolute position
                              query_start + t and slot s is valid iff
                              (s+1)*compress_ratio <= query_start + t + 1;
                              every score row has S entries                    */
} dsa_mask_t;

/* The finite mask bound: the lowest finite bf16 value (bits 0xFF7F), exact
 * in fp32 (bits 0xFF7F0000). */
#define DSA_MASK_BOUND (-3.38953138925153547590470800371487866880e+38f)

typedef struct {
  int32_t T;               /* query tokens (rows), >= 1                          */
  int32_t H;               /* indexer heads, 1 <= H <= 256                       */
  int32_t D;               /* head_dim; must be 128                              */
  int32_t index_topk;      /* k >= 1                                             */
  int64_t S;               /* POSITIONS: slots per key cache, >= 1.
                              COMPRESSED: pooled slots, >= 1. CAUSAL: unused     */
  int64_t k_seq_stride;    /* POSITIONS: elements between consecutive tokens'
                              caches (a multiple of D, >= S*D), or 0 when every
                              token reads one shared cache. COMPRESSED: must be
                              0 (one pooled cache). CAUSAL: unused              */
  int32_t num_seqs;        /* CAUSAL: packed sequences, >= 1. POSITIONS: unused   */
  const int32_t *cu_seqlens; /* CAUSAL: device [num_seqs + 1], cu[0] = 0,
                              non-decreasing, cu[num_seqs] = T                  */
  dsa_kv_dtype_t dtype;
  dsa_mask_t mask;
  int64_t query_start;     /* COMPRESSED: absolute position of token 0, >= 0;
                              query_start + T <= INT32_MAX (positions are 32-bit
                              as in POSITIONS; DSA_ERR_UNSUPPORTED otherwise).
                              Otherwise unused                                  */
  int32_t compress_ratio;  /* COMPRESSED: raw tokens per pooled slot, >= 1.
                              Otherwise unused                                  */
  int32_t page_size;       /* paged POSITIONS cache (block_table != NULL): slots
                              per page, a power of two in [16, 65536]            */
  int32_t pages_per_seq;   /* paged: block-table entries per token, >= 1, with
                              S <= pages_per_seq * page_size                    */
  int32_t num_pages;       /* paged: pages in the pool k points to, >= 1        */
  const int32_t *block_table; /* NULL: not paged. Paged (POSITIONS,
                              k_seq_stride 0): device [T, pages_per_seq] int32;
                              token t's slot s is row s % page_size of page
                              block_table[t*pages_per_seq + s/page_size] of the
                              pool k [num_pages, page_size, D] (FP8: and of the
                              scale pool k_scale [num_pages, page_size, D/32],
                              the same page ids). Entries of pages
                              that hold a valid slot must lie in
                              [0, num_pages); other entries are never used for
                              a score (a page id outside the pool reads as 0)  */
  uint32_t flags;          /* DSA_FLAG_* bits, 0 for none                       */
  uint64_t wait_limit_ns;  /* time limit of any single device-side wait; 0 =
                              the default, 4 s. A wait that runs past it stops
                              the kernel with DSA_ERR_TIMEOUT (see
                              dsa_indexer_get_error)                            */
  const int32_t *cu_seqlens_host; /* CAUSAL with DSA_FLAG_SCORES_IN_WORKSPACE:
                              a HOST copy of cu_seqlens [num_seqs + 1], read by
                              dsa_indexer_workspace_size to size the score rows
                              (the kernels still read the device array). May be
                              NULL otherwise                                   */
} dsa_indexer_desc_t;

/* flags */
/* Top-k only: dsa_indexer_workspace_size adds room for every score row
 * (after the 256-byte header), and dsa_indexer_forward accepts scores = NULL,
 * keeping the rows in the workspace, where they are overwritten by the next
 * call. The index set is the product; the scores are the consumer's optional
 * by-product (DeepSeek-V3.2 Sparse Indexer Kernel API Reference, Returns). */
#define DSA_FLAG_SCORES_IN_WORKSPACE 1u
/* Self-test of the failure path: the score kernel's MMA warp first waits on a
 * barrier that nothing completes. The wait runs out after wait_limit_ns, the
 * kernel records DSA_ERR_TIMEOUT, lets its in-flight copies land and exits
 * with no output written past that point; dsa_indexer_get_error then reports
 * the timeout. For tests of a caller's error handling: nothing faults. */
#define DSA_FLAG_SELFTEST_STALL 2u

/*
 * Layouts (all row-major, innermost index last, no padding):
 *  q        [T, H, D]      bf16, or e4m3 bytes                 (16-byte aligned)
 *  q_scale  [T, H, D/32]   e8m0 bytes (FP8 only; NULL for BF16)
 *  w        [T, H]         fp32
 *  k        POSITIONS: cache of token t at element t*k_seq_stride, [S, D];
 *           paged: the page pool [num_pages, page_size, D]
 *           COMPRESSED: the pooled cache [S, D]
 *           CAUSAL:    [T, D], sequence i at rows cu[i] .. cu[i+1]-1
 *           bf16, or e4m3 bytes                                 (16-byte aligned)
 *  k_scale  same slots as k, [.., D/32] e8m0 bytes (FP8 only; NULL for BF16);
 *           POSITIONS cache t at byte t*(k_seq_stride/32); paged: the scale
 *           page pool [num_pages, page_size, D/32]          (16-byte aligned)
 *  positions [T] int32 (POSITIONS only; ignored for CAUSAL; must be NULL
 *           for COMPRESSED). A negative position leaves the whole row masked.
 *  scores   POSITIONS, COMPRESSED: [T, S] fp32 (a COMPRESSED row that sees
 *           no pooled slot is all mask bound, its top-k all -1).
 *           CAUSAL: sequence i's [L_i, L_i] block at float offset
 *           sum_{j<i} L_j^2; row t of it at + (t - cu[i]) * L_i.
 *  topk     [T, index_topk] int32, sequence-local 0-based slot indices in any
 *           order, -1 padded at the end of the row.
 * Scores must hold no NaN when passed to dsa_indexer_topk.
 */

/* Bytes of workspace every call needs (host only; no device work): a
 * 256-byte header, plus, with DSA_FLAG_SCORES_IN_WORKSPACE, the score rows
 * (4 * T * S bytes; CAUSAL: 4 * sum_i L_i^2 from cu_seqlens_host, which must
 * then be given). The workspace is device memory, 256-byte aligned and owned
 * by the caller. It must be zero-filled once before its first use (e.g.
 * cudaMemsetAsync); each call leaves it ready for the next, so it is reused
 * freely between calls that are ordered on the GPU (one stream). */
dsa_status_t dsa_indexer_workspace_size(const dsa_indexer_desc_t *desc,
                                        size_t *bytes);

/* Scores only: writes every score row (valid slots and mask bound).
 * Asynchronous on `stream`. */
dsa_status_t dsa_indexer_score(const dsa_indexer_desc_t *desc,
                               const void *q, const uint8_t *q_scale,
                               const float *w, const void *k,
                               const uint8_t *k_scale,
                               const int32_t *positions, float *scores,
                               void *workspace, size_t workspace_bytes,
                               dsa_stream_t stream);

/* Top-k only, from score rows laid out as above (by this library or not);
 * validity comes from positions / cu_seqlens / the compressed rule, never
 * from the values.
 * Ties at the k-th score go to the lower slot. Asynchronous on `stream`. */
dsa_status_t dsa_indexer_topk(const dsa_indexer_desc_t *desc,
                              const float *scores, const int32_t *positions,
                              int32_t *topk, void *workspace,
                              size_t workspace_bytes, dsa_stream_t stream);

/* dsa_indexer_score followed by dsa_indexer_topk on the same stream.
 * scores = NULL (top-k only) needs DSA_FLAG_SCORES_IN_WORKSPACE and a
 * workspace of the size dsa_indexer_workspace_size reports for it; the rows
 * then live in the workspace (DSA_ERR_WORKSPACE when it is too small,
 * DSA_ERR_INVALID_ARG without the flag). */
dsa_status_t dsa_indexer_forward(const dsa_indexer_desc_t *desc,
                                 const void *q, const uint8_t *q_scale,
                                 const float *w, const void *k,
                                 const uint8_t *k_scale,
                                 const int32_t *positions, float *scores,
                                 int32_t *topk, void *workspace,
                                 size_t workspace_bytes, dsa_stream_t stream);

/* Forward pass (scores + top-k, as dsa_indexer_forward) that allocates
 * nothing and takes no workspace. The pages have no counterpart: this entry
 * point serves callers that cannot allocate device memory when they run the
 * indexer (an engine plugin handed only its inputs and outputs, a runtime
 * with a fixed memory pool, a path where an allocation could synchronise the
 * device). The kernels' scratch words live in a fixed 4096-byte array inside
 * the library, held by every GPU that loads it until the process exits; a
 * problem whose workspace size exceeds it returns DSA_ERR_WORKSPACE. The
 * first call on a device looks up that array's address (do it before any
 * stream capture); the address is kept for the life of the process, so a
 * cudaDeviceReset after that first call is not supported. Every call clears the scratch on `stream`; all calls share
 * it, so calls that overlap on the GPU race and must be serialised by the
 * caller. Device-side timeouts are not reported by this entry point. */
dsa_status_t dsa_indexer_forward_noalloc(const dsa_indexer_desc_t *desc,
                                         const void *q, const uint8_t *q_scale,
                                         const float *w, const void *k,
                                         const uint8_t *k_scale,
                                         const int32_t *positions,
                                         float *scores, int32_t *topk,
                                         dsa_stream_t stream);

/* Synchronises `stream`, then reports in *device_status the first
 * device-side failure (DSA_ERR_TIMEOUT) recorded in `workspace` since the
 * previous dsa_indexer_get_error on it, or DSA_OK, and clears it. Returns
 * DSA_ERR_CUDA if the synchronisation or the read failed. */
dsa_status_t dsa_indexer_get_error(const void *workspace, dsa_stream_t stream,
                                   dsa_status_t *device_status);

/* A static, human-readable name of a status code. */
const char *dsa_status_string(dsa_status_t status);

#ifdef __cplusplus
}
#endif

#endif /* DSA_INDEXER_H */
