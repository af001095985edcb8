/*
 * dsa_oracle.c -- plain fp64 CPU oracle of the DeepSeek Sparse Attention
 * lightning indexer (scores + top-k).
 *
 * TEST INFRASTRUCTURE. Only the tests, the smoke check and the benchmark's
 * CPU-baseline leg use this file. It shares no code, header or table with the
 * CUDA library, and the library never calls it.
 *
 * What it computes, for every query row t and every key slot s of the row's
 * key cache:
 *     I[t,s] = sum_h w[t,h] * max(0, sum_d q[t,h,d] * k[s,d])   if valid(t,s)
 *     I[t,s] = MASK_BOUND                                        otherwise
 * and per row the set of the min(index_topk, nvalid) valid slots with the
 * largest I, padded with -1.
 *
 * Sources (page titles and sections):
 *  - DeepSeek-V3.2 Sparse Indexer Kernel API Reference, "deepseek_v32_sparse_
 *    indexer": every cached key slot is scored against the step's query; the
 *    key cache is [n_tokens, max_seq_len, head_dim] and is written at each
 *    token's current position, positions[] is the absolute position of each
 *    sequence's current token; the score output is [n_tokens, max_seq_len]
 *    fp32 with slots the token cannot attend to clamped to a mask bound; the
 *    top-k output is [n_tokens, index_topk] int32 and is an unordered set;
 *    Notes: the mask bound is finite (not -inf) because a bf16 consumer reads it.
 *  - Sparse Attention Indexer MX BF16Score Kernel API Reference: head_dim ==
 *    128; phase "all" is self-scoring with queries == keys; the returned
 *    positions are 0-based in [0, end_pos); Notes: the Hadamard rotation is a
 *    mathematical no-op for the score; scales are block-32 e8m0 (qr_scale_hbm).
 *  - NeMo AutoModel optimized_kernels, sparse_attention_torch parameters:
 *    a top-k index of -1 masks an entry.
 *  - tokamax Supported Ops, lightning_indexer: the scores run over a paged
 *    KV cache. Reading: token t's cache slot s lives in page
 *    block_table[t][s / page_size], at row s % page_size of it; the pages
 *    form one pool [num_pages, page_size, D] (and [.., D/32] scales).
 *  - NeMo AutoModel optimized_kernels, dsv4_indexer_scores: the compressed
 *    (C4) indexer scores queries against pooled_kv, keys pooled over
 *    compress_ratio consecutive tokens, for a query chunk that starts at
 *    absolute position query_start.
 *  - The head-weighted ReLU sum itself is the lightning-indexer definition
 *    that the pages name (lightning_indexer in the tokamax Supported Ops
 *    table: query-key relevance scores followed by top-k) but do not print;
 *    the formula above is the standard statement of that indexer.
 *
 * Readings where the pages are silent:
 *  - valid(t,s) is inclusive: s <= positions[t] (decode) or s <= t within the
 *    row's sequence (causal prefill); the token's own key is at its position.
 *  - Compressed mode: pooled slot j covers tokens [j*r, (j+1)*r) (r =
 *    compress_ratio); query t sits at absolute position query_start + t and
 *    sees slot j iff the whole block is at or before it: (j+1)*r <=
 *    query_start + t + 1, i.e. j <= floor((query_start + t + 1) / r) - 1.
 *    Every query scores the one pooled cache; rows are [T, S] like decode.
 *  - MASK_BOUND = -0x1.FEp127, the lowest finite bf16 value (exact in fp32).
 *  - Rows with fewer valid slots than index_topk select all valid slots and
 *    pad with -1; masked slots are never selected.
 *  - Ties at the k-th score go to the lower slot index (only needed for a
 *    bit-exact comparison; the set is otherwise unordered). -0.0 == +0.0.
 *
 * Arithmetic: every input is decoded exactly to double; sums run in the
 * definition's order (d inner, then h), one row per OpenMP task.
 */
#include <math.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>

#define ORC_MODE_POSITIONS 0
#define ORC_MODE_CAUSAL 1
#define ORC_MODE_COMPRESSED 2
#define ORC_DTYPE_BF16 0
#define ORC_DTYPE_FP8 1
#define ORC_MX_BLOCK 32

static const double ORC_MASK_BOUND = -0x1.FEp127;

/* The problem statement, as the pages give it (flat, host pointers). */
typedef struct {
    int32_t mode;            /* ORC_MODE_POSITIONS, _CAUSAL or _COMPRESSED */
    int32_t dtype;           /* ORC_DTYPE_BF16 or ORC_DTYPE_FP8 (q and k) */
    int32_t T, H, D;
    int32_t num_seqs;        /* CAUSAL: packed sequences */
    int64_t S;               /* POSITIONS: slots per cache */
    int64_t k_seq_stride;    /* POSITIONS: elements between caches (0 = shared) */
    const int32_t *positions;   /* POSITIONS: [T] */
    const int32_t *cu_seqlens;  /* CAUSAL: [num_seqs + 1] */
    const void *q;              /* [T, H, D] bf16 bits or e4m3 bytes */
    const uint8_t *q_scale;     /* [T, H, D/32] e8m0 (FP8) */
    const float *w;             /* [T, H] */
    const void *k;              /* [slots, D] */
    const uint8_t *k_scale;     /* [slots, D/32] e8m0 (FP8) */
    int64_t query_start;        /* COMPRESSED: absolute position of query 0 */
    int32_t compress_ratio;     /* COMPRESSED: tokens pooled per slot (>= 1) */
    int32_t page_size;          /* POSITIONS, paged cache: slots per page */
    int32_t pages_per_seq;      /* paged: block-table entries per token */
    int32_t num_pages;          /* paged: pages in the pool k / k_scale */
    const int32_t *block_table; /* paged: [T, pages_per_seq] page ids; NULL = not paged */
} orc_problem;

/* ---- exact decoding of the storage formats -------------------------------- */

/* bf16: the upper half of an IEEE binary32 pattern. */
double orc_bf16_value(uint16_t bits)
{
    uint32_t u = (uint32_t)bits << 16;
    float f;
    memcpy(&f, &u, sizeof f);
    return (double)f;
}

/* e4m3 (OCP FP8 E4M3, "fn" variant): sign, 4 exponent bits with bias 7,
 * 3 mantissa bits; exponent field 0 is subnormal (m * 2^-9); 0x7F / 0xFF are
 * NaN (never produced by the input generator); largest finite value 448. */
double orc_e4m3_value(uint8_t code)
{
    int sign = code >> 7, e = (code >> 3) & 0xF, m = code & 7;
    double mag;
    if (e == 0xF && m == 7)
        return NAN;
    if (e == 0)
        mag = ldexp((double)m, -9);
    else
        mag = ldexp(1.0 + m / 8.0, e - 7);
    return sign ? -mag : mag;
}

/* e8m0: an unsigned biased exponent, value 2^(code - 127); 0xFF is NaN. */
double orc_e8m0_value(uint8_t code)
{
    if (code == 0xFF)
        return NAN;
    return ldexp(1.0, (int)code - 127);
}

/* Element d of a D-vector stored at row index r of a [rows, D] array. */
static double stored_value(int32_t dtype, const void *data,
                           const uint8_t *scale, int64_t r, int32_t D, int32_t d)
{
    if (dtype == ORC_DTYPE_BF16)
        return orc_bf16_value(((const uint16_t *)data)[r * D + d]);
    /* MX: e4m3 element times the e8m0 scale of its 32-wide block along D */
    return orc_e4m3_value(((const uint8_t *)data)[r * D + d]) *
           orc_e8m0_value(scale[r * (D / ORC_MX_BLOCK) + d / ORC_MX_BLOCK]);
}

/* ---- rows of the problem ---------------------------------------------------- */

/* Geometry of query row t: the slot index (row of the k array) holding slot 0
 * of its key cache, the row length (slots scored), the last valid slot
 * (valid(t,s) <=> s <= last_valid) and the row's offset in the packed score
 * output (POSITIONS: t*S; CAUSAL: sum_{j<i} L_j^2 + (t - cu[i]) * L_i).
 * Returns 0, or -1 for an out-of-range t. */
int orc_row_info(const orc_problem *p, int64_t t, int64_t *first_slot,
                 int64_t *row_len, int64_t *last_valid, int64_t *score_offset)
{
    if (t < 0 || t >= p->T)
        return -1;
    if (p->mode == ORC_MODE_POSITIONS) {
        /* a paged cache addresses its slots through the block table */
        *first_slot = p->block_table ? 0 : t * (p->k_seq_stride / p->D);
        *row_len = p->S;
        *last_valid = p->positions[t];          /* s <= positions[t] */
        *score_offset = t * p->S;
        return 0;
    }
    if (p->mode == ORC_MODE_COMPRESSED) {
        *first_slot = 0;                        /* one pooled cache */
        *row_len = p->S;
        /* (j+1)*r <= query_start + t + 1 */
        *last_valid = (p->query_start + t + 1) / p->compress_ratio - 1;
        *score_offset = t * p->S;
        return 0;
    }
    int64_t base = 0;
    for (int32_t i = 0; i < p->num_seqs; ++i) {
        int64_t a = p->cu_seqlens[i], b = p->cu_seqlens[i + 1], L = b - a;
        if (t >= a && t < b) {
            *first_slot = a;
            *row_len = L;
            *last_valid = t - a;                /* s <= t, sequence-local */
            *score_offset = base + (t - a) * L;
            return 0;
        }
        base += L * L;
    }
    return -1;
}

/* Row of the k array holding slot s of token t's cache (first: the row of
 * slot 0, from orc_row_info): the slot itself, or with a block table (paged
 * cache) row s % page_size of page block_table[t][s / page_size]. */
static int64_t key_row(const orc_problem *p, int64_t t, int64_t first, int64_t s)
{
    if (!p->block_table)
        return first + s;
    int64_t page = p->block_table[t * p->pages_per_seq + s / p->page_size];
    return page * p->page_size + s % p->page_size;
}

/* Score row of query token t into out[0 .. row_len). */
static void score_row(const orc_problem *p, int64_t t, double *out,
                      double *qrow, double *krow)
{
    int64_t first, len, last, off;
    orc_row_info(p, t, &first, &len, &last, &off);
    const int32_t H = p->H, D = p->D;
    for (int32_t h = 0; h < H; ++h)
        for (int32_t d = 0; d < D; ++d)
            qrow[h * D + d] = stored_value(p->dtype, p->q, p->q_scale,
                                           t * H + h, D, d);
    for (int64_t s = 0; s < len; ++s) {
        if (!(s <= last)) {
            out[s] = ORC_MASK_BOUND;
            continue;
        }
        for (int32_t d = 0; d < D; ++d)
            krow[d] = stored_value(p->dtype, p->k, p->k_scale, key_row(p, t, first, s),
                                   D, d);
        double I = 0.0;
        for (int32_t h = 0; h < H; ++h) {
            double x = 0.0;                     /* q[t,h,:] . k[s,:] */
            for (int32_t d = 0; d < D; ++d)
                x += qrow[h * D + d] * krow[d];
            double relu = x > 0.0 ? x : 0.0;
            I += (double)p->w[t * H + h] * relu;
        }
        out[s] = I;
    }
}

/* Scores of the listed rows. Row rows[i] is written densely (row_len values)
 * at out + out_offset[i]. Returns 0, or -1 if a row index is out of range. */
int orc_score_rows(const orc_problem *p, int64_t nrows, const int64_t *rows,
                   double *out, const int64_t *out_offset, int nthreads)
{
    for (int64_t i = 0; i < nrows; ++i)
        if (rows[i] < 0 || rows[i] >= p->T)
            return -1;
    int bad = 0;
#pragma omp parallel num_threads(nthreads > 0 ? nthreads : 1)
    {
        double *qrow = malloc(sizeof(double) * (size_t)p->H * p->D);
        double *krow = malloc(sizeof(double) * (size_t)p->D);
        if (!qrow || !krow) {
#pragma omp atomic write
            bad = 1;
        } else {
#pragma omp for schedule(dynamic, 1)
            for (int64_t i = 0; i < nrows; ++i)
                score_row(p, rows[i], out + out_offset[i], qrow, krow);
        }
        free(qrow);
        free(krow);
    }
    return bad ? -2 : 0;
}

/* ---- top-k ----------------------------------------------------------------- */

typedef struct {
    double v;
    int64_t s;
} orc_cand;

/* Larger score first; equal scores (including -0.0 vs +0.0): lower slot first. */
static int cand_order(const void *a, const void *b)
{
    const orc_cand *x = a, *y = b;
    if (x->v > y->v) return -1;
    if (x->v < y->v) return 1;
    return (x->s > y->s) - (x->s < y->s);
}

/* Top-k of one score row: the min(k, nvalid) valid slots with the largest
 * scores (a full sort of the valid slots), then -1 padding up to k. Valid
 * slots are s <= last_valid (by position, never by value). Writes k int32. */
static int topk_row(const double *row, int64_t row_len, int64_t last_valid,
                    int32_t k, int32_t *out)
{
    int64_t nvalid = last_valid + 1;
    if (nvalid > row_len) nvalid = row_len;
    if (nvalid < 0) nvalid = 0;
    orc_cand *c = malloc(sizeof(orc_cand) * (size_t)(nvalid > 0 ? nvalid : 1));
    if (!c)
        return -2;
    for (int64_t s = 0; s < nvalid; ++s) {
        c[s].v = row[s];
        c[s].s = s;
    }
    qsort(c, (size_t)nvalid, sizeof(orc_cand), cand_order);
    for (int32_t j = 0; j < k; ++j)
        out[j] = j < nvalid ? (int32_t)c[j].s : -1;
    free(c);
    return 0;
}

/* Top-k of the listed rows of the problem, given their score rows (dense, at
 * scores + score_offset[i], row_len values each). Writes k values per row at
 * out + i*k. The scores may come from this oracle or from any other source;
 * validity is always the problem's mask rule. */
int orc_topk_rows(const orc_problem *p, int64_t nrows, const int64_t *rows,
                  const double *scores, const int64_t *score_offset, int32_t k,
                  int32_t *out, int nthreads)
{
    for (int64_t i = 0; i < nrows; ++i)
        if (rows[i] < 0 || rows[i] >= p->T)
            return -1;
    int bad = 0;
#pragma omp parallel for schedule(dynamic, 1) num_threads(nthreads > 0 ? nthreads : 1)
    for (int64_t i = 0; i < nrows; ++i) {
        int64_t first, len, last, off;
        orc_row_info(p, rows[i], &first, &len, &last, &off);
        if (topk_row(scores + score_offset[i], len, last, k, out + i * k)) {
#pragma omp atomic write
            bad = 1;
        }
    }
    return bad ? -2 : 0;
}

double orc_mask_bound(void) { return ORC_MASK_BOUND; }
