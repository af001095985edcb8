// score_kernel.cuh -- lightning-indexer score kernel for sm_100a.
//
// Computes I[t,s] = sum_h w[t,h] * ReLU(q[t,h,:] . k[s,:]) for valid slots
// and the finite mask bound elsewhere (DeepSeek-V3.2 Sparse Indexer Kernel
// API Reference: scores over every cached slot, clamped to a finite bound).
//
// Shape of the contraction: q . k^T is the dense [T*H, D] x [D, S] product.
// The MMA puts KEY SLOTS on M (128 per tile) and query (token, head) pairs on
// N, so accumulator lane i of TMEM holds slot i and the head reduction of
// the epilogue is thread-local: no shuffles, and a warp's 32 lanes write 32
// consecutive scores of a row.
//
//   warp 0      : TMA producer (one thread)
//   warp 1      : TMEM allocator + MMA issuer (one thread issues; for fp8 the
//                 whole warp first lays the scale factors out for tcgen05.cp)
//   warps 2..   : epilogue (TMEM -> ReLU, w-weighted head sum, mask, store)
//
// Schedule: a query block is up to tq_sub*NSUB consecutive tokens that read
// one key cache. An "active item" is (query block, key tile) with the tile
// holding at least one valid slot of the block; a "fill item" is a tile of the
// block's score rows where every slot is masked. Both lists are split into
// contiguous ranges, one per CTA (no atomics), by cost: a query block's own
// cost (its query load and pipeline refill; the fixed time of its fill
// stores) counts beside its tiles.
// Per active item the MMA issues one accumulator per sub-block; accumulators
// rotate through NACC TMEM buffers so the epilogue of one overlaps the MMA of
// the next. Fill items are never loaded: the epilogue writes the mask bound,
// before it turns to its active items.
//
// fp8 (MX) variant: e4m3 q and k with one e8m0 scale per 32 elements along D
// (Sparse Attention Indexer MX BF16Score Kernel API Reference: block-32 e8m0
// scales). The scales are applied inside the MMA
// (tcgen05.mma kind::mxf8f6f4.block_scale): TMA brings the scale words next to
// the data, the MMA warp reorders them into the 128-row scale-factor atom and
// copies them into TMEM with tcgen05.cp; no dequantised copy is ever written.
#pragma once

#include <cstdint>

#include "sm100_ptx.cuh"
#include "row_rule.cuh"

namespace dsa {

constexpr int kBlockM = 128;          // key slots per tile (MMA M)
constexpr int kHeadDim = 128;         // D
constexpr float kMaskBound = -0x1.FEp127f;   // lowest finite bf16

// COMPRESSED is POSITIONS over one shared cache with the last valid slot of
// each row given by the compressed rule instead of a positions array.
enum : int { kModePositions = 0, kModeCausal = 1, kModeCompressed = 2 };

struct ScoreParams {
  int mode;
  int T, H;
  int64_t S;                 // POSITIONS: slots per cache
  int shared_cache;          // POSITIONS: every token reads cache 0
  const int *block_table;    // POSITIONS, paged: [T, pages_per_seq] page ids (else NULL)
  int pages_per_seq;         // paged: block-table entries per token
  int num_pages;             // paged: pages in the pool (an id past it reads as zeros)
  int page_shift;            // paged: log2(slots per page)
  int num_seqs;              // CAUSAL
  const int *cu_seqlens;     // CAUSAL
  const int *positions;      // POSITIONS
  int compressed;            // POSITIONS geometry, rows end by the compressed rule
  CompressedRule comp;
  int blk_w;                 // schedule weight of a query block (a key tile weighs 8)
  const float *w;            // [T, H]
  float *scores;
  int tq_sub;                // tokens per MMA sub-block (tq_sub*NSUB divides 128)
  int n_cols;                // MMA N per sub-block: round_up(tq_sub*H, 16)
  unsigned int *err;
  unsigned int *err_info;
  const unsigned int *cu_bad;   // CAUSAL: set by the cu_seqlens check -> no work
  uint64_t wait_limit_ns;       // any single wait
  uint64_t drain_limit_ns;      // the drains on the way out (not the wait limit)
  int selftest_stall;           // the MMA warp first waits on a barrier nothing completes
  int k_once;                   // every key tile is read by one query block only
};

__host__ __device__ constexpr int sf_atoms(int n_cols) { return (n_cols + 127) / 128; }

// fp8 scale windows: TMA loads scale words from a start rounded down to a
// multiple of 4 words (a tiled copy of 32-bit elements must start 16-byte
// aligned along its innermost dimension), so every window holds 4 extra words.
// Every TMA destination in shared memory starts on a 128-byte boundary, so
// the windows' sizes are rounded up to 128 bytes.
constexpr int kSfPad = 4;
__host__ __device__ constexpr uint32_t round128(uint32_t x) { return (x + 127u) & ~127u; }
// bytes one scale-window copy delivers (the mbarrier's expected transaction
// count) and the shared-memory room it takes
constexpr uint32_t kSfBoxBytesK = (kBlockM + kSfPad) * 4;
// A paged tile's scale words come one box per page; a TMA destination must be
// 128-byte aligned, so 16-slot pages (64 bytes of words a box) each get a
// 128-byte slot: 8 slots, 1024 bytes, which also holds the unpaged window.
constexpr uint32_t kSfRawBytesK = 1024;
static_assert(kSfRawBytesK >= round128(kSfBoxBytesK), "scale window room");
__host__ __device__ constexpr uint32_t sf_box_bytes_q(int n_cols) {
  return static_cast<uint32_t>((n_cols + kSfPad) * 4);
}
__host__ __device__ constexpr uint32_t sf_raw_bytes_q(int n_cols) {
  return round128(sf_box_bytes_q(n_cols));
}

// Shared-memory plan, identical on host and device.
constexpr int kPosCap = 2048;          // positions staged in shared memory
constexpr int kWRowsPerWarp = 4;        // H=64 epilogue: w rows a warp keeps

// A stage holds `tiles` key tiles (one pipeline item); each tile slot has
// its own data and (fp8) scale window.
struct ScoreSmem {
  uint32_t k_stage_bytes, k_sf_bytes, q_sub_bytes, q_sf_bytes;
  uint32_t off_k, off_ksf, off_q, off_qsf, off_w, off_pos, off_bar, off_misc, total;
  __host__ __device__ ScoreSmem(int stages, int qbuf, int nsub, int n_cols, bool fp8,
                                int epi_warps, int tiles) {
    // bf16: two 128-byte-wide halves along D; fp8: one 128-byte row.
    // (k_stage_bytes / k_sf_bytes are per tile slot.)
    k_stage_bytes = fp8 ? kBlockM * 128 : kBlockM * 256;
    q_sub_bytes = fp8 ? n_cols * 128 : n_cols * 256;
    // fp8 scale words (4 bytes a row) as loaded -- a window of rows + 4 words
    // that starts at a multiple of 4 words, the TMA alignment rule for 32-bit
    // elements -- followed by the reordered atoms (512 B each).
    k_sf_bytes = fp8 ? kSfRawBytesK + 512 : 0;
    q_sf_bytes = fp8 ? static_cast<uint32_t>(sf_raw_bytes_q(n_cols) + sf_atoms(n_cols) * 512) : 0;
    off_k = 0;
    off_q = off_k + stages * tiles * k_stage_bytes;
    off_ksf = off_q + qbuf * nsub * q_sub_bytes;
    off_qsf = off_ksf + stages * tiles * k_sf_bytes;
    off_w = off_qsf + qbuf * nsub * q_sf_bytes;
    off_w = (off_w + 15) & ~15u;
    off_pos = off_w + epi_warps * kWRowsPerWarp * 64 * 4;
    off_bar = off_pos + kPosCap * 4;
    off_misc = off_bar + 64 * 8;            // up to 64 mbarriers
    total = off_misc + 256 + 1024;          // misc words + alignment slack
  }
};

// TMEM columns: accumulator slots (acc_per_slot accumulators of n_cols each),
// then (fp8) A scales per stage tile slot, then B scales per query-buffer
// sub-block.
__host__ __device__ constexpr int tmem_cols_needed(int nacc, int acc_per_slot, int n_cols,
                                                  int stages, int tiles, int qbuf, int nsub,
                                                  bool fp8) {
  return nacc * acc_per_slot * n_cols +
         (fp8 ? stages * tiles * 4 + qbuf * nsub * 4 * sf_atoms(n_cols) : 0);
}

// ---- the static schedule --------------------------------------------------------

// One query block and the key tiles of its score rows.
struct QBlk {
  int seq, b;          // CAUSAL: sequence and block in it; POSITIONS: seq 0, block b
  int t0, ntok;        // tokens [t0, t0 + ntok)
  int z, y0;           // key cache (3rd TMA coordinate), first key row (2nd)
  int64_t row_len;     // slots per score row
  int64_t out0;        // float offset of token t0's score row
  int64_t seqoff;      // CAUSAL: float offset of the sequence's score block
  int lv0;             // CAUSAL: last valid slot of token t0
  int act, ntr;        // tiles holding a valid slot; tiles in the row
};

__device__ __forceinline__ int last_valid_pos(const ScoreParams &p, int t) {
  // positions: global, or the CTA's shared copy
  const int64_t pos = p.compressed ? compressed_last_slot(p.comp, t) : p.positions[t];
  const int64_t lv = pos < 0 ? -1 : (pos >= p.S ? p.S - 1 : pos);
  return static_cast<int>(lv);
}

// Last valid slot of token t0 + i of block q.
__device__ __forceinline__ int qb_last_valid(const ScoreParams &p, const QBlk &q, int i) {
  return p.mode == kModeCausal ? q.lv0 + i : last_valid_pos(p, q.t0 + i);
}

__device__ __forceinline__ int pos_num_blocks(const ScoreParams &p, int tqt) {
  return p.shared_cache ? (p.T + tqt - 1) / tqt : p.T;
}

__device__ __forceinline__ void make_qb_positions(const ScoreParams &p, int tqt, int b, QBlk &q) {
  q.seq = 0;
  q.b = b;
  q.t0 = b * tqt;
  q.ntok = min(tqt, p.T - q.t0);
  q.z = p.shared_cache ? 0 : q.t0;
  q.y0 = 0;
  q.row_len = p.S;
  q.out0 = static_cast<int64_t>(q.t0) * p.S;
  q.seqoff = 0;
  q.lv0 = 0;
  int mx = -1;
  if (p.compressed) {
    // the compressed rule never decreases along the tokens
    if (q.ntok > 0) mx = last_valid_pos(p, q.t0 + q.ntok - 1);
  } else {
    int m1 = -1, m2 = -1, m3 = -1;      // four independent chains
    int i = 0;
    for (; i + 4 <= q.ntok; i += 4) {
      mx = max(mx, last_valid_pos(p, q.t0 + i));
      m1 = max(m1, last_valid_pos(p, q.t0 + i + 1));
      m2 = max(m2, last_valid_pos(p, q.t0 + i + 2));
      m3 = max(m3, last_valid_pos(p, q.t0 + i + 3));
    }
    for (; i < q.ntok; ++i) mx = max(mx, last_valid_pos(p, q.t0 + i));
    mx = max(max(mx, m1), max(m2, m3));
  }
  q.ntr = static_cast<int>((p.S + kBlockM - 1) / kBlockM);
  q.act = mx < 0 ? 0 : mx / kBlockM + 1;
}

__device__ __forceinline__ void make_qb_causal(const ScoreParams &p, int tqt, int seq, int b,
                               int64_t seqoff, QBlk &q) {
  const int a = __ldg(p.cu_seqlens + seq);
  const int L = __ldg(p.cu_seqlens + seq + 1) - a;
  const int tl0 = b * tqt;
  q.seq = seq;
  q.b = b;
  q.t0 = a + tl0;
  q.ntok = min(tqt, L - tl0);
  q.z = 0;
  q.y0 = a;
  q.row_len = L;
  q.seqoff = seqoff;
  q.out0 = seqoff + static_cast<int64_t>(tl0) * L;
  q.lv0 = tl0;
  q.ntr = (L + kBlockM - 1) / kBlockM;
  q.act = (tl0 + q.ntok - 1) / kBlockM + 1;
}

// CAUSAL, tqt dividing 128: block b of a sequence has floor(b/r) + 1 active
// tiles (r = 128/tqt), so the active tiles of blocks [0, B) number
// B + r*m*(m-1)/2 + m*(B - m*r) with m = B / r.
__device__ __forceinline__ int64_t causal_active_before(int64_t B, int r) {
  const int64_t m = B / r, rem = B - m * r;
  return B + r * m * (m - 1) / 2 + m * rem;
}

// Move q to the next query block (skipping empty sequences). False at the end.
__device__ __forceinline__ bool next_qb(const ScoreParams &p, int tqt, QBlk &q) {
  if (p.mode == kModePositions) {
    if (q.b + 1 >= pos_num_blocks(p, tqt)) return false;
    make_qb_positions(p, tqt, q.b + 1, q);
    return true;
  }
  const int L = static_cast<int>(q.row_len);
  if ((q.b + 1) * tqt < L) {
    make_qb_causal(p, tqt, q.seq, q.b + 1, q.seqoff, q);
    return true;
  }
  int64_t off = q.seqoff + static_cast<int64_t>(L) * L;
  for (int s = q.seq + 1; s < p.num_seqs; ++s) {
    const int Ls = __ldg(p.cu_seqlens + s + 1) - __ldg(p.cu_seqlens + s);
    if (Ls > 0) {
      make_qb_causal(p, tqt, s, 0, off, q);
      return true;
    }
  }
  return false;
}

// Where a CTA starts: its shares of the active and fill lists, and the
// (block, tile) of the first item of each.
struct CtaRange {
  int64_t a_count, f_count;
  int a_seq, a_b, a_j;
  int f_seq, f_b, f_j;
  int64_t a_seqoff, f_seqoff;
};

// Both lists are split between CTAs by cost, not by count. An active tile
// weighs kTileW and every query block with an active tile adds blk_w (its
// query load and the pipeline refill at its start); a fill tile weighs
// kFillTileW and every block with a fill tile adds kFillBlkW (the epilogue's
// walk to the block and the fixed time of its row stores). With a list's
// weights laid end to end, tile j of a block whose weights start at P sits at
// P + (block weight) + (tile weight)*j, and CTA c of G takes the tiles
// sitting in [Wt*c/G, Wt*(c+1)/G) (Wt: the list's total), so a CTA whose
// share crosses many short blocks takes fewer tiles.
constexpr int kTileW = 8;
constexpr int kFillTileW = 1;
constexpr int kFillBlkW = 10;

// Of the n tiles of a block whose weights start at P, the number sitting
// before weight w.
__device__ __forceinline__ int tiles_before(int64_t w, int64_t P, int64_t blk_w, int tile_w,
                                            int n) {
  const int64_t num = w - P - blk_w;
  if (num <= 0) return 0;
  const int64_t k = (num + tile_w - 1) / tile_w;
  return k < n ? static_cast<int>(k) : n;
}

// Inclusive warp scan.
__device__ __forceinline__ int64_t warp_incl_scan(int64_t v, int lane) {
#pragma unroll
  for (int off = 1; off < 32; off <<= 1) {
    const int64_t n = __shfl_up_sync(0xffffffffu, v, off);
    if (lane >= off) v += n;
  }
  return v;
}

// POSITIONS: this CTA's share of both lists, by one warp in one pass over
// the query blocks. Lane l owns a contiguous run of blocks and totals both
// lists' tiles and blocks over it; one warp scan places the runs and gives
// the totals; lanes 0..3 form the four bounds (w0, w1 of the active list,
// v0, v1 of the fill list) so that their divisions overlap; the lane whose
// run holds the first tile at or after a bound walks its run again to find
// it, and broadcasts it. Full warp.
__device__ __forceinline__ void cta_range_positions(const ScoreParams &p, int tqt, CtaRange &R) {
  const int lane = threadIdx.x & 31;
  const int nqb = pos_num_blocks(p, tqt);
  const int64_t bw = p.blk_w;
  const int per = (nqb + 31) / 32;
  const int lo = min(nqb, lane * per), hi = min(nqb, lo + per);
  int64_t sa = 0, sc = 0, sf = 0, sfb = 0;
  for (int b = lo; b < hi; ++b) {
    QBlk q;
    make_qb_positions(p, tqt, b, q);
    sa += q.act;
    sc += q.act > 0;
    sf += q.ntr - q.act;
    sfb += q.ntr > q.act;
  }
  const int64_t ia = warp_incl_scan(sa, lane), ic = warp_incl_scan(sc, lane);
  const int64_t jf = warp_incl_scan(sf, lane), jfb = warp_incl_scan(sfb, lane);
  const int64_t A = __shfl_sync(0xffffffffu, ia, 31), NB = __shfl_sync(0xffffffffu, ic, 31);
  const int64_t F = __shfl_sync(0xffffffffu, jf, 31), NFB = __shfl_sync(0xffffffffu, jfb, 31);
  const int64_t wa = kTileW * A + bw * NB;
  const int64_t wf = kFillTileW * F + kFillBlkW * NFB;
  int64_t bound = 0;
  if (lane < 4) bound = (lane < 2 ? wa : wf) * (blockIdx.x + (lane & 1)) / gridDim.x;
  const int64_t w0 = __shfl_sync(0xffffffffu, bound, 0);
  const int64_t w1 = __shfl_sync(0xffffffffu, bound, 1);
  const int64_t v0 = __shfl_sync(0xffffffffu, bound, 2);
  const int64_t v1 = __shfl_sync(0xffffffffu, bound, 3);
  // where this lane's weights start and where its last tile sits
  const int64_t Pa = kTileW * (ia - sa) + bw * (ic - sc);
  const int64_t Pf = kFillTileW * (jf - sf) + kFillBlkW * (jfb - sfb);
  const int64_t La = kTileW * ia + bw * ic - kTileW;
  const int64_t Lf = kFillTileW * jf + kFillBlkW * jfb - kFillTileW;
  const int l_w0 = __ffs(__ballot_sync(0xffffffffu, w0 < wa && sa > 0 && La >= w0)) - 1;
  const int l_w1 = __ffs(__ballot_sync(0xffffffffu, w1 < wa && sa > 0 && La >= w1)) - 1;
  const int l_v0 = __ffs(__ballot_sync(0xffffffffu, v0 < wf && sf > 0 && Lf >= v0)) - 1;
  const int l_v1 = __ffs(__ballot_sync(0xffffffffu, v1 < wf && sf > 0 && Lf >= v1)) - 1;
  // The owners walk their runs again. g*, h*: list index of the tile found,
  // or the list's length (no tile at or after the bound).
  int a_b = nqb, a_j = 0, f_b = nqb, f_j = 0;
  int64_t g0 = A, g1 = A, h0 = F, h1 = F;
  bool n_w0 = lane == l_w0, n_w1 = lane == l_w1, n_v0 = lane == l_v0, n_v1 = lane == l_v1;
  int64_t P = Pa, Q = Pf, ga = ia - sa, gf = jf - sf;
  for (int b = lo; b < hi && (n_w0 || n_w1 || n_v0 || n_v1); ++b) {
    QBlk q;
    make_qb_positions(p, tqt, b, q);
    const int act = q.act, fil = q.ntr - q.act;
    if (act > 0) {
      const int64_t last = P + bw + static_cast<int64_t>(kTileW) * (act - 1);
      if (n_w0 && last >= w0) {
        a_b = b;
        a_j = tiles_before(w0, P, bw, kTileW, act);
        g0 = ga + a_j;
        n_w0 = false;
      }
      if (n_w1 && last >= w1) {
        g1 = ga + tiles_before(w1, P, bw, kTileW, act);
        n_w1 = false;
      }
      P += bw + static_cast<int64_t>(kTileW) * act;
      ga += act;
    }
    if (fil > 0) {
      const int64_t last = Q + kFillBlkW + static_cast<int64_t>(kFillTileW) * (fil - 1);
      if (n_v0 && last >= v0) {
        const int j = tiles_before(v0, Q, kFillBlkW, kFillTileW, fil);
        f_b = b;
        f_j = act + j;          // fill tiles follow the row's active ones
        h0 = gf + j;
        n_v0 = false;
      }
      if (n_v1 && last >= v1) {
        h1 = gf + tiles_before(v1, Q, kFillBlkW, kFillTileW, fil);
        n_v1 = false;
      }
      Q += kFillBlkW + static_cast<int64_t>(kFillTileW) * fil;
      gf += fil;
    }
  }
  R.a_seq = R.f_seq = 0;
  R.a_seqoff = R.f_seqoff = 0;
  R.a_b = nqb;
  R.a_j = 0;
  R.f_b = nqb;
  R.f_j = 0;
  if (l_w0 >= 0) {
    R.a_b = __shfl_sync(0xffffffffu, a_b, l_w0);
    R.a_j = __shfl_sync(0xffffffffu, a_j, l_w0);
    g0 = __shfl_sync(0xffffffffu, g0, l_w0);
  }
  if (l_w1 >= 0) g1 = __shfl_sync(0xffffffffu, g1, l_w1);
  if (l_v0 >= 0) {
    R.f_b = __shfl_sync(0xffffffffu, f_b, l_v0);
    R.f_j = __shfl_sync(0xffffffffu, f_j, l_v0);
    h0 = __shfl_sync(0xffffffffu, h0, l_v0);
  }
  if (l_v1 >= 0) h1 = __shfl_sync(0xffffffffu, h1, l_v1);
  R.a_count = g1 - g0;
  R.f_count = h1 - h0;
}

// CAUSAL: active or fill items before block B of a sequence.
__device__ __forceinline__ int64_t causal_before(int64_t B, int r, int ntr, bool fill) {
  const int64_t a = causal_active_before(B, r);
  return fill ? B * ntr - a : a;
}

// CAUSAL: weight of blocks [0, B) of a sequence in the active list (every
// block holds an active tile) or in the fill list (block b holds ntr - b/r - 1
// fill tiles: those below b < r*(ntr-1) hold one).
__device__ __forceinline__ int64_t causal_weight_before(int64_t B, int r, int ntr, int64_t bw,
                                                        bool fill) {
  const int64_t act = causal_active_before(B, r);
  if (!fill) return kTileW * act + bw * B;
  const int64_t with_fill = static_cast<int64_t>(r) * (ntr - 1);
  return kFillTileW * (B * ntr - act) + kFillBlkW * (B < with_fill ? B : with_fill);
}

// CAUSAL: the first tile of the active or fill list sitting at or after
// weight w -- its sequence, block, tile in the score row and the sequence's
// score offset -- and its index in the list (the list's length when there is
// none). One thread.
__device__ __forceinline__ int64_t locate_causal_weight(const ScoreParams &p, int tqt, int64_t w,
                                                        bool fill, int &seq_out, int &b_out,
                                                        int &j_out, int64_t &seqoff_out) {
  const int r = kBlockM / tqt;
  const int64_t bw = fill ? kFillBlkW : p.blk_w;
  const int tw = fill ? kFillTileW : kTileW;
  int64_t off = 0, gbase = 0;
  for (int s = 0; s < p.num_seqs; ++s) {
    const int L = __ldg(p.cu_seqlens + s + 1) - __ldg(p.cu_seqlens + s);
    if (L <= 0) continue;
    const int nqb = (L + tqt - 1) / tqt, ntr = (L + kBlockM - 1) / kBlockM;
    const int64_t tot = causal_weight_before(nqb, r, ntr, bw, fill);
    if (w <= tot - tw) {              // the sequence's last tile sits at tot - tw
      int lo = 0, hi = nqb - 1;       // first block whose last tile sits at or after w
      while (lo < hi) {
        const int mid = (lo + hi) / 2;
        if (causal_weight_before(mid + 1, r, ntr, bw, fill) - tw >= w) hi = mid; else lo = mid + 1;
      }
      const int act = lo / r + 1, n = fill ? ntr - act : act;
      const int j = tiles_before(w, causal_weight_before(lo, r, ntr, bw, fill), bw, tw, n);
      seq_out = s;
      b_out = lo;
      j_out = fill ? act + j : j;
      seqoff_out = off;
      return gbase + causal_before(lo, r, ntr, fill) + j;
    }
    w -= tot;
    gbase += causal_before(nqb, r, ntr, fill);
    off += static_cast<int64_t>(L) * L;
  }
  seq_out = p.num_seqs;
  b_out = 0;
  j_out = 0;
  seqoff_out = off;
  return gbase;
}

// CAUSAL: active tiles A, fill tiles F, query blocks NB and blocks holding a
// fill tile NFB of the batch.
__device__ __forceinline__ void count_causal(const ScoreParams &p, int tqt, int64_t &A, int64_t &F,
                                             int64_t &NB, int64_t &NFB) {
  const int r = kBlockM / tqt;
  A = 0;
  F = 0;
  NB = 0;
  NFB = 0;
  for (int s = 0; s < p.num_seqs; ++s) {
    const int L = __ldg(p.cu_seqlens + s + 1) - __ldg(p.cu_seqlens + s);
    if (L <= 0) continue;
    const int nqb = (L + tqt - 1) / tqt, ntr = (L + kBlockM - 1) / kBlockM;
    A += causal_before(nqb, r, ntr, false);
    F += causal_before(nqb, r, ntr, true);
    NB += nqb;
    NFB += nqb < r * (ntr - 1) ? nqb : r * (ntr - 1);
  }
}

// This CTA's share of both lists (executed by a full warp; every lane gets
// the same result).
__device__ __forceinline__ void cta_range(const ScoreParams &p, int tqt, CtaRange &R) {
  if (p.mode == kModePositions) {
    cta_range_positions(p, tqt, R);
    return;
  }
  const int64_t G = gridDim.x, c = blockIdx.x;
  int64_t A = 0, F = 0, NB = 0, NFB = 0;
  count_causal(p, tqt, A, F, NB, NFB);
  const int64_t wa = kTileW * A + p.blk_w * NB;
  const int64_t wf = kFillTileW * F + kFillBlkW * NFB;
  const int64_t w0 = wa * c / G, w1 = wa * (c + 1) / G;
  const int64_t v0 = wf * c / G, v1 = wf * (c + 1) / G;
  R.a_seq = R.f_seq = 0;
  R.a_b = R.f_b = 0;
  R.a_j = R.f_j = 0;
  R.a_seqoff = R.f_seqoff = 0;
  R.a_count = 0;
  R.f_count = 0;
  int s1, b1, j1;
  int64_t off1;
  if (w0 < wa) {
    const int64_t g0 =
        locate_causal_weight(p, tqt, w0, false, R.a_seq, R.a_b, R.a_j, R.a_seqoff);
    R.a_count = locate_causal_weight(p, tqt, w1, false, s1, b1, j1, off1) - g0;
  }
  if (v0 < wf) {
    const int64_t h0 =
        locate_causal_weight(p, tqt, v0, true, R.f_seq, R.f_b, R.f_j, R.f_seqoff);
    R.f_count = locate_causal_weight(p, tqt, v1, true, s1, b1, j1, off1) - h0;
  }
}

__device__ __forceinline__ void make_qb(const ScoreParams &p, int tqt, int seq, int b,
                                        int64_t seqoff, QBlk &q) {
  if (p.mode == kModePositions) make_qb_positions(p, tqt, b, q);
  else make_qb_causal(p, tqt, seq, b, seqoff, q);
}

// A walk over this CTA's share of the active list, one pipeline item at a
// time: up to kG consecutive key tiles of one query block. Every role walks
// the same items in the same order.
struct ItemCursor {
  QBlk q;
  int j;          // first tile of the current item
  int64_t left;   // tiles of the share not yet taken
};

__device__ __forceinline__ void cursor_start(const ScoreParams &p, int tqt, const CtaRange &R,
                                             ItemCursor &c) {
  make_qb(p, tqt, R.a_seq, R.a_b, R.a_seqoff, c.q);
  c.j = R.a_j;
  c.left = R.a_count;
}

// Tiles of the current item.
template <int kG>
__device__ __forceinline__ int cursor_tiles(const ItemCursor &c) {
  const int in_block = c.q.act - c.j < kG ? c.q.act - c.j : kG;
  return c.left < in_block ? static_cast<int>(c.left) : in_block;
}

// Step past the g tiles of the current item. True when the walk left the
// query block (or the share is used up).
__device__ __forceinline__ bool cursor_next_block(const ScoreParams &p, int tqt, ItemCursor &c) {
  do {
    if (!next_qb(p, tqt, c.q)) {
      c.left = 0;
      return true;
    }
  } while (c.q.act == 0);
  c.j = 0;
  return true;
}

__device__ __forceinline__ bool cursor_step(const ScoreParams &p, int tqt, ItemCursor &c, int g) {
  c.j += g;
  c.left -= g;
  if (c.left <= 0) return true;
  if (c.j < c.q.act) return false;
  return cursor_next_block(p, tqt, c);
}

// ---- epilogue helpers ---------------------------------------------------------------

// One token with H == 64 (the tuned head count): heads 0..63 of this slot
// from TMEM in two 32-column halves, the w row from shared memory, eight
// independent partial sums (heads h = 32j + 4i + r into sum 4j + r, in four
// packed pairs), so that the packed fp32 FMAs form four short dependency
// chains instead of two long ones. The w loads of each half are issued
// before the TMEM load they pair with, so their latency is hidden behind it.
__device__ __forceinline__ float head_sum_h64(uint32_t taddr, const float *wrow) {
  const float4 *w4 = reinterpret_cast<const float4 *>(wrow);
  float2 acc[4] = {make_float2(0.f, 0.f), make_float2(0.f, 0.f), make_float2(0.f, 0.f),
                   make_float2(0.f, 0.f)};
  float4 wv[8];
#pragma unroll
  for (int i = 0; i < 8; ++i) wv[i] = w4[i];
#pragma unroll
  for (int half = 0; half < 2; ++half) {
    float r[32];
    tmem_ld32_wait(taddr + 32 * half, r);
    float4 wn[8];
    if (half == 0) {
#pragma unroll
      for (int i = 0; i < 8; ++i) wn[i] = w4[8 + i];
    }
    float2 &p01 = acc[2 * half], &p23 = acc[2 * half + 1];
#pragma unroll
    for (int i = 0; i < 8; ++i) {
      p01 = ffma2(make_float2(wv[i].x, wv[i].y),
                  make_float2(fmaxf(r[4 * i + 0], 0.f), fmaxf(r[4 * i + 1], 0.f)), p01);
      p23 = ffma2(make_float2(wv[i].z, wv[i].w),
                  make_float2(fmaxf(r[4 * i + 2], 0.f), fmaxf(r[4 * i + 3], 0.f)), p23);
    }
    if (half == 0) {
#pragma unroll
      for (int i = 0; i < 8; ++i) wv[i] = wn[i];
    }
  }
  return ((acc[0].x + acc[0].y) + (acc[1].x + acc[1].y)) +
         ((acc[2].x + acc[2].y) + (acc[3].x + acc[3].y));
}

// The same head sums for the tokens [i_lo, i_hi) of one accumulator (64
// columns a token; w rows at wsh, 64 floats each), with the next 32-column
// TMEM load in flight while the current one is reduced: one load is
// outstanding at a time, so each wait covers exactly the load it needs. The
// sums are formed in the same order as head_sum_h64. store(i, sum).
template <typename Store>
__device__ __forceinline__ void head_sums_h64_pipelined(uint32_t tbase, int i_lo, int i_hi,
                                                        const float *wsh, Store store) {
  if (i_lo >= i_hi) return;
  float ra[32], rb[32];
  tmem_ld32_async(tbase + i_lo * 64, ra);
  tmem_wait_ld32(ra);
  for (int i = i_lo; i < i_hi; ++i) {
    const float4 *w4 = reinterpret_cast<const float4 *>(wsh + (i - i_lo) * 64);
    tmem_ld32_async(tbase + i * 64 + 32, rb);            // second half, in flight
    float2 a0 = make_float2(0.f, 0.f), a1 = make_float2(0.f, 0.f);
#pragma unroll
    for (int k = 0; k < 8; ++k) {
      const float4 w = w4[k];
      a0 = ffma2(make_float2(w.x, w.y),
                 make_float2(fmaxf(ra[4 * k + 0], 0.f), fmaxf(ra[4 * k + 1], 0.f)), a0);
      a1 = ffma2(make_float2(w.z, w.w),
                 make_float2(fmaxf(ra[4 * k + 2], 0.f), fmaxf(ra[4 * k + 3], 0.f)), a1);
    }
    tmem_wait_ld32(rb);
    if (i + 1 < i_hi) tmem_ld32_async(tbase + (i + 1) * 64, ra);   // next token, in flight
    float2 a2 = make_float2(0.f, 0.f), a3 = make_float2(0.f, 0.f);
#pragma unroll
    for (int k = 0; k < 8; ++k) {
      const float4 w = w4[8 + k];
      a2 = ffma2(make_float2(w.x, w.y),
                 make_float2(fmaxf(rb[4 * k + 0], 0.f), fmaxf(rb[4 * k + 1], 0.f)), a2);
      a3 = ffma2(make_float2(w.z, w.w),
                 make_float2(fmaxf(rb[4 * k + 2], 0.f), fmaxf(rb[4 * k + 3], 0.f)), a3);
    }
    store(i, ((a0.x + a0.y) + (a1.x + a1.y)) + ((a2.x + a2.y) + (a3.x + a3.y)));
    if (i + 1 < i_hi) tmem_wait_ld32(ra);
  }
}

__device__ __forceinline__ int64_t min64(int64_t a, int64_t b) { return a < b ? a : b; }

// Write the mask bound to row[lo, hi), threads t = 0..nthr-1 of the caller,
// 16-byte stores on the aligned body.
__device__ __forceinline__ void fill_mask(float *row, int64_t lo, int64_t hi, int t, int nthr) {
  if (lo >= hi) return;
  float *base = row + lo;
  const int64_t n = hi - lo;
  const int64_t head =
      min64(n, ((16 - (reinterpret_cast<uintptr_t>(base) & 15)) & 15) / 4);
  if (t < head) base[t] = kMaskBound;
  const int64_t nvec = (n - head) / 4;
  float4 *v = reinterpret_cast<float4 *>(base + head);
  const float4 mb = make_float4(kMaskBound, kMaskBound, kMaskBound, kMaskBound);
  for (int64_t i = t; i < nvec; i += nthr) v[i] = mb;
  const int64_t tail0 = head + 4 * nvec;
  if (tail0 + t < n) base[tail0 + t] = kMaskBound;
}

// Role bookkeeping of a ring of mbarrier pairs.
struct Ring {
  uint32_t idx = 0, phase = 0;
  __device__ __forceinline__ void next(uint32_t n) {
    if (++idx == n) { idx = 0; phase ^= 1u; }
  }
};

// fp8: reorder 128 rows of 4 scale bytes (row-major, as loaded) into the
// scale-factor atom tcgen05.cp copies: row m = m0 + 32*m1 at byte
// 16*m0 + 4*m1 (+ K block). Rows >= nrows read as 0. Full warp.
// The same from the scale words of a paged tile with 16-slot pages: row m at
// word 32 * (m / 16) + m % 16 (one 128-byte slot per page box). Full warp.
__device__ __forceinline__ void sf_reorder_atom_pages16(const uint32_t *slots, uint32_t *atom) {
  const int l = threadIdx.x & 31;
  auto word = [&](int m) { return slots[((m >> 4) << 5) + (m & 15)]; };
  uint4 v;
  v.x = word(l);
  v.y = word(l + 32);
  v.z = word(l + 64);
  v.w = word(l + 96);
  reinterpret_cast<uint4 *>(atom)[l] = v;
}

__device__ __forceinline__ void sf_reorder_atom(const uint32_t *rows, int nrows,
                                                uint32_t *atom) {
  const int l = threadIdx.x & 31;
  uint4 v;
  v.x = l < nrows ? rows[l] : 0u;
  v.y = l + 32 < nrows ? rows[l + 32] : 0u;
  v.z = l + 64 < nrows ? rows[l + 64] : 0u;
  v.w = l + 96 < nrows ? rows[l + 96] : 0u;
  reinterpret_cast<uint4 *>(atom)[l] = v;
}

// kH: 64 selects the tuned epilogue; 0 = any H (generic epilogue).
// kNSUB: MMA sub-blocks per key tile (each its own accumulator, same A).
// kG: key tiles per pipeline item (one smem stage, one accumulator slot of
//     kG accumulators); kG > 1 needs kNSUB == 1. Batching tiles amortises
//     the per-item waits, fences and commits of the issuing threads.
// kNACC: TMEM accumulator slots. kSTAGES: smem stages (kG tiles each).
// kQBUF: query-block smem buffers. kEPI: epilogue warps (4 or 8).
// kFP8: e4m3 + e8m0/32 inputs through the block-scaled MMA.
// kISS: MMA-issuing warps (1 or 2). With 2, items alternate between them so
//     that one warp's waits and commits overlap the other's MMAs.
// kMODE: kModePositions, kModeCausal or kModeCompressed, fixed at compile
//     time so that each instance carries only its own schedule and row rule.
//
// Warps: 0 TMA producer, 1 MMA issuer (+ TMEM owner), 2 .. 1+kEPI epilogue,
// then (fp8) the scale-factor warp, then (kISS == 2) the second issuer.
template <int kH, int kNSUB, int kG, int kNACC, int kSTAGES, int kQBUF, int kEPI, bool kFP8,
          int kISS, int kMODE>
__global__ void __launch_bounds__((2 + kEPI + (kFP8 ? 1 : 0) + (kISS - 1)) * 32, 1)
    score_kernel(const __grid_constant__ CUtensorMap tmap_k,
                 const __grid_constant__ CUtensorMap tmap_q,
                 const __grid_constant__ CUtensorMap tmap_ksf,
                 const __grid_constant__ CUtensorMap tmap_qsf,
                 const ScoreParams p) {
  static_assert(kEPI == 4 || kEPI == 8 || kEPI == 16, "epilogue warps");
  static_assert(kH == 64 || kEPI == 4, "generic epilogue uses 4 warps");
  static_assert(kG == 1 || kNSUB == 1, "tile batching is for single sub-block queries");
  static_assert(kISS == 1 || kISS == 2, "issuers");
  constexpr int kSFWarp = 2 + kEPI;                        // fp8 scale-factor warp
  constexpr int kIss2Warp = 2 + kEPI + (kFP8 ? 1 : 0);     // second MMA issuer
  static_assert(3 * (kSTAGES + kQBUF) + 2 * kNACC <= 63, "barrier budget");
  constexpr int kGroups = kEPI / 4;
  constexpr int kAPS = kG;                       // accumulators per slot
  extern __shared__ uint8_t smem_raw[];
  // 1024-byte aligned, by pointer arithmetic on the shared array, so that
  // the compiler keeps every access through it in the shared address space
  uint8_t *smem = smem_raw + ((1024u - (smem_u32(smem_raw) & 1023u)) & 1023u);
  const ScoreSmem L(kSTAGES, kQBUF, kNSUB, p.n_cols, kFP8, kEPI, kG);
  uint8_t *sk = smem + L.off_k;
  uint8_t *sq = smem + L.off_q;
  uint8_t *sksf = smem + L.off_ksf;
  uint8_t *sqsf = smem + L.off_qsf;
  uint64_t *bars = reinterpret_cast<uint64_t *>(smem + L.off_bar);
  uint64_t *full_k = bars;                       // [kSTAGES]
  uint64_t *empty_k = full_k + kSTAGES;          // [kSTAGES]
  uint64_t *q_full = empty_k + kSTAGES;          // [kQBUF]
  uint64_t *q_empty = q_full + kQBUF;            // [kQBUF]
  uint64_t *acc_full = q_empty + kQBUF;          // [kNACC]
  uint64_t *acc_empty = acc_full + kNACC;        // [kNACC]
  uint64_t *sf_ready = acc_empty + kNACC;        // [kSTAGES] fp8: A scales in TMEM
  uint64_t *sfq_ready = sf_ready + kSTAGES;      // [kQBUF]   fp8: B scales in TMEM
  uint64_t *stall_bar = bars + 63;               // self-test: never completed
  uint32_t *misc = reinterpret_cast<uint32_t *>(smem + L.off_misc);
  uint32_t *tmem_base_slot = misc;               // written by tcgen05.alloc
  volatile int *abort_flag = reinterpret_cast<volatile int *>(misc + 1);
  CtaRange *range_slot = reinterpret_cast<CtaRange *>(misc + 16);

  const int warp = threadIdx.x / 32;
  const int lane = threadIdx.x % 32;
  const int tqt = p.tq_sub * kNSUB;              // tokens per query block
  const int n_cols = p.n_cols;
  const int atoms = sf_atoms(n_cols);
  uint32_t tmem_cols = 32;
  while (tmem_cols < static_cast<uint32_t>(tmem_cols_needed(kNACC, kAPS, n_cols, kSTAGES, kG,
                                                            kQBUF, kNSUB, kFP8)))
    tmem_cols <<= 1;

  // Set-up that reads nothing written by earlier work on the stream runs
  // before the dependency wait, overlapping the previous kernel's tail.
  if (warp == 0 && lane == 0) {
    for (int i = 0; i < kSTAGES; ++i) { mbar_init(full_k + i, 1); mbar_init(empty_k + i, 1); }
    for (int i = 0; i < kQBUF; ++i) { mbar_init(q_full + i, 1); mbar_init(q_empty + i, kISS); }
    for (int i = 0; i < kNACC; ++i) { mbar_init(acc_full + i, 1); mbar_init(acc_empty + i, kEPI); }
    if constexpr (kFP8) {
      for (int i = 0; i < kSTAGES; ++i) mbar_init(sf_ready + i, 1);
      for (int i = 0; i < kQBUF; ++i) mbar_init(sfq_ready + i, 1);
    }
    mbar_init(stall_bar, 1);
    *abort_flag = 0;
    fence_mbar_init();
    tma_prefetch_desc(&tmap_k);
    tma_prefetch_desc(&tmap_q);
    if constexpr (kFP8) {
      tma_prefetch_desc(&tmap_ksf);
      tma_prefetch_desc(&tmap_qsf);
    }
  } else if (warp == 1) {
    tmem_alloc(tmem_base_slot, tmem_cols);
    tmem_relinquish();
  }
  grid_dep_wait();
  grid_dep_launch_dependents();

  // Decode positions are read by every role many times: keep a copy here.
  int *spos = reinterpret_cast<int *>(smem + L.off_pos);
  const bool pos_staged = kMODE == kModePositions && p.T <= kPosCap;
  if (pos_staged)
    for (int i = threadIdx.x; i < p.T; i += blockDim.x) spos[i] = __ldg(p.positions + i);
  __syncthreads();
  ScoreParams P = p;
  // constants from here on: the other modes' code folds away
  P.mode = kMODE == kModeCompressed ? static_cast<int>(kModePositions) : kMODE;
  P.compressed = kMODE == kModeCompressed;
  if (pos_staged) P.positions = spos;
  if (warp == 0) {
    CtaRange R;
    // CAUSAL: a cu_seqlens array that failed its check leaves the CTA no work
    if (kMODE == kModeCausal && *p.cu_bad) {
      R = CtaRange{};
    } else {
      cta_range(P, tqt, R);
    }
    if (lane == 0) *range_slot = R;
  }
  tc_fence_before_sync();
  __syncthreads();
  tc_fence_after_sync();
  const uint32_t tmem_base = *tmem_base_slot;
  const CtaRange R = *range_slot;
  const WaitCtl ctl{abort_flag, p.err, p.err_info, p.wait_limit_ns};
  const uint32_t sfa_col0 = kNACC * kAPS * n_cols;             // fp8 only
  const uint32_t sfb_col0 = sfa_col0 + kSTAGES * kG * 4;       // fp8 only

  if (warp == 0) {
    // ---------------- TMA producer ----------------
    if (lane == 0 && R.a_count > 0) {
      Ring st, qb;
      uint32_t k_issued = 0, q_issued = 0, k_last_phase = 0, q_last_phase = 0;
      ItemCursor c;
      cursor_start(P, tqt, R, c);
      // fp8: a paged tile's scale words come page by page, each box at its
      // row offset (no window padding: page boxes start on 4-word rows)
      const uint32_t tile_tx =
          L.k_stage_bytes + (kFP8 ? (p.block_table ? kBlockM * 4 : kSfBoxBytesK) : 0);
      // keys read once (a cache per token) leave L2 first
      const bool k_once = p.k_once != 0;
      const uint64_t pol = l2_policy_evict_first();
      auto load_k3 = [&](void *dst, int32_t c0, int32_t c1, int32_t c2) {
        if (k_once) tma_load_3d_hint(dst, &tmap_k, full_k + st.idx, c0, c1, c2, pol);
        else tma_load_3d(dst, &tmap_k, full_k + st.idx, c0, c1, c2);
      };
      auto load_ksf2 = [&](void *dst, int32_t c0, int32_t c1) {
        if (k_once) tma_load_2d_hint(dst, &tmap_ksf, full_k + st.idx, c0, c1, pol);
        else tma_load_2d(dst, &tmap_ksf, full_k + st.idx, c0, c1);
      };
      bool need_q = true;
      while (c.left > 0) {
        const int g = cursor_tiles<kG>(c);
        if (need_q) {
          const int nsub = (c.q.ntok + p.tq_sub - 1) / p.tq_sub;
          if (!mbar_wait(q_empty + qb.idx, qb.phase ^ 1u, ctl, 2)) break;
          mbar_arrive_expect_tx(q_full + qb.idx,
                                nsub * (L.q_sub_bytes + (kFP8 ? sf_box_bytes_q(n_cols) : 0)));
          for (int s = 0; s < nsub; ++s) {
            uint8_t *dst = sq + (qb.idx * kNSUB + s) * L.q_sub_bytes;
            const int row = (c.q.t0 + s * p.tq_sub) * p.H;
            if constexpr (kFP8) {
              tma_load_2d(dst, &tmap_q, q_full + qb.idx, 0, row);
              tma_load_2d(sqsf + (qb.idx * kNSUB + s) * L.q_sf_bytes, &tmap_qsf,
                          q_full + qb.idx, row & ~(kSfPad - 1), 0);
            } else {
              tma_load_2d(dst, &tmap_q, q_full + qb.idx, 0, row);
              tma_load_2d(dst + n_cols * 128, &tmap_q, q_full + qb.idx, 64, row);
            }
          }
          q_issued |= 1u << qb.idx;
          q_last_phase = (q_last_phase & ~(1u << qb.idx)) | (qb.phase << qb.idx);
          need_q = false;
        }
        if (!mbar_wait(empty_k + st.idx, st.phase ^ 1u, ctl, 3)) break;
        mbar_arrive_expect_tx(full_k + st.idx, g * tile_tx);
        for (int i = 0; i < g; ++i) {
          uint8_t *dst = sk + (st.idx * kG + i) * L.k_stage_bytes;
          const int y = c.q.y0 + (c.j + i) * kBlockM;
          if (p.block_table) {
            // paged cache: the tile's slots y .. y+127 from one page, or from
            // 128/page_size pages (one box each, at its row offset in the
            // tile; 128-byte swizzle atoms are 8 rows, boxes >= 16 rows).
            // Past the block table, an id past the pool: TMA fills zeros.
            // fp8: each box's scale words land at the same row offset of the
            // tile's scale window (a box starts on a page row that is a
            // multiple of 16, so its words are 16-byte aligned).
            const int box = p.page_shift >= 7 ? kBlockM : (1 << p.page_shift);
            for (int b = 0; b < kBlockM; b += box) {
              const int lp = (y + b) >> p.page_shift;
              const int row = (y + b) & ((1 << p.page_shift) - 1);
              const int page =
                  lp < p.pages_per_seq
                      ? __ldg(p.block_table + static_cast<int64_t>(c.q.z) * p.pages_per_seq + lp)
                      : p.num_pages;
              load_k3(dst + b * 128, 0, row, page);
              if constexpr (kFP8) {
                // boxes of >= 32 rows: at their row offset (a multiple of 128
                // bytes); 16-row boxes: one 128-byte slot each
                const int sf_off = box >= 32 ? 4 * b : 8 * b;
                load_ksf2(sksf + (st.idx * kG + i) * L.k_sf_bytes + sf_off, row, page);
              } else {
                load_k3(dst + kBlockM * 128 + b * 128, 64, row, page);
              }
            }
            continue;
          }
          load_k3(dst, 0, y, c.q.z);
          if constexpr (kFP8) {
            load_ksf2(sksf + (st.idx * kG + i) * L.k_sf_bytes, y & ~(kSfPad - 1), c.q.z);
          } else {
            load_k3(dst + kBlockM * 128, 64, y, c.q.z);
          }
        }
        k_issued |= 1u << st.idx;
        k_last_phase = (k_last_phase & ~(1u << st.idx)) | (st.phase << st.idx);
        st.next(kSTAGES);
        if (cursor_step(P, tqt, c, g) && c.left > 0) {
          need_q = true;
          qb.next(kQBUF);
        }
      }
      // Let every copy this thread started land before the CTA can exit.
      for (int i = 0; i < kSTAGES; ++i)
        if (k_issued >> i & 1u) mbar_drain(full_k + i, k_last_phase >> i & 1u, p.drain_limit_ns);
      for (int i = 0; i < kQBUF; ++i)
        if (q_issued >> i & 1u) mbar_drain(q_full + i, q_last_phase >> i & 1u, p.drain_limit_ns);
    }
  } else if (warp == 1 || (kISS == 2 && warp == kIss2Warp)) {
    // ---------------- MMA issuers (each walks every item, issues its own) ----
    const int my_parity = warp == 1 ? 0 : 1;
    // self-test of the failure path: a wait that runs out (nothing arrives)
    const bool stalled = p.selftest_stall && warp == 1 && !mbar_wait(stall_bar, 0, ctl, 31);
    if (R.a_count > 0 && !stalled) {
      Ring st, qb, ac;
      uint64_t *last_commit = nullptr;
      uint32_t last_commit_phase = 0;
      ItemCursor c;
      cursor_start(P, tqt, R, c);
      bool new_q = true;
      int nsub = 1;
      // Shared-memory descriptors advance by (bytes >> 4) in their low field.
      const uint64_t k_desc0 = sdesc_kmajor_sw128(smem_u32(sk));
      const uint64_t q_desc0 = sdesc_kmajor_sw128(smem_u32(sq));
      const uint32_t k_tile_step = L.k_stage_bytes >> 4;
      const uint32_t q_sub_step = L.q_sub_bytes >> 4;
      int item = 0;
      while (c.left > 0) {
        const int g = cursor_tiles<kG>(c);
        const bool mine = kISS == 1 || (item & 1) == my_parity;
        ++item;
        if (new_q) {
          nsub = (c.q.ntok + p.tq_sub - 1) / p.tq_sub;
          // fp8: the scale warp has also put the block's B scales in TMEM
          if (!mbar_wait(kFP8 ? sfq_ready + qb.idx : q_full + qb.idx, qb.phase, ctl, 12)) break;
          tc_fence_after_sync();
          new_q = false;
        }
        const int nslots = kG > 1 ? 1 : nsub;
        if (!mine) {   // the other issuer's item: keep the rings in step
          for (int s = 0; s < nslots; ++s) ac.next(kNACC);
          st.next(kSTAGES);
          if (cursor_step(P, tqt, c, g)) {
            if (lane == 0) mma_commit(q_empty + qb.idx);
            __syncwarp();
            qb.next(kQBUF);
            new_q = true;
          }
          continue;
        }
        if (!mbar_wait(full_k + st.idx, st.phase, ctl, 13)) break;
        if constexpr (kFP8) {   // and the item's A scales
          if (!mbar_wait(sf_ready + st.idx, st.phase, ctl, 15)) break;
        }
        tc_fence_after_sync();
        bool ok = true;
        for (int s = 0; s < nslots; ++s) {
          if (!mbar_wait(acc_empty + ac.idx, ac.phase ^ 1u, ctl, 14)) { ok = false; break; }
          tc_fence_after_sync();
          if (lane == 0) {
            const int sub = kG > 1 ? 0 : s;
            const uint64_t bdesc = q_desc0 + (qb.idx * kNSUB + sub) * q_sub_step;
            const int nacc = kG > 1 ? g : 1;
            for (int i = 0; i < nacc; ++i) {
              const uint32_t d_tmem = tmem_base + (ac.idx * kAPS + i) * n_cols;
              const uint64_t adesc = k_desc0 + (st.idx * kG + i) * k_tile_step;
              if constexpr (kFP8) {
                const uint32_t sfa = tmem_base + sfa_col0 + (st.idx * kG + i) * 4;
                const uint32_t sfb = tmem_base + sfb_col0 + (qb.idx * kNSUB + sub) * 4 * atoms;
                const uint32_t idesc = idesc_mxf8_e4m3(kBlockM, n_cols, 0, 0);
#pragma unroll
                for (int kk = 0; kk < kHeadDim / 32; ++kk)
                  mma_mxf8_ss(d_tmem, adesc + kk * 2, bdesc + kk * 2,
                              idesc | idesc_mxf8_e4m3(0, 0, kk, kk), sfa, sfb, kk > 0 ? 1u : 0u);
              } else {
                const uint32_t idesc = idesc_bf16_f32(kBlockM, n_cols);
                const uint32_t a_half = (kBlockM * 128) >> 4;
                const uint32_t b_half = (n_cols * 128) >> 4;
#pragma unroll
                for (int kk = 0; kk < kHeadDim / 16; ++kk) {
                  const uint32_t half = kk / 4, koff = (kk % 4) * 2;
                  mma_f16_ss(d_tmem, adesc + half * a_half + koff, bdesc + half * b_half + koff,
                             idesc, kk > 0 ? 1u : 0u);
                }
              }
            }
            mma_commit(acc_full + ac.idx);
            last_commit = acc_full + ac.idx;
            last_commit_phase = ac.phase;
          }
          __syncwarp();
          ac.next(kNACC);
        }
        if (!ok) break;
        if (lane == 0) mma_commit(empty_k + st.idx);   // stage free once these MMAs finish
        __syncwarp();
        st.next(kSTAGES);
        if (cursor_step(P, tqt, c, g)) {
          if (lane == 0) mma_commit(q_empty + qb.idx);
          __syncwarp();
          qb.next(kQBUF);
          new_q = true;
        }
      }
      // MMAs still in flight must finish before TMEM is released.
      if (lane == 0 && last_commit) mbar_drain(last_commit, last_commit_phase, p.drain_limit_ns);
      __syncwarp();
    }
  } else if (kFP8 && warp == kSFWarp) {
    // ---------------- fp8 scale factors ----------------
    // Reorders each item's (and each query block's) scale words into the
    // 128-row atoms tcgen05.cp copies, copies them into TMEM and commits to
    // sf_ready / sfq_ready, so the MMA warp only waits and issues.
    if (R.a_count > 0) {
      Ring st, qb;
      ItemCursor c;
      cursor_start(P, tqt, R, c);
      bool new_q = true;
      uint64_t *last_commit = nullptr;
      uint32_t last_commit_phase = 0;
      while (c.left > 0) {
        const int g = cursor_tiles<kG>(c);
        if (new_q) {
          const int nsub = (c.q.ntok + p.tq_sub - 1) / p.tq_sub;
          if (!mbar_wait(q_full + qb.idx, qb.phase, ctl, 16)) break;
          for (int s = 0; s < nsub; ++s) {
            uint8_t *sf = sqsf + (qb.idx * kNSUB + s) * L.q_sf_bytes;
            const int r = ((c.q.t0 + s * p.tq_sub) * p.H) & (kSfPad - 1);
            for (int a = 0; a < atoms; ++a)
              sf_reorder_atom(reinterpret_cast<const uint32_t *>(sf) + r + 128 * a,
                              min(128, n_cols - 128 * a),
                              reinterpret_cast<uint32_t *>(sf + sf_raw_bytes_q(n_cols) + 512 * a));
          }
          fence_proxy_async_smem();
          __syncwarp();
          if (lane == 0) {
            tc_fence_after_sync();
            for (int s = 0; s < nsub; ++s) {
              uint8_t *sf = sqsf + (qb.idx * kNSUB + s) * L.q_sf_bytes;
              for (int a = 0; a < atoms; ++a)
                tmem_cp_32x128b_x4(
                    tmem_base + sfb_col0 + (qb.idx * kNSUB + s) * 4 * atoms + 4 * a,
                    sdesc_rows16_noswizzle(smem_u32(sf + sf_raw_bytes_q(n_cols) + 512 * a)));
            }
            mma_commit(sfq_ready + qb.idx);
            last_commit = sfq_ready + qb.idx;
            last_commit_phase = qb.phase;
          }
          __syncwarp();
          new_q = false;
        }
        if (!mbar_wait(full_k + st.idx, st.phase, ctl, 17)) break;
        for (int i = 0; i < g; ++i) {
          uint8_t *sf = sksf + (st.idx * kG + i) * L.k_sf_bytes;
          const int r = (c.q.y0 + (c.j + i) * kBlockM) & (kSfPad - 1);
          if (p.block_table && p.page_shift < 5)
            sf_reorder_atom_pages16(reinterpret_cast<const uint32_t *>(sf),
                                    reinterpret_cast<uint32_t *>(sf + kSfRawBytesK));
          else
            sf_reorder_atom(reinterpret_cast<const uint32_t *>(sf) + r, 128,
                            reinterpret_cast<uint32_t *>(sf + kSfRawBytesK));
        }
        fence_proxy_async_smem();
        __syncwarp();
        if (lane == 0) {
          tc_fence_after_sync();
          for (int i = 0; i < g; ++i)
            tmem_cp_32x128b_x4(tmem_base + sfa_col0 + (st.idx * kG + i) * 4,
                               sdesc_rows16_noswizzle(smem_u32(
                                   sksf + (st.idx * kG + i) * L.k_sf_bytes + kSfRawBytesK)));
          mma_commit(sf_ready + st.idx);
          last_commit = sf_ready + st.idx;
          last_commit_phase = st.phase;
        }
        __syncwarp();
        st.next(kSTAGES);
        if (cursor_step(P, tqt, c, g) && c.left > 0) {
          qb.next(kQBUF);
          new_q = true;
        }
      }
      // copies still in flight must land before TMEM is released
      if (lane == 0 && last_commit) mbar_drain(last_commit, last_commit_phase, p.drain_limit_ns);
      __syncwarp();
    }
  } else if (warp < 2 + kEPI) {
    // ---------------- epilogue ----------------
    const int epi = warp - 2;                  // 0 .. kEPI-1
    const int quad = warp & 3;                 // TMEM lane quadrant of this warp
    const int group = epi / 4;                 // token subset of this warp
    const uint32_t lane_addr = static_cast<uint32_t>(quad * 32) << 16;
    // Fully masked tiles first, while the first loads are in flight: each run
    // of masked tiles of a query block is one contiguous slot range per
    // token, written with 16-byte stores. The block's rows go to different
    // warps (kEPI / ntok warps a row when there are fewer rows than warps), so
    // that the stores of all rows are in flight together: a row's stores take
    // a fixed time of their own, which one warp walking the rows in turn paid
    // once per row.
    if (R.f_count > 0) {
      QBlk q;
      int j = R.f_j;
      make_qb(P, tqt, R.f_seq, R.f_b, R.f_seqoff, q);
      int64_t left = R.f_count;
      while (left > 0) {
        const int64_t seg = min64(left, q.ntr - j);
        const int64_t lo = static_cast<int64_t>(j) * kBlockM;
        const int64_t hi = min64(static_cast<int64_t>(j + seg) * kBlockM, q.row_len);
        const int ntok = q.ntok;
        const int wpr = kEPI / ntok > 1 ? kEPI / ntok : 1;   // warps per row
        const int ngrp = kEPI / wpr;                          // >= ntok
        float *const rows = p.scores + q.out0;
        const int64_t row_len = q.row_len;
        for (int i = epi / wpr; i < ntok; i += ngrp)
          fill_mask(rows + i * row_len, lo, hi, (epi % wpr) * 32 + lane, wpr * 32);
        left -= seg;
        if (left > 0) {
          do {
            if (!next_qb(P, tqt, q)) { left = 0; break; }
          } while (q.act == q.ntr);
          j = q.act;
        }
      }
    }
    if (R.a_count > 0) {
      Ring ac;
      ItemCursor c;
      cursor_start(P, tqt, R, c);
      bool ok = true, new_q = true;
      int nsub = 1;
      // H=64: this warp's w rows for the current query block (warp-private).
      // kG == 1: the warp groups split each sub-block's tokens; kG > 1: they
      // split the item's tiles, and every group takes all tokens.
      float *wrows = reinterpret_cast<float *>(smem + L.off_w) + epi * kWRowsPerWarp * 64;
      const int per = kG > 1 ? p.tq_sub : (p.tq_sub + kGroups - 1) / kGroups;
      while (c.left > 0 && ok) {
        const int g = cursor_tiles<kG>(c);
        const QBlk &q = c.q;
        if (new_q) {
          nsub = (q.ntok + p.tq_sub - 1) / p.tq_sub;
          if constexpr (kH == 64) {
            __syncwarp();
            for (int s = 0; s < nsub; ++s) {
              const int ntok_s = min(p.tq_sub, q.ntok - s * p.tq_sub);
              const int i_lo = kG > 1 ? 0 : min(ntok_s, group * per);
              const int i_hi = kG > 1 ? ntok_s : min(ntok_s, i_lo + per);
              for (int idx = lane; idx < (i_hi - i_lo) * 16; idx += 32) {
                const int u = idx / 16, cc = idx % 16;
                const int t = q.t0 + s * p.tq_sub + i_lo + u;
                reinterpret_cast<float4 *>(wrows + (s * per + u) * 64)[cc] =
                    __ldg(reinterpret_cast<const float4 *>(p.w + static_cast<int64_t>(t) * 64) + cc);
              }
            }
            __syncwarp();
          }
          new_q = false;
        }
        const int nslots = kG > 1 ? 1 : nsub;
        for (int s = 0; s < nslots; ++s) {
          if (!mbar_wait(acc_full + ac.idx, ac.phase, ctl, 22)) { ok = false; break; }
          tc_fence_after_sync();
          const int sub = kG > 1 ? 0 : s;
          const int i0 = sub * p.tq_sub;
          const int ntok_s = min(p.tq_sub, q.ntok - i0);
          const int nacc = kG > 1 ? g : 1;
          for (int a = 0; a < nacc; ++a) {
            if (kG > 1 && kGroups > 1 && a % kGroups != group) continue;
            const int64_t slot = static_cast<int64_t>(c.j + a) * kBlockM + quad * 32 + lane;
            const bool in_row = slot < q.row_len;
            const uint32_t tbase = tmem_base + lane_addr + (ac.idx * kAPS + a) * n_cols;
            if constexpr (kH == 64) {
              // this warp's tokens of the sub-block: adjacent pair (or one)
              const int i_lo = kG > 1 ? 0 : min(ntok_s, group * per);
              const int i_hi = kG > 1 ? ntok_s : min(ntok_s, i_lo + per);
              const float *wsh = wrows + (sub * per) * 64;
              if constexpr (kG == 1) {
                head_sums_h64_pipelined(tbase, i_lo, i_hi, wsh, [&](int i, float acc) {
                  const int lv = qb_last_valid(P, q, i0 + i);
                  if (in_row)
                    p.scores[q.out0 + (i0 + i) * q.row_len + slot] =
                        slot <= lv ? acc : kMaskBound;
                });
              } else {
                for (int i = i_lo; i < i_hi; ++i) {
                  const float acc = head_sum_h64(tbase + i * 64, wsh + (i - i_lo) * 64);
                  const int lv = qb_last_valid(P, q, i0 + i);
                  if (in_row)
                    p.scores[q.out0 + (i0 + i) * q.row_len + slot] = slot <= lv ? acc : kMaskBound;
                }
              }
            } else {
              // any H: walk the sub-block's columns in 16-wide chunks
              const int H = p.H, ncols = ntok_s * H;
              const float *wsub = p.w + static_cast<int64_t>(q.t0 + i0) * H;
              float acc = 0.f;
              int tok = 0, h = 0;
              for (int c0 = 0; c0 < ncols; c0 += 16) {
                float v[16];
                tmem_ld16_wait(tbase + c0, v);
#pragma unroll
                for (int cc = 0; cc < 16; ++cc) {
                  if (c0 + cc < ncols) {
                    acc = fmaf(__ldg(wsub + c0 + cc), fmaxf(v[cc], 0.f), acc);
                    if (++h == H) {
                      const int lv = qb_last_valid(P, q, i0 + tok);
                      if (in_row)
                        p.scores[q.out0 + (i0 + tok) * q.row_len + slot] =
                            slot <= lv ? acc : kMaskBound;
                      acc = 0.f;
                      h = 0;
                      ++tok;
                    }
                  }
                }
              }
            }
          }
          tc_fence_before_sync();
          __syncwarp();
          if (lane == 0) mbar_arrive(acc_empty + ac.idx);
          ac.next(kNACC);
        }
        if (ok && cursor_step(P, tqt, c, g)) new_q = true;
      }
    }
  }

  tc_fence_before_sync();
  __syncthreads();
  tc_fence_after_sync();
  if (warp == 1) tmem_dealloc(tmem_base, tmem_cols);
}

}  // namespace dsa
