"""Seeded synthetic inputs for the lightning indexer (score + top-k).

This module is shared by the fp64 oracle and the CUDA path. It draws the
inputs and encodes them into the storage formats the indexer reads (bf16 bit
patterns; fp8-e4m3 bytes with block-32 e8m0 scale bytes). It holds none of the
indexer's arithmetic: it never decodes a stored value back into a number and
never computes a score or a selection.

Recipe (all workloads): ``numpy.random.default_rng(seed)`` (PCG64), draws in
the order q, k, w, positions. Gaussian values are drawn as float32 in fixed
chunks of ``CHUNK`` elements; bf16 storage is round-to-nearest-even of those
float32 values. w is float32 ``N(0,1) * w_scale``. positions are
``rng.integers(lo, hi)`` (int32, hi exclusive).

Workload shapes follow the pages' decode and prefill statements: DeepSeek-V3.2
Sparse Indexer Kernel API Reference (decode step, n_tokens one per sequence,
head_dim = 128, key cache ``[n_tokens, max_seq_len, head_dim]``), and Sparse
Attention Indexer MX BF16Score Kernel API Reference (prefill self-scoring,
queries == keys, head_dim == 128, block-32 e8m0 scales).
"""
from __future__ import annotations

import dataclasses
import os
from typing import Optional

import numpy as np

CHUNK = 1 << 22          # gaussian draws per call (fixes the stream layout)
MX_BLOCK = 32            # e8m0 scale block along D
E4M3_MAX = 448.0         # largest finite e4m3 magnitude

MODE_POSITIONS = 0       # decode: slot s valid iff s <= positions[t]
MODE_CAUSAL = 1          # packed prefill: slot s valid iff s <= t (sequence-local)
MODE_COMPRESSED = 2      # pooled (C4) keys: slot j valid iff (j+1)*r <= query_start+t+1
DTYPE_BF16 = 0
DTYPE_FP8 = 1


@dataclasses.dataclass(frozen=True)
class Workload:
    """One synthetic indexer problem (sizes, mask rule, value distributions)."""
    name: str
    mode: int                      # MODE_POSITIONS, MODE_CAUSAL or MODE_COMPRESSED
    T: int                         # query tokens
    H: int                         # indexer heads
    D: int                         # head_dim
    index_topk: int
    dtype: int = DTYPE_BF16
    S: int = 0                     # POSITIONS: slots per sequence cache; COMPRESSED: pooled slots
    shared_cache: bool = False     # POSITIONS: one cache for every token
    pos_lo: int = 0                # POSITIONS: positions ~ U[pos_lo, pos_hi)
    pos_hi: int = 0
    seqlens: tuple = ()            # CAUSAL: packed sequence lengths
    w_scale: float = 1.0
    seed: int = 0
    query_start: int = 0           # COMPRESSED: absolute position of query 0
    compress_ratio: int = 0        # COMPRESSED: tokens pooled per slot
    page_size: int = 0             # POSITIONS, one cache per token: > 0 = paged cache

    @property
    def paged(self) -> bool:
        return self.mode == MODE_POSITIONS and not self.shared_cache and self.page_size > 0

    @property
    def pages_per_seq(self) -> int:
        """Block-table entries per token (paged caches)."""
        return -(-self.S // self.page_size) if self.paged else 0

    @property
    def num_pages(self) -> int:
        """Pages in the pool (paged caches): exactly the pages the tokens use."""
        return self.T * self.pages_per_seq

    @property
    def num_seqs(self) -> int:
        if self.mode == MODE_CAUSAL:
            return len(self.seqlens)
        if self.mode == MODE_COMPRESSED:
            return 1
        return 1 if self.shared_cache else self.T

    @property
    def key_slots(self) -> int:
        """Rows of the key cache buffer (slots of all sequences; paged: of
        all pages)."""
        if self.mode == MODE_CAUSAL:
            return int(sum(self.seqlens))
        if self.paged:
            return self.num_pages * self.page_size
        return self.S * self.num_seqs

    @property
    def k_seq_stride(self) -> int:
        """Elements between consecutive sequences' caches (POSITIONS)."""
        if self.mode != MODE_POSITIONS or self.shared_cache or self.paged:
            return 0
        return self.S * self.D

    def cu_seqlens(self) -> np.ndarray:
        return np.concatenate([[0], np.cumsum(self.seqlens)]).astype(np.int32)


# The five workloads: a tiny decode case, a decode batch, a long-context fp8
# decode, a causal prefill and a packed ragged prefill.
WORKLOADS = {
    "tiny_decode": Workload("tiny_decode", MODE_POSITIONS, T=4, H=4, D=128,
                            index_topk=64, S=1024, pos_lo=64, pos_hi=1024,
                            w_scale=1.0 / 2.0),
    "decode_batch": Workload("decode_batch", MODE_POSITIONS, T=16, H=64, D=128,
                             index_topk=2048, S=32768, pos_lo=2048,
                             pos_hi=32768, w_scale=1.0 / 8.0),
    "long_decode_fp8": Workload("long_decode_fp8", MODE_POSITIONS, T=64, H=64,
                                D=128, index_topk=1024, dtype=DTYPE_FP8,
                                S=131072, pos_lo=1024, pos_hi=131072,
                                w_scale=1.0 / 8.0),
    "prefill_causal": Workload("prefill_causal", MODE_CAUSAL, T=8192, H=64,
                               D=128, index_topk=2048, seqlens=(8192,),
                               w_scale=1.0 / 8.0),
    "ragged_prefill": Workload("ragged_prefill", MODE_CAUSAL, T=118784, H=64,
                               D=128, index_topk=2048,
                               seqlens=(4096, 16384, 32768, 65536),
                               w_scale=1.0 / 8.0),
    # the decode batch over a paged cache (pages of 64 slots, scattered over
    # the pool by a random block table)
    "decode_batch_paged": Workload("decode_batch_paged", MODE_POSITIONS, T=16, H=64,
                                   D=128, index_topk=2048, S=32768, pos_lo=2048,
                                   pos_hi=32768, w_scale=1.0 / 8.0, page_size=64),
    # the long-context fp8 decode over a paged cache: 64-slot pages of e4m3
    # keys and of their e8m0 scale rows, scattered by a random block table
    "long_decode_fp8_paged": Workload("long_decode_fp8_paged", MODE_POSITIONS, T=64,
                                      H=64, D=128, index_topk=1024, dtype=DTYPE_FP8,
                                      S=131072, pos_lo=1024, pos_hi=131072,
                                      w_scale=1.0 / 8.0, page_size=64),
    # compressed (C4) indexer, the next step beyond the five: an 8192-token
    # prefill chunk against its 2048 keys pooled 4:1, DSV4's index_topk 1024
    "c4_prefill": Workload("c4_prefill", MODE_COMPRESSED, T=8192, H=64, D=128,
                           index_topk=1024, S=2048, compress_ratio=4,
                           query_start=0, w_scale=1.0 / 8.0),
}


def gaussian_f32(rng: np.random.Generator, n: int) -> np.ndarray:
    """n float32 N(0,1) draws, taken in chunks of CHUNK."""
    out = np.empty(n, dtype=np.float32)
    for i in range(0, n, CHUNK):
        m = min(CHUNK, n - i)
        out[i:i + m] = rng.standard_normal(m, dtype=np.float32)
    return out


def f32_to_bf16_bits(x: np.ndarray) -> np.ndarray:
    """Round float32 to bf16 (nearest, ties to even); returns uint16 bits."""
    u = np.ascontiguousarray(x, dtype=np.float32).view(np.uint32)
    out = np.empty(u.shape, dtype=np.uint16)
    step = 1 << 24
    flat_u, flat_o = u.reshape(-1), out.reshape(-1)
    for i in range(0, flat_u.size, step):
        v = flat_u[i:i + step].astype(np.uint64)
        v = (v + 0x7FFF + ((v >> 16) & 1)) >> 16
        flat_o[i:i + step] = v.astype(np.uint16)
    return out


def f32_to_mx_e4m3(x: np.ndarray):
    """Encode float32 values [..., D] as e4m3 bytes with block-32 e8m0 scales.

    Per block of 32 along D (the MX layout the pages use for ``qr_scale_hbm``,
    ``wq_b_scale`` and ``k_scale_cache``): the scale is the power of two 2^e
    with the smallest e such that 448 * 2^e >= amax (amax over the block,
    floored at 448 * 2^-127 so that e >= -127); byte = e + 127. Each element is
    then x * 2^-e rounded to the nearest e4m3 value, ties to even (|x * 2^-e|
    <= 448, so nothing saturates). Returns (data uint8 [..., D], scale uint8
    [..., D/32]). Row chunks are encoded on a thread pool; every step is exact
    power-of-two arithmetic, so the result does not depend on the chunking.
    """
    x = np.ascontiguousarray(x, dtype=np.float32)
    D = x.shape[-1]
    assert D % MX_BLOCK == 0
    lead = x.shape[:-1]
    blocks = x.reshape(-1, D // MX_BLOCK, MX_BLOCK)
    data = np.empty(blocks.shape, dtype=np.uint8)
    scale = np.empty(blocks.shape[:2], dtype=np.uint8)
    step = max(1, (1 << 20) // D)

    def work(i):
        b = blocks[i:i + step]
        amax = np.maximum(np.abs(b).max(axis=-1).astype(np.float64),
                          E4M3_MAX * 2.0 ** -127)
        m, E = np.frexp(amax)                    # amax = m * 2^E, m in [0.5, 1)
        # 448 = 0.875 * 2^9: 448 * 2^e >= m * 2^E  <=>  e >= E - 9 + log2(m/0.875)
        e = E.astype(np.int64) - 9 + (m > 0.875)
        assert e.min() >= -127 and e.max() <= 127
        scale[i:i + step] = (e + 127).astype(np.uint8)
        y = np.ldexp(b.astype(np.float64), -e[..., None])   # exact scaling
        data[i:i + step] = _e4m3_rne_bytes(y)

    starts = range(0, blocks.shape[0], step)
    if blocks.shape[0] > 4 * step:
        from concurrent.futures import ThreadPoolExecutor
        with ThreadPoolExecutor(max_workers=os.cpu_count() or 1) as ex:
            list(ex.map(work, starts))
    else:
        for i in starts:
            work(i)
    return data.reshape(lead + (D,)), scale.reshape(lead + (D // MX_BLOCK,))


def _e4m3_rne_bytes(y: np.ndarray) -> np.ndarray:
    """Nearest-even e4m3 (bias 7, 3 mantissa bits) code of |y| <= 448."""
    a = np.abs(y)
    sign = np.signbit(y).astype(np.uint16) << 7
    _, F = np.frexp(a)                           # a = m * 2^F, m in [0.5, 1)
    unb = F.astype(np.int64) - 1                 # floor(log2 a) for a > 0
    # subnormal range (a < 2^-6): quantum 2^-9; a carry to 8 is the code of 2^-6
    sub = np.rint(np.ldexp(a, 9))
    # normal range: quantum 2^(unb-3); a mantissa carry to 8 bumps the exponent
    unb_c = np.maximum(unb, -6)
    mant = np.rint((np.ldexp(a, -unb_c) - 1.0) * 8.0)
    normal = ((unb_c + 7) << 3) + mant.astype(np.int64)
    code = np.where((a == 0) | (unb < -6), sub.astype(np.int64), normal)
    assert code.max() <= 0x7E
    return (code.astype(np.uint16) | sign).astype(np.uint8)


def _values(rng, n, kind):
    if kind == "int":
        return rng.integers(-3, 4, size=n).astype(np.float32)
    return gaussian_f32(rng, n)


def _encode(xf, dtype):
    if dtype == DTYPE_BF16:
        return f32_to_bf16_bits(xf), None
    return f32_to_mx_e4m3(xf)


def generate(wl: Workload, value_kind: str = "gauss",
             seed: Optional[int] = None) -> dict:
    """Draw one workload's inputs (host numpy arrays, storage formats).

    value_kind "gauss": q, k ~ N(0,1), w ~ N(0,1) * w_scale (the pages'
    workloads). "int": q, k uniform integers in [-3, 3], w uniform in
    {-1, -1/2, 1/2, 1}: every product and sum of the indexer is then an exact
    fp32 value, so a correct fp32 kernel reproduces the exact result.

    Keys of the returned dict: q ([T,H,D] uint16 bf16 bits or uint8 e4m3),
    q_scale ([T,H,D/32] uint8 or None), k ([key_slots, D]), k_scale, w
    ([T,H] float32), positions ([T] int32, POSITIONS only), cu_seqlens
    ([num_seqs+1] int32, CAUSAL only). COMPRESSED draws neither: validity
    follows from query_start and compress_ratio. A paged cache (page_size >
    0) draws k as a pool of num_pages pages ([num_pages*page_size, D]) and,
    after the positions, block_table ([T, pages_per_seq] int32): a random
    permutation of the page ids, so that each token's pages are scattered
    over the pool.
    """
    rng = np.random.default_rng(wl.seed if seed is None else seed)
    T, H, D = wl.T, wl.H, wl.D
    q, q_scale = _encode(_values(rng, T * H * D, value_kind).reshape(T, H, D),
                         wl.dtype)
    k, k_scale = _encode(
        _values(rng, wl.key_slots * D, value_kind).reshape(wl.key_slots, D),
        wl.dtype)
    if value_kind == "int":
        w = rng.choice(np.array([-1.0, -0.5, 0.5, 1.0], dtype=np.float32),
                       size=T * H).reshape(T, H)
    else:
        w = (gaussian_f32(rng, T * H) * np.float32(wl.w_scale)).reshape(T, H)
    out = dict(q=q, q_scale=q_scale, k=k, k_scale=k_scale, w=w,
               positions=None, cu_seqlens=None, block_table=None)
    if wl.mode == MODE_POSITIONS:
        out["positions"] = rng.integers(wl.pos_lo, wl.pos_hi, size=T,
                                        dtype=np.int32)
        if wl.paged:
            out["block_table"] = rng.permutation(wl.num_pages).astype(
                np.int32).reshape(T, wl.pages_per_seq)
    elif wl.mode == MODE_CAUSAL:
        out["cu_seqlens"] = wl.cu_seqlens()
    return out


# ---- the indexer's consumer: sparse MQA over top-k key indices ----------------

@dataclasses.dataclass(frozen=True)
class MqaWorkload:
    """One synthetic sparse-MQA problem: q [B,S,H,D], one kv head [B,K,D],
    sinks [H], index rows [B,S,K_top] (NeMo AutoModel optimized_kernels,
    sparse_attention_torch)."""
    name: str
    B: int
    S: int
    H: int
    K: int
    K_top: int
    D: int = 128
    causal: bool = False        # token s of a batch picks among keys [0, s]
    seed: int = 0

    @property
    def sm_scale(self) -> float:
        return float(self.D) ** -0.5


MQA_WORKLOADS = {
    # the decode batch's consumer: one token per sequence, its 2048 selected
    # slots of a 32768-slot cache
    "mqa_decode": MqaWorkload("mqa_decode", B=16, S=1, H=64, K=32768, K_top=2048),
    # the causal prefill's consumer: 8192 tokens, each its 2048 selected keys
    # among the ones at or before it (-1 padded below 2048 visible keys)
    "mqa_prefill": MqaWorkload("mqa_prefill", B=1, S=8192, H=64, K=8192, K_top=2048,
                               causal=True),
}


def generate_mqa(wl: MqaWorkload, seed: Optional[int] = None) -> dict:
    """Draw a sparse-MQA problem (host arrays, storage formats).

    ``numpy.random.default_rng(seed)``, draws in the order q, kv, sinks,
    index rows. q, kv ~ N(0,1) as bf16 bits; sinks ~ N(0,1) float32. Each
    token's index row holds K_top distinct key rows drawn uniformly from the
    keys it may see (all K, or [0, s] for a causal batch), in random order,
    -1 padded when it sees fewer than K_top keys -- the form of the indexer's
    top-k sets."""
    rng = np.random.default_rng(wl.seed if seed is None else seed)
    B, S, H, D, K = wl.B, wl.S, wl.H, wl.D, wl.K
    q = f32_to_bf16_bits(gaussian_f32(rng, B * S * H * D).reshape(B, S, H, D))
    kv = f32_to_bf16_bits(gaussian_f32(rng, B * K * D).reshape(B, K, D))
    sinks = gaussian_f32(rng, H)
    idx = np.full((B, S, wl.K_top), -1, np.int32)
    for b in range(B):
        for s in range(S):
            n = min(K, s + 1) if wl.causal else K
            m = min(n, wl.K_top)
            if n <= 4 * wl.K_top:
                pick = rng.permutation(n)[:m]
            else:                   # sample without a full permutation of n
                pick = np.unique(rng.integers(0, n, size=2 * m))
                while pick.size < m:
                    pick = np.unique(np.concatenate([pick, rng.integers(0, n, size=m)]))
                pick = rng.permutation(pick)[:m]
            idx[b, s, :m] = pick
    return dict(q=q, kv=kv, sinks=sinks, idx=idx)


# ---- the indexer's front end: projections, LayerNorm, RoPE -------------------

@dataclasses.dataclass(frozen=True)
class PrepareWorkload:
    """One synthetic front-end problem (DeepSeek-V3.2 Sparse Indexer Kernel API
    Reference, Parameters). The pages fix head_dim = 128 and the 64-head
    configuration; hidden, q_lora_rank and rope_dim take the published
    DeepSeek-V3.2 sizes (7168, 1536, 64) unless stated."""
    name: str
    T: int
    H: int = 64
    hidden: int = 7168
    q_lora_rank: int = 1536
    rope_dim: int = 64
    D: int = 128
    seed: int = 0

    @property
    def w_scale(self) -> float:
        return float(self.H * self.D) ** -0.5


PREPARE_WORKLOADS = {
    "prepare_decode": PrepareWorkload("prepare_decode", T=16),
    "prepare_prefill": PrepareWorkload("prepare_prefill", T=8192),
}


def generate_prepare(wl: PrepareWorkload, seed: Optional[int] = None,
                     positions: Optional[np.ndarray] = None) -> dict:
    """Draw a front-end problem (host arrays; bf16 as bit patterns).

    ``numpy.random.default_rng(seed)``, draws in the order x, qr, wq_b, wk,
    weights_proj, gain, bias. Activations ~ N(0,1); weights ~ N(0,1) /
    sqrt(in_features) (so projections are ~ N(0,1)); LayerNorm gain ~
    1 + N(0,1)/10, bias ~ N(0,1)/10; cos/sin of the angles pos * 10000^(-2i /
    rope_dim) at each token's position (positions t when not given)."""
    rng = np.random.default_rng(wl.seed if seed is None else seed)
    T, H, D, hid, ql = wl.T, wl.H, wl.D, wl.hidden, wl.q_lora_rank
    x = f32_to_bf16_bits(gaussian_f32(rng, T * hid).reshape(T, hid))
    qr = f32_to_bf16_bits(gaussian_f32(rng, T * ql).reshape(T, ql))
    wq_b = f32_to_bf16_bits((gaussian_f32(rng, H * D * ql) / np.float32(np.sqrt(ql)))
                            .reshape(H * D, ql))
    wk = f32_to_bf16_bits((gaussian_f32(rng, D * hid) / np.float32(np.sqrt(hid))).reshape(D, hid))
    wp = f32_to_bf16_bits((gaussian_f32(rng, H * hid) / np.float32(np.sqrt(hid))).reshape(H, hid))
    gain = (1.0 + gaussian_f32(rng, D) / 10).astype(np.float32)
    bias = (gaussian_f32(rng, D) / 10).astype(np.float32)
    pos = np.arange(T, dtype=np.int32) if positions is None else np.asarray(positions, np.int32)
    half = wl.rope_dim // 2
    theta = 10000.0 ** (-2.0 * np.arange(half) / max(wl.rope_dim, 1))
    ang = pos[:, None].astype(np.float64) * theta[None, :]
    return dict(x=x, qr=qr, wq_b=wq_b, wk=wk, wp=wp, gain=gain, bias=bias,
                cos=np.cos(ang).astype(np.float32), sin=np.sin(ang).astype(np.float32),
                positions=pos)
