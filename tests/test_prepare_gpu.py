"""The front end (dsa_indexer_prepare) vs the fp64 oracle
(oracle/front_end.py), through the C ABI (GPU only).

Tolerance, from the kernel's arithmetic: bf16 inputs, products exact in
fp32, sums accumulated in fp32 over K terms (relative error ~ K * 2^-24 in
the worst case, far smaller in practice), RoPE and LayerNorm in fp32, and q
and k rounded to bf16 at the end (<= 2^-9 relative). q and k must lie within
2^-8 * |oracle| + 2^-12 * max |oracle row|; the fp32 head weights within
1e-4 * max |oracle row|.
"""
import numpy as np
import pytest
import torch

import dsa_synth as syn
from oracle.front_end import bf16_to_f64, front_end

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def dsa():
    assert torch.cuda.is_available(), "GPU tests need a CUDA device"
    import sparse_attention_lightning_tcgen05_b200 as m
    return m


def dev(a):
    a = np.ascontiguousarray(a)
    if a.dtype == np.uint16:
        a = a.view(np.int16)
    return torch.from_numpy(a).cuda()


def run(m, wl, inp, *, S=None, k_seq_stride=0, positions=None, eps=1e-6):
    T, H, D = wl.T, wl.H, wl.D
    S = T if S is None else S
    desc = m.make_prepare_desc(T, H, wl.hidden, wl.q_lora_rank, wl.rope_dim, k_norm_eps=eps,
                               w_scale=wl.w_scale, S=S, k_seq_stride=k_seq_stride)
    q = torch.zeros((T, H, D), dtype=torch.int16, device="cuda")
    w = torch.zeros((T, H), dtype=torch.float32, device="cuda")
    ncache = (T if k_seq_stride else 1) * S
    cache = torch.full((ncache, D), 0x7F7F, dtype=torch.int16, device="cuda")  # a sentinel
    nbytes = m.dsa_indexer_prepare_workspace_size(desc)
    ws = torch.zeros(nbytes, dtype=torch.uint8, device="cuda")
    pos = None if positions is None else dev(np.asarray(positions, np.int32))
    t = {k: dev(inp[k]) for k in ("x", "qr", "wq_b", "wk", "wp", "gain", "bias", "cos", "sin")}
    m.dsa_indexer_prepare(desc, t["x"], t["qr"], t["wq_b"], t["wk"], t["wp"], t["gain"],
                          t["bias"], t["cos"], t["sin"], pos, q, w, cache, ws, nbytes,
                          torch.cuda.current_stream().cuda_stream)
    assert m.dsa_indexer_get_error(ws) == m.DSA_OK
    return (bf16_to_f64(q.cpu().numpy().view(np.uint16)), w.cpu().numpy().astype(np.float64),
            cache.cpu().numpy().view(np.uint16), nbytes)


def oracle(wl, inp, eps=1e-6):
    return front_end(inp["x"], inp["qr"], inp["wq_b"], inp["wk"], inp["wp"], inp["gain"],
                     inp["bias"], inp["cos"], inp["sin"], H=wl.H, D=wl.D,
                     rope_dim=wl.rope_dim, eps=eps, w_scale=wl.w_scale)


def close_bf16(g, o):
    rowmax = np.abs(o).max(axis=-1, keepdims=True)
    bound = 2.0 ** -8 * np.abs(o) + 2.0 ** -12 * rowmax
    assert np.all(np.abs(g - o) <= bound), float((np.abs(g - o) / bound).max())


def close_w(g, o):
    rowmax = np.abs(o).max(axis=-1, keepdims=True)
    assert np.all(np.abs(g - o) <= 1e-4 * rowmax)


def check(wl, inp, q, w, cache, key_rows, eps=1e-6):
    oq, ok, ow = oracle(wl, inp, eps)
    close_bf16(q, oq)
    close_w(w, ow)
    for t, row in key_rows:
        if row is None:
            continue
        close_bf16(bf16_to_f64(cache[row]), ok[t])


def test_prepare_decode_split_k(dsa):
    """The decode batch's front end (16 tokens, hidden 7168, q_lora_rank 1536):
    both projections split their K range over the SMs; each token's key goes
    to its own cache at its position."""
    wl = syn.PREPARE_WORKLOADS["prepare_decode"]
    S = 4096
    pos = np.random.default_rng(1).integers(0, S, wl.T).astype(np.int32)
    inp = syn.generate_prepare(wl, positions=pos)
    q, w, cache, nbytes = run(dsa, wl, inp, S=S, k_seq_stride=S * 128, positions=pos)
    assert nbytes > 256
    check(wl, inp, q, w, cache, [(t, t * S + int(pos[t])) for t in range(wl.T)])
    untouched = np.ones(wl.T * S, bool)
    untouched[[t * S + int(pos[t]) for t in range(wl.T)]] = False
    assert np.all(cache[untouched] == 0x7F7F)


@pytest.mark.parametrize("H,rope_dim", [(64, 64), (16, 0), (32, 128), (128, 64)])
def test_prepare_short_contractions(dsa, H, rope_dim):
    """hidden = q_lora_rank = 256, 300 tokens (three token tiles, a ragged
    last one), keys packed at slot t (prefill): the query GEMM runs unsplit
    with its epilogue fused, the key/weight GEMM splits its four K steps."""
    wl = syn.PrepareWorkload("p", T=300, H=H, hidden=256, q_lora_rank=256, rope_dim=rope_dim,
                             seed=H + rope_dim)
    inp = syn.generate_prepare(wl)
    q, w, cache, nbytes = run(dsa, wl, inp)
    assert nbytes > 256
    check(wl, inp, q, w, cache, [(t, t) for t in range(wl.T)])


@pytest.mark.parametrize("H,rope_dim", [(64, 64), (16, 0)])
def test_prepare_fused_epilogues(dsa, H, rope_dim):
    """19000 tokens (149 token tiles) with K = 256: both GEMMs fill the SMs
    unsplit, so the LayerNorm / RoPE / cache-write and the head-weight
    epilogues run inside the GEMM kernel. Sampled rows."""
    wl = syn.PrepareWorkload("pf", T=19000, H=H, hidden=256, q_lora_rank=256,
                             rope_dim=rope_dim, seed=7 + H)
    inp = syn.generate_prepare(wl)
    q, w, cache, nbytes = run(dsa, wl, inp)
    assert nbytes == 256
    rows = [0, 1, 127, 128, 9000, 18943, 18944, 18999]
    sub = {k: (v[rows] if k in ("x", "qr", "cos", "sin", "positions") else v)
           for k, v in inp.items()}
    oq, ok, ow = oracle(wl, sub)
    close_bf16(q[rows], oq)
    close_w(w[rows], ow)
    for i, t in enumerate(rows):
        close_bf16(bf16_to_f64(cache[t]), ok[i])


def test_prepare_prefill_sizes(dsa):
    """2048 tokens with the full projection sizes: the query GEMM has enough
    tiles (16 x 64) to run unsplit, the key/weight GEMM splits its K range."""
    wl = syn.PrepareWorkload("pp", T=2048, seed=3)
    inp = syn.generate_prepare(wl)
    q, w, cache, _ = run(dsa, wl, inp)
    rows = [0, 1, 127, 128, 1000, 2047]
    sub = {k: (v[rows] if k in ("x", "qr", "cos", "sin", "positions") else v)
           for k, v in inp.items()}
    oq, ok, ow = oracle(wl, sub)
    close_bf16(q[rows], oq)
    close_w(w[rows], ow)
    for i, t in enumerate(rows):
        close_bf16(bf16_to_f64(cache[t]), ok[i])


def test_prepare_positions_outside_the_cache_write_nothing(dsa):
    """A position < 0 or >= S writes no key; q and w are still computed."""
    wl = syn.PrepareWorkload("po", T=6, hidden=256, q_lora_rank=256, seed=4)
    S = 100
    pos = np.array([0, 99, -1, 100, 50, 7], np.int32)
    inp = syn.generate_prepare(wl, positions=np.clip(pos, 0, None))
    q, w, cache, _ = run(dsa, wl, inp, S=S, k_seq_stride=S * 128, positions=pos)
    rows = [(t, t * S + int(pos[t]) if 0 <= pos[t] < S else None) for t in range(wl.T)]
    check(wl, inp, q, w, cache, rows)
    written = {r for _, r in rows if r is not None}
    untouched = np.array([i not in written for i in range(wl.T * S)])
    assert np.all(cache[untouched] == 0x7F7F)
