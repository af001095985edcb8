"""Pins of the fp64 oracle against things other than itself (CPU only).

Each test fixes the oracle to something the pages or the mathematics decide:
hand-worked golden rows, brute-force sorts, a BLAS matmul, linear identities
that the ReLU and the head weights must satisfy, the Hadamard identity, exact
integer arithmetic and the library's e4m3 decoding table.
"""
import dataclasses
import json
import os

import numpy as np
import pytest
import torch

import dsa_synth as syn
import oracle

MB = float.fromhex("-0x1.FEp127")   # lowest finite bf16


def _sparse_vecs(rows, D):
    out = np.zeros((len(rows), D), np.float32)
    for i, r in enumerate(rows):
        for d, v in r.items():
            out[i, int(d)] = v
    return out


def _problem_from_golden(g):
    D, H, T = g["D"], g["H"], g["T"]
    q = np.stack([_sparse_vecs(heads, D) for heads in g["q"]])      # [T,H,D]
    k = _sparse_vecs(g["k"], D)
    w = np.asarray(g["w"], np.float32).reshape(T, H)
    if g["mode"] == "positions":
        wl = syn.Workload("golden", syn.MODE_POSITIONS, T=T, H=H, D=D,
                          index_topk=1, S=g["S"], shared_cache=True)
        inputs = dict(positions=np.asarray(g["positions"], np.int32),
                      cu_seqlens=None)
    elif g["mode"] == "compressed":
        wl = syn.Workload("golden", syn.MODE_COMPRESSED, T=T, H=H, D=D,
                          index_topk=1, S=g["S"],
                          compress_ratio=g["compress_ratio"],
                          query_start=g["query_start"])
        inputs = dict(positions=None, cu_seqlens=None)
    else:
        cu = g["cu_seqlens"]
        wl = syn.Workload("golden", syn.MODE_CAUSAL, T=T, H=H, D=D,
                          index_topk=1,
                          seqlens=tuple(np.diff(cu).tolist()))
        inputs = dict(positions=None, cu_seqlens=np.asarray(cu, np.int32))
    inputs.update(q=syn.f32_to_bf16_bits(q), q_scale=None,
                  k=syn.f32_to_bf16_bits(k), k_scale=None, w=w)
    return wl, inputs


@pytest.mark.parametrize("name", ["decode_hand.json", "causal_hand.json",
                                  "compressed_hand.json"])
def test_golden_hand_worked(golden_dir, name):
    g = json.load(open(os.path.join(golden_dir, name)))
    wl, inputs = _problem_from_golden(g)
    P = oracle.Problem(wl, inputs)
    rows = list(range(wl.T))
    got = P.scores(rows)
    for t, exp in enumerate(g["expected_scores"]):
        exp = np.array([MB if v == "MASK" else v for v in exp], np.float64)
        np.testing.assert_array_equal(got[t], exp)
    for k, exp_sets in g["topk"].items():
        tk = P.topk(rows, got, int(k))
        for t, exp in enumerate(exp_sets):
            assert sorted(tk[t].tolist()) == sorted(exp), (k, t)


def test_mask_bound_is_lowest_finite_bf16():
    mb = oracle.mask_bound()
    assert mb == MB
    # 0xFF7F is the lowest finite bf16 pattern; the next one down is -inf
    assert oracle.bf16_value(0xFF7F) == mb
    assert np.isinf(oracle.bf16_value(0xFF80))
    assert np.float32(mb) == mb          # exact in fp32


def _small_decode(T=3, H=4, S=200, seed=1, shared=False, dtype=syn.DTYPE_BF16,
                  pos_lo=0, pos_hi=200, kind="gauss"):
    wl = syn.Workload("t", syn.MODE_POSITIONS, T=T, H=H, D=128, index_topk=16,
                      S=S, shared_cache=shared, pos_lo=pos_lo, pos_hi=pos_hi,
                      w_scale=0.5, seed=seed, dtype=dtype)
    return wl, syn.generate(wl, value_kind=kind)


def _small_causal(seqlens=(5, 37, 130), H=3, seed=2, dtype=syn.DTYPE_BF16,
                  kind="gauss"):
    wl = syn.Workload("c", syn.MODE_CAUSAL, T=sum(seqlens), H=H, D=128,
                      index_topk=16, seqlens=tuple(seqlens), w_scale=0.5,
                      seed=seed, dtype=dtype)
    return wl, syn.generate(wl, value_kind=kind)


def _bf16_f64(bits):
    return (np.asarray(bits, np.uint32) << 16).view(np.float32).astype(np.float64)


def _np_dot_rows(wl, inputs, P, t):
    """q[t] . k[s] for the slots of row t, by a numpy (BLAS) matmul."""
    first, L, last, _ = P.row_info(t)
    q = _bf16_f64(inputs["q"][t])                 # [H, D]
    k = _bf16_f64(inputs["k"][first:first + L])   # [L, D]
    return q @ k.T, last                          # [H, L]


@pytest.mark.parametrize("maker", [_small_decode, _small_causal])
def test_h1_w1_reduces_to_relu_matmul(maker):
    wl, inputs = maker(H=1)
    inputs["w"] = np.ones_like(inputs["w"])
    P = oracle.Problem(wl, inputs)
    rows = list(range(wl.T))
    got = P.scores(rows)
    for t in rows:
        x, last = _np_dot_rows(wl, inputs, P, t)
        exp = np.maximum(x[0], 0.0)
        exp[last + 1:] = MB
        np.testing.assert_allclose(got[t], exp, rtol=1e-12, atol=1e-12)


@pytest.mark.parametrize("maker", [_small_decode, _small_causal])
def test_relu_split_identity(maker):
    """I(q) - I(-q) = sum_h w_h (q_h . k): relu(x) - relu(-x) = x.

    Negating bf16 is exact (sign bit). Catches a missing/misplaced ReLU, an
    abs() in its place, or w applied inside the ReLU."""
    wl, inputs = maker()
    neg = dict(inputs)
    neg["q"] = inputs["q"] ^ np.uint16(0x8000)
    Pp, Pn = oracle.Problem(wl, inputs), oracle.Problem(wl, neg)
    rows = list(range(wl.T))
    ip, ineg = Pp.scores(rows), Pn.scores(rows)
    for t in rows:
        x, last = _np_dot_rows(wl, inputs, Pp, t)
        lin = inputs["w"][t].astype(np.float64) @ x
        n = last + 1
        scale = np.abs(lin[:n]).max() + 1e-30
        np.testing.assert_allclose((ip[t] - ineg[t])[:n], lin[:n],
                                   rtol=0, atol=1e-12 * scale)
        assert np.all(ip[t][n:] == MB) and np.all(ineg[t][n:] == MB)


def test_head_permutation_invariance():
    wl, inputs = _small_decode(H=8)
    perm = np.random.default_rng(5).permutation(8)
    p2 = dict(inputs, q=inputs["q"][:, perm, :].copy(),
              w=inputs["w"][:, perm].copy())
    rows = list(range(wl.T))
    a = oracle.Problem(wl, inputs).scores(rows)
    b = oracle.Problem(wl, p2).scores(rows)
    for x, y in zip(a, b):
        np.testing.assert_allclose(x, y, rtol=1e-12, atol=0)


def test_additivity_in_w():
    """I(w1 + w2) = I(w1) + I(w2), with w1, w2 and w1+w2 exact in fp32."""
    wl, inputs = _small_causal()
    rng = np.random.default_rng(9)
    w1 = (rng.integers(-8, 9, inputs["w"].shape) / 8).astype(np.float32)
    w2 = (rng.integers(-8, 9, inputs["w"].shape) / 4).astype(np.float32)
    rows = list(range(wl.T))
    s = [oracle.Problem(wl, dict(inputs, w=w)).scores(rows)
         for w in (w1, w2, (w1 + w2).astype(np.float32))]
    for t in rows:
        P = oracle.Problem(wl, inputs)
        n = P.row_info(t)[2] + 1
        ref = s[0][t][:n] + s[1][t][:n]
        np.testing.assert_allclose(s[2][t][:n], ref, rtol=0,
                                   atol=1e-12 * (np.abs(ref).max() + 1e-30))


def test_positive_homogeneity_in_q():
    """I(2q) = 2 I(q) exactly (scaling a bf16 by 2 is exact)."""
    wl, inputs = _small_decode()
    qf = _bf16_f64(inputs["q"]).astype(np.float32)
    q2 = syn.f32_to_bf16_bits(qf * np.float32(2.0))
    rows = list(range(wl.T))
    a = oracle.Problem(wl, inputs).scores(rows)
    b = oracle.Problem(wl, dict(inputs, q=q2)).scores(rows)
    for t, (x, y) in enumerate(zip(a, b)):
        n = inputs["positions"][t] + 1
        np.testing.assert_array_equal(y[:n], 2.0 * x[:n])


def _sylvester(n):
    h = np.array([[1.0]])
    while h.shape[0] < n:
        h = np.block([[h, h], [h, -h]])
    return h


def test_hadamard_identity():
    """(q H)(k H)^T = q H H^T k^T = 128 q k^T for the unnormalised Sylvester H
    (Sparse Attention Indexer MX BF16Score Kernel API Reference, Notes: the
    rotation is a no-op for the score). With sparse {-1,0,1} inputs, q H has
    small integer entries, so both sides are exact in bf16 and I_rot = 128 I.
    Catches a transposed or mis-indexed operand in the contraction."""
    rng = np.random.default_rng(3)
    T, H, D, S = 2, 3, 128, 40
    Hm = _sylvester(D)

    def sparse(n):
        x = np.zeros((n, D))
        for r in range(n):
            idx = rng.choice(D, 6, replace=False)
            x[r, idx] = rng.choice([-1.0, 1.0], 6)
        return x
    qf, kf = sparse(T * H), sparse(T * S)
    wl = syn.Workload("h", syn.MODE_POSITIONS, T=T, H=H, D=D, index_topk=4,
                      S=S)
    base = dict(positions=np.array([S - 1, 17], np.int32), cu_seqlens=None,
                q_scale=None, k_scale=None,
                w=rng.normal(size=(T, H)).astype(np.float32))
    enc = lambda a: syn.f32_to_bf16_bits(a.astype(np.float32))
    assert np.abs(qf @ Hm).max() <= 6 and np.abs(kf @ Hm).max() <= 6
    plain = oracle.Problem(wl, dict(base, q=enc(qf).reshape(T, H, D),
                                    k=enc(kf))).scores(range(T))
    rot = oracle.Problem(wl, dict(base, q=enc(qf @ Hm).reshape(T, H, D),
                                  k=enc(kf @ Hm))).scores(range(T))
    for t in range(T):
        n = base["positions"][t] + 1
        np.testing.assert_array_equal(rot[t][:n], 128.0 * plain[t][:n])
        assert np.all(rot[t][n:] == MB)


def _brute_topk(row, last_valid, k):
    n = min(last_valid + 1, len(row))
    order = sorted(range(max(n, 0)), key=lambda s: (-row[s], s))
    sel = order[:k]
    return sel + [-1] * (k - len(sel))


@pytest.mark.parametrize("maker", [_small_decode, _small_causal])
def test_topk_brute_force_all_k(maker):
    wl, inputs = maker(H=2)
    P = oracle.Problem(wl, inputs)
    rows = list(range(min(wl.T, 8))) + [wl.T - 1]
    sc = P.scores(rows)
    for k in (1, 2, 7, 64, 199, 200, 257):
        tk = P.topk(rows, sc, k)
        for i, t in enumerate(rows):
            last = P.row_info(t)[2]
            assert tk[i].tolist() == _brute_topk(sc[i], last, k) or \
                sorted(tk[i].tolist()) == sorted(_brute_topk(sc[i], last, k))


def test_topk_set_properties_with_ties():
    """Rows full of exact ties (integer inputs): size, distinctness, validity,
    the -1 count, the order property and lowest-index tie-breaking."""
    wl, inputs = _small_causal(seqlens=(300,), H=2, kind="int")
    P = oracle.Problem(wl, inputs)
    rows = [0, 1, 63, 64, 150, 299]
    sc = P.scores(rows)
    for k in (1, 64, 128):
        tk = P.topk(rows, sc, k)
        for i, t in enumerate(rows):
            n = P.row_info(t)[2] + 1
            sel = [s for s in tk[i] if s >= 0]
            assert len(sel) == min(k, n) and len(set(sel)) == len(sel)
            assert (tk[i] == -1).sum() == k - min(k, n)
            assert all(0 <= s < n for s in sel)
            rest = np.setdiff1d(np.arange(n), sel)
            if len(rest) and len(sel):
                kth = sc[i][sel].min()
                assert sc[i][rest].max() <= kth
                # ties at the threshold: every unselected tie has a larger index
                tied_out = rest[sc[i][rest] == kth]
                tied_in = [s for s in sel if sc[i][s] == kth]
                if len(tied_out):
                    assert max(tied_in) < tied_out.min()


def test_integer_inputs_are_exact():
    """Integer q, k in [-3,3] and w in {+-1, +-1/2}: every score is an exact
    small dyadic number; compare with exact integer arithmetic."""
    wl, inputs = _small_decode(H=5, kind="int")
    P = oracle.Problem(wl, inputs)
    rows = list(range(wl.T))
    got = P.scores(rows)
    for t in rows:
        first, L, last, _ = P.row_info(t)
        q = _bf16_f64(inputs["q"][t]).astype(np.int64)
        k = _bf16_f64(inputs["k"][first:first + L]).astype(np.int64)
        x = q @ k.T                                  # exact int64
        w2 = (inputs["w"][t] * 2).astype(np.int64)   # exact: w in {+-1, +-1/2}
        exp2 = w2 @ np.maximum(x, 0)                 # 2 * I, exact int64
        np.testing.assert_array_equal(got[t][:last + 1] * 2,
                                      exp2[:last + 1].astype(np.float64))


def test_positions_edges():
    """pos = 0: one valid slot; pos >= S-1: the whole row is valid."""
    wl, inputs = _small_decode(T=3, S=64)
    inputs["positions"] = np.array([0, 63, 1000], np.int32)
    P = oracle.Problem(wl, inputs)
    sc = P.scores([0, 1, 2])
    assert sc[0][0] != MB and np.all(sc[0][1:] == MB)
    assert np.all(sc[1] != MB) and np.all(sc[2] != MB)
    tk = P.topk([0, 1, 2], sc, 4)
    assert tk[0].tolist() == [0, -1, -1, -1]


def test_shared_cache_rows_read_the_same_keys():
    """k_seq_stride = 0: every token reads the one cache; equal queries give
    equal rows up to their own positions."""
    wl, inputs = _small_decode(T=2, S=50, shared=True)
    inputs["q"][1] = inputs["q"][0]
    inputs["w"][1] = inputs["w"][0]
    inputs["positions"] = np.array([49, 20], np.int32)
    sc = oracle.Problem(wl, inputs).scores([0, 1])
    np.testing.assert_array_equal(sc[0][:21], sc[1][:21])


def _small_compressed(T=40, H=3, S=23, r=4, qs=5, seed=4, dtype=syn.DTYPE_BF16):
    wl = syn.Workload("c", syn.MODE_COMPRESSED, T=T, H=H, D=128, index_topk=8,
                      S=S, compress_ratio=r, query_start=qs, dtype=dtype,
                      w_scale=0.5, seed=seed)
    return wl, syn.generate(wl)


@pytest.mark.parametrize("r,qs", [(4, 0), (4, 5), (1, 0), (3, 17), (128, 100)])
def test_compressed_visibility_by_raw_tokens(r, qs):
    """A pooled slot is visible exactly when every raw token it pools sits at
    or before the query's absolute position: enumerated token by token."""
    wl, inputs = _small_compressed(T=50, S=30, r=r, qs=qs)
    P = oracle.Problem(wl, inputs)
    sc = P.scores(list(range(wl.T)))
    for t in range(wl.T):
        p = qs + t
        vis = np.array([all(x <= p for x in range(j * r, (j + 1) * r))
                        for j in range(wl.S)])
        assert np.array_equal(sc[t] != MB, vis), (t, p)
        first, L, last, off = P.row_info(t)
        assert first == 0 and L == wl.S and off == t * wl.S
        assert min(last, wl.S - 1) == int(vis.sum()) - 1   # unclamped, like a position


@pytest.mark.parametrize("dtype", [syn.DTYPE_BF16, syn.DTYPE_FP8])
def test_compressed_equals_shared_cache_positions(dtype):
    """With every token reading the one pooled cache, the compressed rule is
    the positions rule with position = the last fully pooled slot; rows that
    see no slot are all at the mask bound and select nothing."""
    wl, inputs = _small_compressed(T=37, S=19, r=4, qs=2, dtype=dtype)
    rows = list(range(wl.T))
    P = oracle.Problem(wl, inputs)
    sc = P.scores(rows)
    last = np.array([(wl.query_start + t + 1) // wl.compress_ratio - 1
                     for t in rows])
    wp = syn.Workload("p", syn.MODE_POSITIONS, T=wl.T, H=wl.H, D=wl.D,
                      index_topk=8, S=wl.S, shared_cache=True, dtype=dtype)
    ip = dict(inputs, positions=np.maximum(last, 0).astype(np.int32),
              cu_seqlens=None)
    sp = oracle.Problem(wp, ip).scores(rows)
    for t in rows:
        if last[t] < 0:
            assert np.all(sc[t] == MB)
        else:
            np.testing.assert_array_equal(sc[t], sp[t])
    for k in (1, 5, 19, 24):
        tk = P.topk(rows, sc, k)
        for t in rows:
            n = max(0, min(k, int(last[t]) + 1))
            got = tk[t].tolist()
            assert got[n:] == [-1] * (k - n)
            assert sorted(got[:n]) == sorted(_brute_topk(sc[t], int(last[t]), k)[:n])


def _small_paged(T=6, H=4, S=300, page=64, seed=7, dtype=syn.DTYPE_BF16):
    wl = syn.Workload("pg", syn.MODE_POSITIONS, T=T, H=H, D=128, index_topk=16,
                      S=S, pos_lo=0, pos_hi=S, page_size=page, dtype=dtype,
                      w_scale=0.5, seed=seed)
    return wl, syn.generate(wl)


def _gather_pages(wl, inputs, key):
    """Each token's cache as one dense [S, ...] array, pages taken in block-table
    order (numpy fancy indexing, no oracle code)."""
    pool = inputs[key].reshape(wl.num_pages, wl.page_size, -1)
    return np.concatenate([pool[inputs["block_table"][t]].reshape(-1, pool.shape[-1])[:wl.S]
                           for t in range(wl.T)])


@pytest.mark.parametrize("dtype,page", [(syn.DTYPE_BF16, 64), (syn.DTYPE_BF16, 16),
                                        (syn.DTYPE_BF16, 128), (syn.DTYPE_FP8, 32)])
def test_paged_cache_equals_gathered_dense_cache(dtype, page):
    """A paged cache scores like the dense per-token cache its block table
    describes (the pages gathered in numpy)."""
    wl, inputs = _small_paged(page=page, dtype=dtype, S=333)
    rows = list(range(wl.T))
    P = oracle.Problem(wl, inputs)
    sp = P.scores(rows)
    wd = dataclasses.replace(wl, page_size=0)
    dense = dict(inputs, k=_gather_pages(wl, inputs, "k"), block_table=None,
                 k_scale=None if inputs["k_scale"] is None else _gather_pages(wl, inputs, "k_scale"))
    Pd = oracle.Problem(wd, dense)
    sd = Pd.scores(rows)
    for t in rows:
        np.testing.assert_array_equal(sp[t], sd[t])
    for k in (1, 16, 400):
        assert [sorted(x) for x in P.topk(rows, sp, k).tolist()] == \
               [sorted(x) for x in Pd.topk(rows, sd, k).tolist()]


def test_paged_cache_page_permutation_invariance():
    """Moving the pages within the pool, and the block table with them,
    changes nothing."""
    wl, inputs = _small_paged(page=32)
    rows = list(range(wl.T))
    base = oracle.Problem(wl, inputs).scores(rows)
    perm = np.random.default_rng(5).permutation(wl.num_pages)     # new home of page i
    pool = inputs["k"].reshape(wl.num_pages, wl.page_size, -1)
    moved = np.empty_like(pool)
    moved[perm] = pool
    moved_inputs = dict(inputs, k=moved.reshape(inputs["k"].shape),
                        block_table=perm[inputs["block_table"]].astype(np.int32))
    got = oracle.Problem(wl, moved_inputs).scores(rows)
    for t in rows:
        np.testing.assert_array_equal(got[t], base[t])


def test_paged_cache_reads_only_valid_slots():
    """Pages (and rows of a token's last page) past its position may hold
    anything: NaN there changes no score."""
    wl, inputs = _small_paged(page=16, S=200)
    rows = list(range(wl.T))
    base = oracle.Problem(wl, inputs).scores(rows)
    k = inputs["k"].copy().reshape(wl.num_pages, wl.page_size, -1)
    for t in rows:
        pos = int(inputs["positions"][t])
        for lp, page in enumerate(inputs["block_table"][t]):
            for r in range(wl.page_size):
                if lp * wl.page_size + r > pos:
                    k[page, r] = 0x7FC0                         # a bf16 NaN
    got = oracle.Problem(wl, dict(inputs, k=k.reshape(inputs["k"].shape))).scores(rows)
    for t in rows:
        np.testing.assert_array_equal(got[t], base[t])


def test_causal_layout_tiles_packed_buffer():
    wl, inputs = _small_causal(seqlens=(1, 7, 64, 3))
    P = oracle.Problem(wl, inputs)
    cover = np.zeros(sum(L * L for L in wl.seqlens), np.int32)
    for t in range(wl.T):
        first, L, last, off = P.row_info(t)
        cover[off:off + L] += 1
        assert 0 <= last < L
    assert np.all(cover == 1)


# ---- fp8 e4m3 + block-32 e8m0 (the MX storage format) -----------------------

def test_e4m3_table_matches_torch():
    codes = torch.arange(256, dtype=torch.uint8)
    ref = codes.view(torch.float8_e4m3fn).to(torch.float64).numpy()
    for c in range(256):
        got = oracle.e4m3_value(c)
        if np.isnan(ref[c]):
            assert np.isnan(got), c
        else:
            assert got == ref[c], (c, got, ref[c])


def test_e8m0_table_matches_torch():
    codes = torch.arange(255, dtype=torch.uint8)
    ref = codes.view(torch.float8_e8m0fnu).to(torch.float64).numpy()
    for c in range(255):
        assert oracle.e8m0_value(c) == ref[c], c
    assert np.isnan(oracle.e8m0_value(255))


def _torch_mx_decode(data, scale):
    """Reference decode by torch's float8 types: value * scale per 32-block."""
    v = torch.from_numpy(np.ascontiguousarray(data)).view(
        torch.float8_e4m3fn).to(torch.float64)
    s = torch.from_numpy(np.ascontiguousarray(scale)).view(
        torch.float8_e8m0fnu).to(torch.float64)
    return (v * s.repeat_interleave(32, dim=-1)).numpy()


def test_fp8_scores_match_torch_decode_matmul():
    """MX path: the oracle's scores equal a numpy matmul over torch-decoded
    q and k (pins the per-block scale indexing along D and per slot)."""
    wl, inputs = _small_decode(T=3, H=4, S=96, dtype=syn.DTYPE_FP8)
    P = oracle.Problem(wl, inputs)
    rows = [0, 1, 2]
    got = P.scores(rows)
    q = _torch_mx_decode(inputs["q"], inputs["q_scale"])      # [T,H,D]
    k = _torch_mx_decode(inputs["k"], inputs["k_scale"])      # [slots,D]
    for t in rows:
        first, L, last, _ = P.row_info(t)
        x = q[t] @ k[first:first + L].T
        exp = inputs["w"][t].astype(np.float64) @ np.maximum(x, 0)
        exp[last + 1:] = MB
        np.testing.assert_allclose(got[t], exp, rtol=1e-12, atol=1e-12)


def test_fp8_integer_inputs_are_exact():
    """Integer values in [-3,3] survive MX quantisation exactly (scale 2^-7
    for a block whose amax is 3 or 2^-8 for 2; 1 -> 2^-8..), so fp8 scores of
    integer inputs equal the exact integer result."""
    wl, inputs = _small_decode(T=2, H=3, S=64, dtype=syn.DTYPE_FP8, kind="int")
    q = _torch_mx_decode(inputs["q"], inputs["q_scale"])
    k = _torch_mx_decode(inputs["k"], inputs["k_scale"])
    assert np.all(q == np.round(q)) and np.abs(q).max() <= 3
    P = oracle.Problem(wl, inputs)
    got = P.scores([0, 1])
    for t in (0, 1):
        first, L, last, _ = P.row_info(t)
        x = (q[t].astype(np.int64) @ k[first:first + L].astype(np.int64).T)
        exp2 = (inputs["w"][t] * 2).astype(np.int64) @ np.maximum(x, 0)
        np.testing.assert_array_equal(got[t][:last + 1] * 2,
                                      exp2[:last + 1].astype(np.float64))


# ---- the input generator's encoders (library cross-checks) ------------------

def test_generator_bf16_rounding_matches_torch():
    x = np.random.default_rng(0).standard_normal(1 << 16).astype(np.float32)
    x[:4] = [1.00390625, 1.01171875, -2.00781250, 3.0e38]    # ties and large
    ref = torch.from_numpy(x).to(torch.bfloat16).view(torch.uint16).numpy()
    np.testing.assert_array_equal(syn.f32_to_bf16_bits(x), ref)


def test_generator_mx_encoding_matches_torch_cast():
    """Each block's data equals torch's e4m3 cast of x * 2^-e, the scale byte
    is e + 127 with 448 * 2^(e-1) < amax <= 448 * 2^e, and the relative error
    of quantise -> dequantise is at most 2^-4 for normal-range elements."""
    x = np.random.default_rng(1).standard_normal((64, 128)).astype(np.float32)
    x[0, :32] *= 1e-3
    x[1, 32:64] = 0.0
    x[1, 32] = 448.0 * 2.0 ** -20
    data, scale = syn.f32_to_mx_e4m3(x)
    e = scale.astype(np.int64) - 127
    blocks = x.reshape(64, 4, 32).astype(np.float64)
    amax = np.abs(blocks).max(-1)
    assert np.all(amax <= 448.0 * 2.0 ** e)
    assert np.all(amax > 448.0 * 2.0 ** (e - 1))
    y = torch.from_numpy(np.ldexp(blocks, -e[..., None]).reshape(64, 128))
    ref = y.to(torch.float8_e4m3fn).view(torch.uint8).numpy()
    np.testing.assert_array_equal(data, ref)
    back = _torch_mx_decode(data, scale)
    big = np.abs(np.ldexp(blocks, -e[..., None])).reshape(64, 128) >= 2.0 ** -6
    rel = np.abs(back - x) / np.maximum(np.abs(x.astype(np.float64)), 1e-300)
    assert rel[big].max() <= 2.0 ** -4
