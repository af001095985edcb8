"""CUDA path vs the fp64 oracle, through the C ABI (GPU only)."""
import numpy as np
import pytest
import torch

import dsa_synth as syn
import oracle
from parity_util import TOL_BF16, check_scores, check_topk, gpu_rows

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def dsa():
    assert torch.cuda.is_available(), "GPU tests need a CUDA device"
    import sparse_attention_lightning_tcgen05_b200 as m
    from sparse_attention_lightning_tcgen05_b200.problem import DeviceProblem
    return m, DeviceProblem


def run_and_check(dsa, wl, inputs, rows=None, tol=TOL_BF16, exact=False):
    m, DeviceProblem = dsa
    dp = DeviceProblem.from_workload(wl, inputs)
    dp.forward()
    assert dp.device_status() == m.DSA_OK
    torch.cuda.synchronize()
    P = oracle.Problem(wl, inputs)
    rows = list(range(wl.T)) if rows is None else [int(r) for r in rows]
    orc = P.scores(rows)
    gpu = gpu_rows(P, dp.scores, rows)
    if exact:
        for t, g, o in zip(rows, gpu, orc):
            np.testing.assert_array_equal(g, o, err_msg=f"row {t}")
    worst = check_scores(P, rows, gpu, orc, tol)
    tk = dp.topk.cpu().numpy()[rows]
    check_topk(P, rows, tk, gpu, orc, wl.index_topk, tol)
    return worst


def decode_wl(T=4, H=4, S=1024, k=64, shared=False, pos=(64, 1024), seed=0):
    return syn.Workload("d", syn.MODE_POSITIONS, T=T, H=H, D=128, index_topk=k,
                        S=S, shared_cache=shared, pos_lo=pos[0], pos_hi=pos[1],
                        w_scale=1.0 / np.sqrt(H), seed=seed)


def causal_wl(seqlens, H=64, k=64, seed=0):
    return syn.Workload("c", syn.MODE_CAUSAL, T=int(sum(seqlens)), H=H, D=128,
                        index_topk=k, seqlens=tuple(seqlens),
                        w_scale=1.0 / np.sqrt(H), seed=seed)


def test_tiny_decode_full(dsa):
    wl = syn.WORKLOADS["tiny_decode"]
    run_and_check(dsa, wl, syn.generate(wl))


@pytest.mark.parametrize("H", [1, 4, 8, 16, 32, 64, 128])
def test_decode_heads(dsa, H):
    wl = decode_wl(T=3, H=H, S=700, k=100, pos=(0, 700), seed=H)
    run_and_check(dsa, wl, syn.generate(wl))


@pytest.mark.parametrize("H", [4, 64])
def test_decode_integer_inputs_bit_exact(dsa, H):
    wl = decode_wl(T=3, H=H, S=520, k=32, pos=(100, 520), seed=3)
    run_and_check(dsa, wl, syn.generate(wl, value_kind="int"), exact=True)


@pytest.mark.parametrize("H", [4, 64])
def test_causal_integer_inputs_bit_exact(dsa, H):
    wl = causal_wl((1, 130, 257), H=H, k=16, seed=4)
    run_and_check(dsa, wl, syn.generate(wl, value_kind="int"), exact=True)


def test_decode_position_edges(dsa):
    """pos = 0, pos = S-1, pos >= S, negative pos, S not a multiple of 128."""
    wl = decode_wl(T=6, H=64, S=333, k=40, seed=5)
    inputs = syn.generate(wl)
    inputs["positions"] = np.array([0, 332, 5000, -1, 127, 128], np.int32)
    run_and_check(dsa, wl, inputs)


def test_decode_many_tokens(dsa):
    """More than 32 query blocks (the positions schedule scans blocks 32 at a
    time) and pipeline items of two key tiles that end at token boundaries."""
    wl = decode_wl(T=100, H=64, S=1000, k=64, pos=(0, 1000), seed=40)
    run_and_check(dsa, wl, syn.generate(wl))


def test_decode_shared_cache(dsa):
    wl = decode_wl(T=11, H=64, S=900, k=50, shared=True, pos=(0, 900), seed=6)
    run_and_check(dsa, wl, syn.generate(wl))


def test_decode_shared_cache_generic_heads(dsa):
    wl = decode_wl(T=70, H=4, S=300, k=20, shared=True, pos=(0, 300), seed=7)
    run_and_check(dsa, wl, syn.generate(wl))


@pytest.mark.parametrize("H", [1, 4, 16, 32, 64, 128])
def test_causal_ragged_small(dsa, H):
    wl = causal_wl((1, 7, 127, 128, 129, 300, 1000), H=H, k=64, seed=H)
    run_and_check(dsa, wl, syn.generate(wl))


def test_k_larger_than_rows(dsa):
    wl = causal_wl((50, 3), H=64, k=2048, seed=8)
    run_and_check(dsa, wl, syn.generate(wl))


def test_topk_ties_integer_scores(dsa):
    """Many exact ties (H=1 integer inputs): the tie rule picks the lower
    slots, bit-exact."""
    wl = causal_wl((600,), H=1, k=100, seed=9)
    run_and_check(dsa, wl, syn.generate(wl, value_kind="int"), exact=True)


def test_decode_batch_full_size(dsa):
    wl = syn.WORKLOADS["decode_batch"]
    run_and_check(dsa, wl, syn.generate(wl))


def test_prefill_causal_full_size_sampled(dsa):
    wl = syn.WORKLOADS["prefill_causal"]
    rng = np.random.default_rng(11)
    rows = [0, 1, 127, 128, 2046, 2047, 2048, 4095, 8191] + \
        list(rng.integers(0, 8192, 12))
    run_and_check(dsa, wl, syn.generate(wl), rows=rows)


def test_ragged_prefill_full_size_sampled(dsa):
    wl = syn.WORKLOADS["ragged_prefill"]
    cu = wl.cu_seqlens()
    rng = np.random.default_rng(12)
    rows = []
    for i in range(len(wl.seqlens)):
        rows += [cu[i], cu[i] + 1, cu[i] + 2049, cu[i + 1] - 1]
    rows += list(rng.integers(0, wl.T, 8))
    run_and_check(dsa, wl, syn.generate(wl), rows=sorted(set(int(r) for r in rows)))


# ---- fp8 e4m3 + block-32 e8m0 (block-scaled MMA) -------------------------------

from parity_util import TOL_FP8  # noqa: E402


def fp8_decode_wl(T=3, H=64, S=700, k=50, shared=False, pos=(0, 700), seed=0):
    return syn.Workload("d8", syn.MODE_POSITIONS, T=T, H=H, D=128, index_topk=k,
                        S=S, shared_cache=shared, pos_lo=pos[0], pos_hi=pos[1],
                        dtype=syn.DTYPE_FP8, w_scale=1.0 / np.sqrt(H), seed=seed)


def fp8_causal_wl(seqlens, H=64, k=64, seed=0):
    return syn.Workload("c8", syn.MODE_CAUSAL, T=int(sum(seqlens)), H=H, D=128,
                        index_topk=k, seqlens=tuple(seqlens), dtype=syn.DTYPE_FP8,
                        w_scale=1.0 / np.sqrt(H), seed=seed)


@pytest.mark.parametrize("H", [4, 16, 64, 128])
def test_fp8_decode_heads(dsa, H):
    wl = fp8_decode_wl(T=3, H=H, S=700, k=100, seed=20 + H)
    run_and_check(dsa, wl, syn.generate(wl), tol=TOL_FP8)


@pytest.mark.parametrize("H", [4, 64])
def test_fp8_integer_inputs_bit_exact(dsa, H):
    wl = fp8_decode_wl(T=3, H=H, S=520, k=32, pos=(100, 520), seed=5)
    run_and_check(dsa, wl, syn.generate(wl, value_kind="int"), tol=TOL_FP8, exact=True)


@pytest.mark.parametrize("H", [4, 64, 128])
def test_fp8_causal_ragged(dsa, H):
    wl = fp8_causal_wl((1, 127, 129, 300, 1000), H=H, k=64, seed=30 + H)
    run_and_check(dsa, wl, syn.generate(wl), tol=TOL_FP8)


def test_fp8_causal_integer_bit_exact(dsa):
    wl = fp8_causal_wl((130, 257), H=64, k=16, seed=6)
    run_and_check(dsa, wl, syn.generate(wl, value_kind="int"), tol=TOL_FP8, exact=True)


def test_fp8_shared_cache(dsa):
    wl = fp8_decode_wl(T=9, H=64, S=900, k=50, shared=True, seed=7)
    run_and_check(dsa, wl, syn.generate(wl), tol=TOL_FP8)


def test_long_decode_fp8_full_size_sampled(dsa):
    wl = syn.WORKLOADS["long_decode_fp8"]
    rng = np.random.default_rng(13)
    rows = sorted(set([0, 1, 63] + list(rng.integers(0, wl.T, 5))))
    run_and_check(dsa, wl, syn.generate(wl), rows=rows, tol=TOL_FP8)


def test_fp8_decode_many_tokens(dsa):
    wl = fp8_decode_wl(T=70, H=64, S=1300, k=80, pos=(0, 1300), seed=41)
    run_and_check(dsa, wl, syn.generate(wl), tol=TOL_FP8)


# ---- compressed (C4) keys: one pooled cache, validity from the ratio --------

def c4_wl(T, H, S, k, r=4, qs=0, dtype=syn.DTYPE_BF16, seed=0):
    return syn.Workload("c4", syn.MODE_COMPRESSED, T=T, H=H, D=128, index_topk=k,
                        S=S, compress_ratio=r, query_start=qs, dtype=dtype,
                        w_scale=1.0 / np.sqrt(H), seed=seed)


@pytest.mark.parametrize("H", [4, 16, 64, 128])
def test_compressed_small(dsa, H):
    """Rows that see no pooled slot, a few, and all of them; S ragged."""
    wl = c4_wl(T=300, H=H, S=70, k=24, r=4, qs=0, seed=50 + H)
    run_and_check(dsa, wl, syn.generate(wl))


@pytest.mark.parametrize("H", [4, 64])
def test_compressed_integer_inputs_bit_exact(dsa, H):
    wl = c4_wl(T=200, H=H, S=140, k=32, r=3, qs=7, seed=51)
    run_and_check(dsa, wl, syn.generate(wl, value_kind="int"), exact=True)


def test_compressed_query_start_and_ratios(dsa):
    """A late chunk (query_start past the pooled cache for some rows: those
    rows are all valid) and a ratio of 1 (the causal rule on pooled keys)."""
    for r, qs, T, S in ((4, 1000, 90, 300), (1, 37, 50, 120), (128, 0, 300, 5)):
        wl = c4_wl(T=T, H=64, S=S, k=40, r=r, qs=qs, seed=52 + r)
        run_and_check(dsa, wl, syn.generate(wl))


def test_compressed_many_tokens_unstaged(dsa):
    """More tokens than the score kernel stages in shared memory: every row
    derives its last valid slot from the ratio on the fly."""
    wl = c4_wl(T=2600, H=64, S=700, k=64, r=4, qs=5, seed=53)
    rng = np.random.default_rng(14)
    rows = sorted(set([0, 1, 2, 3, 4, 2047, 2048, 2599] +
                      list(rng.integers(0, wl.T, 24))))
    run_and_check(dsa, wl, syn.generate(wl), rows=rows)


@pytest.mark.parametrize("H", [16, 64])
def test_fp8_compressed(dsa, H):
    wl = c4_wl(T=260, H=H, S=90, k=30, r=4, qs=3, dtype=syn.DTYPE_FP8, seed=54 + H)
    run_and_check(dsa, wl, syn.generate(wl), tol=TOL_FP8)


def test_c4_prefill_full_size_sampled(dsa):
    wl = syn.WORKLOADS["c4_prefill"]
    rng = np.random.default_rng(15)
    rows = sorted(set([0, 2, 3, 4, 511, 4095, 4096, 8190, 8191] +
                      list(rng.integers(0, wl.T, 12))))
    run_and_check(dsa, wl, syn.generate(wl), rows=rows)


# ---- top-k of short decode-style rows (the register path) -------------------

def test_decode_topk_ties_integer_scores(dsa):
    """H=1 integer inputs: many equal scores around the threshold; the set
    must be the oracle's, lower slots first among ties (bit-exact)."""
    wl = decode_wl(T=24, H=1, S=2000, k=300, shared=True, pos=(400, 2000), seed=60)
    run_and_check(dsa, wl, syn.generate(wl, value_kind="int"), exact=True)


def test_decode_topk_all_scores_equal(dsa):
    """Every score 0 (q = 0): the threshold's ties fill the whole set, which
    must be the lowest k slots of each row."""
    wl = decode_wl(T=6, H=64, S=3000, k=700, shared=True, pos=(800, 3000), seed=61)
    inputs = syn.generate(wl)
    inputs["q"] = np.zeros_like(inputs["q"])
    run_and_check(dsa, wl, inputs, exact=True)


@pytest.mark.parametrize("S", [33, 2048, 2049, 4096])
def test_decode_topk_row_lengths(dsa, S):
    """Rows at the register path's boundaries (one and two chunk rows, the
    largest rows it takes) and a misaligned row start (S odd)."""
    wl = decode_wl(T=5, H=16, S=S, k=min(32, S - 1), shared=True, pos=(0, S), seed=62)
    inputs = syn.generate(wl)
    inputs["positions"] = np.array([S - 1, S // 2, 31, 32, S + 5], np.int32)
    run_and_check(dsa, wl, inputs)


# ---- paged key caches (block tables) ------------------------------------------

def paged_wl(T, H, S, k, page, seed=0, dtype=syn.DTYPE_BF16):
    return syn.Workload("pg", syn.MODE_POSITIONS, T=T, H=H, D=128, index_topk=k, S=S,
                        pos_lo=0, pos_hi=S, page_size=page, dtype=dtype,
                        w_scale=1.0 / np.sqrt(H), seed=seed)


@pytest.mark.parametrize("page", [16, 32, 64, 128, 256])
def test_paged_decode(dsa, page):
    """Pages smaller than a key tile (several pages a tile), equal to it and
    larger; S not a multiple of the page."""
    wl = paged_wl(T=5, H=64, S=1000, k=64, page=page, seed=70 + page)
    run_and_check(dsa, wl, syn.generate(wl))


def test_paged_decode_integer_bit_exact(dsa):
    wl = paged_wl(T=4, H=64, S=700, k=40, page=32, seed=71)
    run_and_check(dsa, wl, syn.generate(wl, value_kind="int"), exact=True)


def test_paged_generic_heads(dsa):
    wl = paged_wl(T=6, H=4, S=900, k=50, page=64, seed=72)
    run_and_check(dsa, wl, syn.generate(wl))


def test_paged_unused_table_entries(dsa):
    """Block-table entries of pages past a token's position may be anything
    (-1, past the pool): the scores of the valid slots do not change."""
    wl = paged_wl(T=6, H=64, S=1200, k=64, page=64, seed=73)
    inputs = syn.generate(wl)
    inputs["positions"] = np.array([0, 63, 64, 500, 1199, 129], np.int32)
    bt = inputs["block_table"].copy()
    for t, pos in enumerate(inputs["positions"]):
        bt[t, pos // 64 + 1:] = np.where(np.arange(bt.shape[1] - pos // 64 - 1) % 2, -1, 1 << 30)
    inputs["block_table"] = bt
    run_and_check(dsa, wl, inputs)


def test_decode_batch_paged_full_size(dsa):
    wl = syn.WORKLOADS["decode_batch_paged"]
    run_and_check(dsa, wl, syn.generate(wl))


def test_causal_with_empty_sequences(dsa):
    """Zero-length sequences in a packed batch (cu_seqlens repeats a value):
    the schedule and the top-k's row lookup skip them."""
    wl = causal_wl((0, 5, 0, 130, 0, 257), H=64, k=64, seed=80)
    run_and_check(dsa, wl, syn.generate(wl))


def test_paged_single_large_page(dsa):
    """One page holds the whole cache (pages of 4096 slots, S = 3000)."""
    wl = paged_wl(T=3, H=64, S=3000, k=100, page=4096, seed=81)
    run_and_check(dsa, wl, syn.generate(wl))


# ---- paged fp8 caches: e4m3 pages and their e8m0 scale pages ------------------

@pytest.mark.parametrize("page", [16, 32, 64, 128, 256, 1024])
def test_paged_fp8_decode(dsa, page):
    """Pages smaller than a key tile (several data and scale boxes a tile),
    equal to it and larger; S not a multiple of the page."""
    wl = paged_wl(T=5, H=64, S=1000, k=64, page=page, seed=90 + page, dtype=syn.DTYPE_FP8)
    run_and_check(dsa, wl, syn.generate(wl), tol=TOL_FP8)


def test_paged_fp8_integer_bit_exact(dsa):
    wl = paged_wl(T=4, H=64, S=700, k=40, page=32, seed=91, dtype=syn.DTYPE_FP8)
    run_and_check(dsa, wl, syn.generate(wl, value_kind="int"), tol=TOL_FP8, exact=True)


def test_paged_fp8_generic_heads(dsa):
    wl = paged_wl(T=6, H=16, S=900, k=50, page=64, seed=92, dtype=syn.DTYPE_FP8)
    run_and_check(dsa, wl, syn.generate(wl), tol=TOL_FP8)


def test_paged_fp8_unused_table_entries(dsa):
    """Table entries past a token's position (-1, far past the pool) are
    never used for a score, in the data pool or the scale pool."""
    wl = paged_wl(T=6, H=64, S=1200, k=64, page=64, seed=93, dtype=syn.DTYPE_FP8)
    inputs = syn.generate(wl)
    inputs["positions"] = np.array([0, 63, 64, 500, 1199, 129], np.int32)
    bt = inputs["block_table"].copy()
    for t, pos in enumerate(inputs["positions"]):
        bt[t, pos // 64 + 1:] = np.where(np.arange(bt.shape[1] - pos // 64 - 1) % 2, -1, 1 << 30)
    inputs["block_table"] = bt
    run_and_check(dsa, wl, inputs, tol=TOL_FP8)


def test_long_decode_fp8_paged_full_size_sampled(dsa):
    wl = syn.WORKLOADS["long_decode_fp8_paged"]
    rng = np.random.default_rng(16)
    rows = sorted(set([0, 1, 63] + list(rng.integers(0, wl.T, 9))))
    run_and_check(dsa, wl, syn.generate(wl), rows=rows, tol=TOL_FP8)
