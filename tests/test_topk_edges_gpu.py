"""Top-k edge cases at full row lengths, through the C ABI (GPU only).

Decode rows longer than 4093 slots go to the cluster kernel (one
thread-block cluster per row), causal rows longer than 12288 slots stream
from L2 on every pass of the causal kernel. Both are checked here on rows
with exact ties around the threshold, all-equal rows, a threshold bin
holding more candidates than a cluster rank gathers at once, and partial
ties (only some of the keys equal to the k-th score are taken): the GPU set
must be the oracle's selection on the GPU's own scores, lower slots first
among ties (DeepSeek-V3.2 Sparse Indexer Kernel API Reference, Notes: an
unordered set). Rows whose buffer starts off a 16-byte boundary are checked
at the largest lengths of the register path.
"""
import numpy as np
import pytest
import torch

import dsa_synth as syn
import oracle
from parity_util import TOL_BF16, TOL_FP8, check_scores, check_topk, gpu_rows

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def dsa():
    assert torch.cuda.is_available(), "GPU tests need a CUDA device"
    import sparse_attention_lightning_tcgen05_b200 as m
    from sparse_attention_lightning_tcgen05_b200.problem import DeviceProblem
    return m, DeviceProblem


def run(dsa, wl, inputs, rows=None, tol=TOL_BF16, exact=False, **kw):
    m, DeviceProblem = dsa
    dp = DeviceProblem.from_workload(wl, inputs, **kw)
    dp.forward()
    assert dp.device_status() == m.DSA_OK
    P = oracle.Problem(wl, inputs)
    rows = list(range(wl.T)) if rows is None else sorted(set(int(r) for r in rows))
    orc = P.scores(rows)
    gpu = gpu_rows(P, dp.scores, rows)
    if exact:
        for t, g, o in zip(rows, gpu, orc):
            np.testing.assert_array_equal(g, o, err_msg=f"row {t}")
    check_scores(P, rows, gpu, orc, tol)
    check_topk(P, rows, dp.topk.cpu().numpy()[rows], gpu, orc, wl.index_topk, tol)
    return dp, P, rows, gpu


def decode_wl(T, H, S, k, pos, seed, shared=False):
    return syn.Workload("d", syn.MODE_POSITIONS, T=T, H=H, D=128, index_topk=k, S=S,
                        shared_cache=shared, pos_lo=pos[0], pos_hi=pos[1],
                        w_scale=1.0 / np.sqrt(H), seed=seed)


# ---- the cluster kernel (decode rows > 4093 slots) ----------------------------

@pytest.mark.parametrize("S,k", [(8192, 2048), (32768, 2048), (131072, 1024)])
def test_cluster_topk_integer_ties(dsa, S, k):
    """H=1 integer inputs: a few hundred distinct score values over the row,
    so thousands of keys tie at the k-th score and only some are taken."""
    wl = decode_wl(T=4, H=1, S=S, k=k, pos=(S // 2, S), seed=100 + S % 97)
    inputs = syn.generate(wl, value_kind="int")
    inputs["positions"][0] = S - 1          # a full row
    run(dsa, wl, inputs, exact=True)


@pytest.mark.parametrize("S", [8192, 32768, 131072])
def test_cluster_topk_all_scores_equal(dsa, S):
    """q = 0: every valid score is 0, the key range is empty (no value
    round), and the set is the k lowest slots."""
    wl = decode_wl(T=3, H=64, S=S, k=2048, pos=(S // 3, S), seed=110)
    inputs = syn.generate(wl)
    inputs["q"] = np.zeros_like(inputs["q"])
    run(dsa, wl, inputs, exact=True)


@pytest.mark.parametrize("S", [8192, 32768, 131072])
def test_cluster_topk_crowded_threshold_bin(dsa, S):
    """Most keys are zero rows (score exactly 0) and a few hundred are not:
    the k-th score is 0, its bin holds far more than the 1024 candidates a
    rank gathers, so the histogram rounds repeat down to the last key bit and
    only the lowest of the tied slots are taken."""
    wl = decode_wl(T=4, H=8, S=S, k=2048, pos=(S - 64, S), seed=120)
    inputs = syn.generate(wl, value_kind="int")
    k = inputs["k"].reshape(wl.T, S, 128)
    rng = np.random.default_rng(7)
    for t in range(wl.T):
        keep = rng.choice(S, size=300, replace=False)
        mask = np.zeros(S, bool)
        mask[keep] = True
        k[t][~mask] = 0
    inputs["k"] = k.reshape(-1, 128)
    run(dsa, wl, inputs, exact=True)


def test_cluster_topk_few_distinct_values(dsa):
    """Scores from {0, 1, 2}: every histogram round sees two or three crowded
    bins and the threshold's ties are a partial set."""
    S = 32768
    wl = decode_wl(T=2, H=1, S=S, k=2048, pos=(S - 1, S), seed=130)
    inputs = syn.generate(wl, value_kind="int")
    rng = np.random.default_rng(8)
    q = np.zeros((wl.T, 1, 128), np.float32)
    q[:, :, 0] = 1.0
    kk = np.zeros((wl.T * S, 128), np.float32)
    kk[:, 0] = rng.integers(0, 3, size=wl.T * S)
    inputs["q"] = syn.f32_to_bf16_bits(q)
    inputs["k"] = syn.f32_to_bf16_bits(kk)
    inputs["w"] = np.ones((wl.T, 1), np.float32)
    run(dsa, wl, inputs, exact=True)


def test_long_decode_fp8_all_rows(dsa):
    """Every one of the 64 rows of the long-context fp8 decode (131072 slots a
    cache, cluster top-k of 1024)."""
    wl = syn.WORKLOADS["long_decode_fp8"]
    run(dsa, wl, syn.generate(wl), tol=TOL_FP8)


# ---- causal rows longer than the 12288-key stage --------------------------------

def test_causal_streamed_rows_integer_ties(dsa):
    """One packed sequence of 20000 tokens, H=1 integer inputs: rows past
    12288 slots stream from L2 on every pass, with many exact ties."""
    wl = syn.Workload("c", syn.MODE_CAUSAL, T=20000, H=1, D=128, index_topk=2048,
                      seqlens=(20000,), w_scale=1.0, seed=140)
    inputs = syn.generate(wl, value_kind="int")
    rng = np.random.default_rng(9)
    rows = [0, 1, 2047, 2048, 12287, 12288, 12289, 16383, 19998, 19999] + \
        list(rng.integers(12288, 20000, 6))
    run(dsa, wl, inputs, rows=rows, exact=True)


def test_causal_streamed_rows_crowded_and_equal(dsa):
    """Streamed causal rows (> 12288 slots) where most keys are zero rows
    (a crowded threshold bin, partial ties) and a sequence whose queries are
    all zero (every score 0)."""
    wl = syn.Workload("c", syn.MODE_CAUSAL, T=2 * 14000, H=4, D=128, index_topk=2048,
                      seqlens=(14000, 14000), w_scale=0.5, seed=141)
    inputs = syn.generate(wl, value_kind="int")
    rng = np.random.default_rng(10)
    kz = rng.random(wl.T) < 0.97
    inputs["k"][kz] = 0
    inputs["q"][14000:] = 0
    rows = [12287, 12288, 13000, 13999, 14000 + 12288, 14000 + 13999] + \
        list(rng.integers(12288, 14000, 3))
    run(dsa, wl, inputs, rows=rows, exact=True)


# ---- the register path at its largest rows, rows off a 16-byte boundary --------

@pytest.mark.parametrize("S", [2045, 2046, 2047, 4093, 4094, 4095])
def test_misaligned_rows_at_full_capacity(dsa, S):
    """Rows 1-3 start 1-3 floats past a 16-byte boundary (S odd or 2 mod 4)
    and hold S or S-1 valid slots: together with the offset they fill the
    register path's buffer (or exceed it, then another kernel takes them)."""
    wl = decode_wl(T=5, H=16, S=S, k=64, pos=(0, S), seed=150, shared=True)
    inputs = syn.generate(wl)
    inputs["positions"] = np.array([S - 1, S - 1, S - 2, S - 1, S + 9], np.int32)
    run(dsa, wl, inputs)


@pytest.mark.parametrize("S", [2048, 4096])
def test_topk_of_a_score_buffer_off_16_bytes(dsa, S):
    """dsa_indexer_topk on score rows that start 4 bytes past a 16-byte
    boundary (a caller's buffer), at the register path's full row length."""
    m, _ = dsa
    wl = decode_wl(T=4, H=16, S=S, k=100, pos=(0, S), seed=151, shared=True)
    inputs = syn.generate(wl)
    inputs["positions"] = np.array([S - 1, S - 2, S - 1, 1000], np.int32)
    dp, P, rows, gpu = run(dsa, wl, inputs)
    buf = torch.empty(dp.scores.numel() + 1, dtype=torch.float32, device="cuda")
    shifted = buf[1:]
    assert shifted.data_ptr() % 16 == 4
    shifted.copy_(dp.scores)
    out = torch.full_like(dp.topk, -7)
    m.dsa_indexer_topk(dp.desc, shifted, dp.positions, out, dp.workspace, dp.ws_bytes,
                       torch.cuda.current_stream().cuda_stream)
    assert dp.device_status() == m.DSA_OK
    exact = P.topk(rows, gpu, wl.index_topk)
    got = out.cpu().numpy()
    for i, t in enumerate(rows):
        assert np.array_equal(np.sort(got[t]), np.sort(exact[i])), t
