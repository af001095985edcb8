"""Top-k-only forward (scores = NULL, DSA_FLAG_SCORES_IN_WORKSPACE), through
the C ABI (GPU only): the score rows live in the caller's workspace after
its header and the index set is the product (DeepSeek-V3.2 Sparse Indexer
Kernel API Reference, Returns). The set must be the oracle's selection on
those rows, and the rows must match the oracle's scores."""
import numpy as np
import pytest
import torch

import dsa_synth as syn
import oracle
from parity_util import TOL_BF16, TOL_FP8, check_scores, check_topk, gpu_rows

pytestmark = pytest.mark.gpu


@pytest.mark.parametrize("name,rows", [
    ("decode_batch", None),
    ("long_decode_fp8", [0, 17, 63]),
    ("c4_prefill", [0, 3, 4, 5000, 8191]),
    ("prefill_causal", [0, 1, 2047, 2048, 8191]),
])
def test_topk_only_forward(name, rows):
    assert torch.cuda.is_available()
    import sparse_attention_lightning_tcgen05_b200 as m
    from sparse_attention_lightning_tcgen05_b200.problem import DeviceProblem
    wl = syn.WORKLOADS[name]
    inputs = syn.generate(wl)
    dp = DeviceProblem.from_workload(wl, inputs, topk_only=True)
    n_scores = dp.scores.numel()
    assert dp.ws_bytes == 256 + 4 * n_scores
    dp.forward()
    assert dp.device_status() == m.DSA_OK
    tol = TOL_FP8 if wl.dtype == syn.DTYPE_FP8 else TOL_BF16
    rows = list(range(wl.T)) if rows is None else rows
    P = oracle.Problem(wl, inputs)
    orc = P.scores(rows)
    gpu = gpu_rows(P, dp.scores, rows)
    check_scores(P, rows, gpu, orc, tol)
    check_topk(P, rows, dp.topk.cpu().numpy()[rows], gpu, orc, wl.index_topk, tol)


def test_topk_only_rejects_a_short_workspace():
    import sparse_attention_lightning_tcgen05_b200 as m
    from sparse_attention_lightning_tcgen05_b200.problem import DeviceProblem
    wl = syn.WORKLOADS["tiny_decode"]
    dp = DeviceProblem.from_workload(wl, syn.generate(wl), topk_only=True)
    with pytest.raises(m.DsaError) as e:
        m.dsa_indexer_forward(dp.desc, dp.q, None, dp.w, dp.k_cache, None, dp.positions,
                              None, dp.topk, dp.workspace, dp.ws_bytes - 4)
    assert e.value.status == m.DSA_ERR_WORKSPACE
