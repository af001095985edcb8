"""dsa_indexer_forward_noalloc, the entry point for callers that cannot
allocate device memory (no workspace argument: the kernels' scratch is a
fixed array inside the library). Its outputs must equal those of
dsa_indexer_forward with a caller workspace, on two calls in a row (the
second call reuses the scratch the first one left behind).

Kept in a file of its own that pytest collects last."""
import numpy as np
import pytest
import torch

import dsa_synth as syn
from parity_util import TOL_BF16, TOL_FP8

pytestmark = pytest.mark.gpu


def _compare(ref_scores, ref_topk, scores, topk, tol=TOL_BF16):
    r, g = ref_scores.double().cpu().numpy(), scores.double().cpu().numpy()
    scale = np.abs(r[r > -1e38]).max()
    assert np.abs(g - r).max() <= tol * scale
    masked = r < -1e38
    assert np.array_equal(g[masked], r[masked])
    assert np.array_equal(np.sort(ref_topk.cpu().numpy(), axis=1),
                          np.sort(topk.cpu().numpy(), axis=1))


@pytest.mark.parametrize("name", ["tiny_decode", "decode_batch", "long_decode_fp8"])
def test_noalloc_matches_forward_twice(name):
    assert torch.cuda.is_available()
    import sparse_attention_lightning_tcgen05_b200 as dsa
    from sparse_attention_lightning_tcgen05_b200.problem import DeviceProblem
    wl = syn.WORKLOADS[name]
    dp = DeviceProblem.from_workload(wl, syn.generate(wl))
    dp.forward()
    assert dp.device_status() == dsa.DSA_OK
    stream = torch.cuda.current_stream().cuda_stream
    for _ in range(2):
        scores = torch.full_like(dp.scores, float("nan"))
        topk = torch.full_like(dp.topk, -7)
        dsa.dsa_indexer_forward_noalloc(dp.desc, dp.q, dp.q_scale, dp.w,
                                        dp.k_cache, dp.k_scale, dp.positions,
                                        scores, topk, stream)
        torch.cuda.synchronize()
        _compare(dp.scores, dp.topk, scores, topk,
                 TOL_FP8 if wl.dtype == syn.DTYPE_FP8 else TOL_BF16)


def test_noalloc_causal_matches_forward():
    import sparse_attention_lightning_tcgen05_b200 as dsa
    from sparse_attention_lightning_tcgen05_b200.problem import DeviceProblem
    wl = syn.Workload("c", syn.MODE_CAUSAL, T=1500, H=64, D=128, index_topk=256,
                      seqlens=(300, 1200), w_scale=0.125)
    dp = DeviceProblem.from_workload(wl, syn.generate(wl))
    dp.forward()
    for _ in range(2):
        scores = torch.full_like(dp.scores, float("nan"))
        topk = torch.full_like(dp.topk, -7)
        dsa.dsa_indexer_forward_noalloc(dp.desc, dp.q, dp.q_scale, dp.w,
                                        dp.k_cache, dp.k_scale, dp.positions,
                                        scores, topk,
                                        torch.cuda.current_stream().cuda_stream)
        torch.cuda.synchronize()
        _compare(dp.scores, dp.topk, scores, topk)
