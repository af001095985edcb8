"""Device-side failure detection, through the C ABI (GPU only).

Nothing here faults, traps or hangs a GPU. DSA_FLAG_SELFTEST_STALL makes the
score kernel's MMA warp wait on a barrier that nothing completes; with a wait
limit of one millisecond (desc.wait_limit_ns) that wait runs out: the kernel
records DSA_ERR_TIMEOUT in the workspace, lets the copies it has in flight
land (those drains have their own 4 s bound) and exits. A cu_seqlens array that breaks the
descriptor's promise is caught by the device-side check before any score or
top-k is written. In both cases dsa_indexer_get_error reports the status,
and the next call on the same workspace runs normally.
"""
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


def check_against_oracle(dp, wl, inputs, rows):
    P = oracle.Problem(wl, inputs)
    orc = P.scores(rows)
    gpu = gpu_rows(P, dp.scores, rows)
    check_scores(P, rows, gpu, orc, TOL_BF16)
    check_topk(P, rows, dp.topk.cpu().numpy()[rows], gpu, orc, wl.index_topk, TOL_BF16)


@pytest.mark.parametrize("name", ["decode_batch", "prefill_causal"])
def test_wait_timeout_is_reported_and_the_next_call_is_clean(dsa, name):
    m, DeviceProblem = dsa
    wl = syn.WORKLOADS[name]
    inputs = syn.generate(wl)
    dp = DeviceProblem.from_workload(wl, inputs, wait_limit_ns=1_000_000)
    dp.desc.flags |= m.DSA_FLAG_SELFTEST_STALL
    dp.scores.zero_()
    dp.score()
    assert dp.device_status() == m.DSA_ERR_TIMEOUT
    assert dp.device_status() == m.DSA_OK            # read and cleared
    dp.forward()                                      # the whole forward, stalled
    assert dp.device_status() == m.DSA_ERR_TIMEOUT
    dp.desc.flags &= ~m.DSA_FLAG_SELFTEST_STALL       # a normal call, same workspace
    dp.desc.wait_limit_ns = 0                         # the default limit again
    dp.forward()
    assert dp.device_status() == m.DSA_OK
    rows = [0, 1, wl.T // 2, wl.T - 1]
    check_against_oracle(dp, wl, inputs, rows)


@pytest.mark.parametrize("bad", ["first_not_zero", "decreasing", "last_not_T",
                                 "last_past_T"])
def test_bad_cu_seqlens_write_nothing(dsa, bad):
    m, DeviceProblem = dsa
    seqlens = (5, 130, 257)
    wl = syn.Workload("c", syn.MODE_CAUSAL, T=sum(seqlens), H=64, D=128, index_topk=64,
                      seqlens=seqlens, w_scale=0.125, seed=160)
    inputs = syn.generate(wl)
    dp = DeviceProblem.from_workload(wl, inputs)
    good = dp.cu_seqlens.clone()
    cu = good.cpu().numpy().copy()
    if bad == "first_not_zero":
        cu[0] = 1
    elif bad == "decreasing":
        cu[1], cu[2] = cu[2], cu[1]
    elif bad == "last_not_T":
        cu[-1] -= 1
    else:
        cu[-1] += 100
    dp.cu_seqlens.copy_(torch.from_numpy(cu))
    dp.scores.fill_(7.0)
    dp.topk.fill_(-7)
    dp.forward()
    assert dp.device_status() == m.DSA_ERR_INVALID_ARG
    assert torch.all(dp.scores == 7.0) and torch.all(dp.topk == -7)
    dp.run_topk()                                     # a top-k call of its own
    assert dp.device_status() == m.DSA_ERR_INVALID_ARG
    assert torch.all(dp.topk == -7)
    dp.cu_seqlens.copy_(good)                         # the same workspace, a good array
    dp.forward()
    assert dp.device_status() == m.DSA_OK
    check_against_oracle(dp, wl, inputs, [0, 4, 5, 134, 135, wl.T - 1])
