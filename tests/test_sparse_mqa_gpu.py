"""The sparse-MQA consumer kernel vs the fp64 oracle (oracle/sparse_mqa.py),
through the C ABI (GPU only).

Tolerance, from the kernel's arithmetic: the logits and the sums are fp32
(products of bf16 values exact, errors ~1e-7 relative), the exponentials
2^x come from the hardware approximation (relative error ~2^-22), the
probabilities P enter the P.V product rounded to bf16 (relative error
<= 2^-9 each, so the weighted sum of values moves by <= 2^-9 * max|v|), and
the output is rounded to bf16 (<= 2^-9 * |out|). Every element must lie within
twice that bound: |gpu - oracle| <= 2^-8 * (max |kv| over the token's kept
rows + |oracle|).
"""
import numpy as np
import pytest
import torch

import dsa_synth as syn
from oracle.sparse_mqa import bf16_to_f64, sparse_mqa

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def dsa():
    assert torch.cuda.is_available(), "GPU tests need a CUDA device"
    import sparse_attention_lightning_tcgen05_b200 as m
    return m


def run_gpu(m, inputs, H, sm_scale, wait_limit_ns=0):
    q, kv, sinks, idx = inputs["q"], inputs["kv"], inputs["sinks"], inputs["idx"]
    B, S, _, D = q.shape
    K, K_top = kv.shape[1], idx.shape[2]
    desc = m.make_mqa_desc(B, S, H, K, K_top, sm_scale, wait_limit_ns=wait_limit_ns)
    dq = torch.from_numpy(q.view(np.int16)).cuda()
    dkv = torch.from_numpy(kv.view(np.int16)).cuda()
    ds = torch.from_numpy(np.ascontiguousarray(sinks, np.float32)).cuda()
    di = torch.from_numpy(np.ascontiguousarray(idx, np.int32)).cuda()
    out = torch.full((B, S, H, D), -7, dtype=torch.int16, device="cuda")
    nbytes = m.dsa_sparse_mqa_workspace_size(desc)
    ws = torch.zeros(nbytes, dtype=torch.uint8, device="cuda")
    m.dsa_sparse_mqa_forward(desc, dq, dkv, ds, di, out, ws, nbytes,
                             torch.cuda.current_stream().cuda_stream)
    assert m.dsa_indexer_get_error(ws) == m.DSA_OK
    return bf16_to_f64(out.cpu().numpy().view(np.uint16)), nbytes


def check(inputs, gpu, sm_scale, tokens=None):
    """Compare the listed (b, s) tokens (all when None) with the oracle."""
    q, kv, sinks, idx = inputs["q"], inputs["kv"], inputs["sinks"], inputs["idx"]
    B, S = q.shape[:2]
    tokens = [(b, s) for b in range(B) for s in range(S)] if tokens is None else tokens
    kvf = bf16_to_f64(kv)
    worst = 0.0
    for b, s in tokens:
        ref = sparse_mqa(q[b:b + 1, s:s + 1], kv[b:b + 1], sinks, idx[b:b + 1, s:s + 1],
                         sm_scale)[0, 0]
        g = gpu[b, s]
        kept = [int(j) for j in idx[b, s] if 0 <= int(j) < kv.shape[1]]
        if not kept:
            assert np.all(g == 0.0), (b, s)
            continue
        vmax = np.abs(kvf[b, kept]).max()
        err = np.abs(g - ref)
        bound = 2.0 ** -8 * (vmax + np.abs(ref))
        assert np.all(err <= bound), (b, s, float((err / bound).max()))
        worst = max(worst, float((err / (vmax + np.abs(ref))).max()))
    return worst


def small_inputs(B, S, H, K, K_top, seed, masked_frac=0.1):
    rng = np.random.default_rng(seed)
    q = syn.f32_to_bf16_bits(rng.standard_normal((B, S, H, 128), dtype=np.float32))
    kv = syn.f32_to_bf16_bits(rng.standard_normal((B, K, 128), dtype=np.float32))
    sinks = rng.standard_normal(H).astype(np.float32)
    idx = rng.integers(0, K, size=(B, S, K_top)).astype(np.int32)
    drop = rng.random((B, S, K_top)) < masked_frac
    idx[drop] = np.where(rng.random(drop.sum()) < 0.5, -1, K + rng.integers(0, 50, drop.sum()))
    return dict(q=q, kv=kv, sinks=sinks, idx=idx)


@pytest.mark.parametrize("H", [1, 4, 16, 64, 100, 128])
def test_sparse_mqa_heads(dsa, H):
    """Index rows of 300 entries (a partial third tile), -1 and out-of-range
    entries masked, repeated entries counted once per occurrence."""
    inputs = small_inputs(2, 3, H, 500, 300, seed=H)
    gpu, _ = run_gpu(dsa, inputs, H, 128 ** -0.5)
    check(inputs, gpu, 128 ** -0.5)


def test_sparse_mqa_decode_split_ranges(dsa):
    """The decode consumer: 16 tokens, 2048 entries each -- every index row
    is split into ranges over the SMs and merged by the second kernel."""
    wl = syn.MQA_WORKLOADS["mqa_decode"]
    inputs = syn.generate_mqa(wl)
    gpu, nbytes = run_gpu(dsa, inputs, wl.H, wl.sm_scale)
    assert nbytes > 256                                  # partial results in use
    check(inputs, gpu, wl.sm_scale)


def test_sparse_mqa_many_tokens_per_cta(dsa):
    """More tokens than SMs: one range per token, each CTA walks many items
    (the TMEM accumulator and the query tile reused item after item)."""
    inputs = small_inputs(2, 400, 64, 3000, 640, seed=5)
    gpu, nbytes = run_gpu(dsa, inputs, 64, 128 ** -0.5)
    assert nbytes == 256
    rng = np.random.default_rng(6)
    tokens = [(0, 0), (1, 399)] + [(int(b), int(s)) for b, s in
                                   zip(rng.integers(0, 2, 30), rng.integers(0, 400, 30))]
    check(inputs, gpu, 128 ** -0.5, tokens)


def test_sparse_mqa_no_kept_entry_and_sinks(dsa):
    """Tokens whose entries are all masked give 0; a very large sink takes
    nearly all the weight, a very small one none."""
    inputs = small_inputs(1, 6, 8, 400, 256, seed=7)
    inputs["idx"][0, 0] = -1
    inputs["idx"][0, 1] = 400                              # all out of range
    inputs["idx"][0, 2, 128:] = -1                         # a whole masked tile
    inputs["sinks"][:4] = np.array([30.0, -30.0, 0.0, 5.0], np.float32)
    gpu, _ = run_gpu(dsa, inputs, 8, 128 ** -0.5)
    assert np.all(gpu[0, 0] == 0) and np.all(gpu[0, 1] == 0)
    check(inputs, gpu, 128 ** -0.5)


def test_sparse_mqa_growing_max_rescales(dsa):
    """A large logit scale with the entries ordered by increasing logit: the
    running max grows by far more than 2^8 across tiles, so the accumulated
    output is rescaled in TMEM."""
    inputs = small_inputs(1, 2, 16, 2000, 1024, seed=8, masked_frac=0.0)
    q = bf16_to_f64(inputs["q"])
    kv = bf16_to_f64(inputs["kv"])
    for s in range(2):
        logit = kv[0][inputs["idx"][0, s]] @ q[0, s, 0]
        inputs["idx"][0, s] = inputs["idx"][0, s][np.argsort(logit)]
    gpu, _ = run_gpu(dsa, inputs, 16, 1.0)
    check(inputs, gpu, 1.0)


def test_sparse_mqa_prefill_sampled(dsa):
    """The prefill consumer: 8192 tokens with causal index rows (-1 padded
    below 2048 visible keys), checked on sampled tokens."""
    wl = syn.MQA_WORKLOADS["mqa_prefill"]
    inputs = syn.generate_mqa(wl)
    gpu, _ = run_gpu(dsa, inputs, wl.H, wl.sm_scale)
    rng = np.random.default_rng(9)
    tokens = [(0, s) for s in [0, 1, 2046, 2047, 2048, 8191]] + \
        [(0, int(s)) for s in rng.integers(0, 8192, 10)]
    check(inputs, gpu, wl.sm_scale, tokens)


def test_sparse_mqa_on_the_indexer_top_k(dsa):
    """The path end to end: the decode batch's indexer forward selects 2048
    slots per token; sparse MQA attends over them (q and kv drawn for it)."""
    from sparse_attention_lightning_tcgen05_b200.problem import DeviceProblem
    wl = syn.WORKLOADS["decode_batch"]
    dp = DeviceProblem.from_workload(wl, syn.generate(wl), topk_only=True)
    dp.forward()
    assert dp.device_status() == dsa.DSA_OK
    idx = dp.topk.cpu().numpy().reshape(wl.T, 1, wl.index_topk)
    mwl = syn.MqaWorkload("chain", B=wl.T, S=1, H=64, K=wl.S, K_top=wl.index_topk)
    inputs = syn.generate_mqa(mwl, seed=3)
    inputs["idx"] = idx
    gpu, _ = run_gpu(dsa, inputs, 64, mwl.sm_scale)
    check(inputs, gpu, mwl.sm_scale)
