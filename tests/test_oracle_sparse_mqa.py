"""Pins of the sparse-MQA oracle (the indexer's consumer) on the CPU: closed
forms, a dense softmax from scipy, masking and order invariance."""
import numpy as np
import pytest
from scipy.special import softmax

import dsa_synth as syn
from oracle.sparse_mqa import bf16_to_f64, sparse_mqa


def _inputs(B=2, S=3, H=4, D=128, K=50, ktop=8, seed=0):
    rng = np.random.default_rng(seed)
    q = syn.f32_to_bf16_bits(rng.standard_normal((B, S, H, D), dtype=np.float32))
    kv = syn.f32_to_bf16_bits(rng.standard_normal((B, K, D), dtype=np.float32))
    sinks = rng.standard_normal(H).astype(np.float32)
    idx = np.stack([np.stack([rng.permutation(K)[:ktop] for _ in range(S)]) for _ in range(B)])
    return q, kv, sinks, idx.astype(np.int32)


def test_one_kept_key_closed_form():
    q, kv, sinks, idx = _inputs(B=1, S=1, ktop=4)
    idx[0, 0, 1:] = -1
    out = sparse_mqa(q, kv, sinks, idx, 0.1)
    kvf, qf = bf16_to_f64(kv), bf16_to_f64(q)
    j = idx[0, 0, 0]
    for h in range(4):
        l = 0.1 * float(qf[0, 0, h] @ kvf[0, j])
        weight = 1.0 / (1.0 + np.exp(float(sinks[h]) - l))
        np.testing.assert_allclose(out[0, 0, h], weight * kvf[0, j], rtol=1e-13, atol=1e-15)


def test_zero_query_is_a_mean_with_the_sink():
    q, kv, sinks, idx = _inputs(ktop=6)
    q[:] = 0
    out = sparse_mqa(q, kv, sinks, idx, 0.5)
    kvf = bf16_to_f64(kv)
    for b in range(2):
        for s in range(3):
            for h in range(4):
                exp = kvf[b, idx[b, s]].sum(axis=0) / (6 + np.exp(float(sinks[h])))
                np.testing.assert_allclose(out[b, s, h], exp, rtol=1e-13, atol=1e-15)


def test_all_keys_kept_is_dense_attention_with_a_sink_column():
    q, kv, sinks, _ = _inputs(B=1, S=2, K=40)
    idx = np.tile(np.arange(40, dtype=np.int32), (1, 2, 1))
    scale = 1.0 / np.sqrt(128)
    out = sparse_mqa(q, kv, sinks, idx, scale)
    qf, kvf = bf16_to_f64(q), bf16_to_f64(kv)
    for s in range(2):
        for h in range(4):
            logits = np.concatenate([scale * (kvf[0] @ qf[0, s, h]), [float(sinks[h])]])
            p = softmax(logits)
            np.testing.assert_allclose(out[0, s, h], p[:-1] @ kvf[0], rtol=1e-12, atol=1e-14)


def test_masked_and_out_of_range_entries_are_removed():
    q, kv, sinks, idx = _inputs(ktop=8)
    kept = idx[:, :, :5].copy()
    noisy = idx.copy()
    noisy[:, :, 5] = -1
    noisy[:, :, 6] = 50          # == K: out of range
    noisy[:, :, 7] = -7
    np.testing.assert_array_equal(sparse_mqa(q, kv, sinks, noisy, 0.3),
                                  sparse_mqa(q, kv, sinks, kept, 0.3))


def test_index_order_does_not_matter():
    q, kv, sinks, idx = _inputs(ktop=8)
    perm = idx[:, :, ::-1].copy()
    np.testing.assert_allclose(sparse_mqa(q, kv, sinks, perm, 0.2),
                               sparse_mqa(q, kv, sinks, idx, 0.2), rtol=1e-13, atol=1e-15)


def test_no_kept_key_gives_zero_and_sink_limits():
    q, kv, sinks, idx = _inputs(ktop=4)
    none = np.full_like(idx, -1)
    assert np.all(sparse_mqa(q, kv, sinks, none, 0.2) == 0.0)
    # sink -> -inf: a plain softmax over the kept keys (weights sum to 1)
    q0 = q.copy()
    q0[:] = 0
    out = sparse_mqa(q0, kv, np.full(4, -np.inf, np.float32), idx, 0.2)
    kvf = bf16_to_f64(kv)
    np.testing.assert_allclose(out[1, 2, 3], kvf[1, idx[1, 2]].mean(axis=0), rtol=1e-13)
    # a sink far above every logit takes all the weight
    big = sparse_mqa(q, kv, np.full(4, 1e4, np.float32), idx, 0.2)
    assert np.abs(big).max() == 0.0


@pytest.mark.parametrize("seed", [1, 2])
def test_weights_are_a_convex_combination(seed):
    """With one-hot values, output feature j is key j's softmax weight, with
    the sink in the denominator: positive, and exactly the closed form."""
    rng = np.random.default_rng(seed)
    K, D = 4, 128
    basis = np.zeros((1, K, D), np.float32)
    for j in range(K):
        basis[0, j, j] = 1.0                      # one-hot values: out[j] is weight j
    q = syn.f32_to_bf16_bits(rng.standard_normal((1, 1, 2, D), dtype=np.float32))
    kv = syn.f32_to_bf16_bits(basis)
    sinks = np.array([0.5, -2.0], np.float32)
    idx = np.array([[[0, 1, 2, 3]]], np.int32)
    out = sparse_mqa(q, kv, sinks, idx, 1.0)
    for h in range(2):
        w = out[0, 0, h, :K]
        assert np.all(w > 0) and np.all(out[0, 0, h, K:] == 0)
        l = bf16_to_f64(q)[0, 0, h, :K]
        exp = np.exp(l) / (np.exp(l).sum() + np.exp(float(sinks[h])))
        np.testing.assert_allclose(w, exp, rtol=1e-13)
