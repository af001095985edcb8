"""fp64 oracle of the indexer's front end -- TEST INFRASTRUCTURE.

Only the tests use this module; the CUDA library never calls it.

What it computes, per query token t (DeepSeek-V3.2 Sparse Indexer Kernel API
Reference, deepseek_v32_sparse_indexer, Parameters: hidden_states [n_tokens,
hidden], qr [n_tokens, q_lora_rank] (q_norm(wq_a(x)) from the MLA block), wq_b
(the query projection), wk [hidden, head_dim] (the key projection),
k_norm_weight / k_norm_bias (fp32 LayerNorm gain and bias of the key),
weights_proj [hidden, n_heads] (the per-head weight projection), cos / sin
[n_tokens, rope_dim // 2] (RoPE tables, rope_dim = the leading feature span
RoPE rotates), key_cache written in place at each token's position; Sparse
Attention Indexer MX BF16Score Kernel API Reference: the bf16 score path drops
the Hadamard rotation, a no-op for q . k; tokamax Supported Ops,
deepseek_rope: DeepSeek applies interleaved RoPE):

    q[t, h, :]  = rope(qr[t] @ wq_b[h*D:(h+1)*D, :]^T, t)
    k[t, :]     = rope(layernorm(x[t] @ wk^T), t)
    w[t, :]     = w_scale * (x[t] @ weights_proj^T)

    rope(v, t): for i < rope_dim / 2, the pair (v[2i], v[2i+1]) becomes
                (v[2i] cos[t,i] - v[2i+1] sin[t,i], v[2i] sin[t,i] + v[2i+1] cos[t,i]);
                features from rope_dim on are unchanged;
    layernorm(v) = (v - mean(v)) / sqrt(var(v) + eps) * gain + bias
                   (mean and the biased variance over the D features).

Readings where the pages are silent: weights are stored [out_features,
in_features] (the contraction contiguous); wq_b's output features are head
major (feature h*D + d is head h, dim d); RoPE rotates interleaved pairs of
the leading rope_dim features of every head (and of the key); LayerNorm comes
before RoPE; the per-head weights carry one scalar factor w_scale (the pages
give none; the softmax scale folds into it). The Hadamard rotation is left
out: the pages' bf16 score path drops it.

Inputs are decoded to float64 first (bf16 bit patterns; float32 tables and
norm parameters); the projections are numpy fp64 matrix products.
"""
from __future__ import annotations

import numpy as np


def bf16_to_f64(bits: np.ndarray) -> np.ndarray:
    """bf16 bit patterns (uint16) to float64, exactly."""
    return (np.asarray(bits, np.uint16).astype(np.uint32) << 16).view(np.float32).astype(
        np.float64)


def rope(v: np.ndarray, cos: np.ndarray, sin: np.ndarray, rope_dim: int) -> np.ndarray:
    """Interleaved RoPE on the leading rope_dim features of the last axis.
    v [..., D]; cos, sin broadcastable to [..., rope_dim // 2]."""
    out = np.array(v, dtype=np.float64, copy=True)
    even = v[..., 0:rope_dim:2]
    odd = v[..., 1:rope_dim:2]
    c = np.asarray(cos, np.float64)
    s = np.asarray(sin, np.float64)
    out[..., 0:rope_dim:2] = even * c - odd * s
    out[..., 1:rope_dim:2] = even * s + odd * c
    return out


def layernorm(v: np.ndarray, gain: np.ndarray, bias: np.ndarray, eps: float) -> np.ndarray:
    """LayerNorm over the last axis: biased variance, eps inside the root."""
    v = np.asarray(v, np.float64)
    mean = v.mean(axis=-1, keepdims=True)
    var = ((v - mean) ** 2).mean(axis=-1, keepdims=True)
    return (v - mean) / np.sqrt(var + eps) * np.asarray(gain, np.float64) + \
        np.asarray(bias, np.float64)


def front_end(x_bits, qr_bits, wq_b_bits, wk_bits, wp_bits, gain, bias, cos, sin, *,
              H: int, D: int, rope_dim: int, eps: float, w_scale: float):
    """(q [T, H, D], k [T, D], w [T, H]) in float64."""
    x = bf16_to_f64(x_bits)
    qr = bf16_to_f64(qr_bits)
    wq_b = bf16_to_f64(wq_b_bits)
    wk = bf16_to_f64(wk_bits)
    wp = bf16_to_f64(wp_bits)
    T = x.shape[0]
    q = (qr @ wq_b.T).reshape(T, H, D)
    q = rope(q, np.asarray(cos)[:, None, :], np.asarray(sin)[:, None, :], rope_dim)
    k = layernorm(x @ wk.T, gain, bias, eps)
    k = rope(k, cos, sin, rope_dim)
    w = w_scale * (x @ wp.T)
    return q, k, w
