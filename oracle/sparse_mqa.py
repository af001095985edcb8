"""fp64 oracle of the indexer's consumer: sparse MQA over top-k key indices.

TEST INFRASTRUCTURE. Only the tests use this module; the CUDA library never
calls it.

What it computes (NeMo AutoModel optimized_kernels, sparse_attention_torch
and dense_attention_topk_torch: q [B, S, H, D], a single-head kv [B, K, D],
per-head sink logits sinks [H], key indices topk_idxs [B, S, K_top] where -1
masks an entry, sm_scale; the DeepSeek-V4 inference kernel write-up, sparse
attention section: keys gathered by index, masked entries scored -inf, an
online softmax whose denominator gains exp(sink - max) at the end), for
every query (b, s, h):

    l_j   = sm_scale * q[b,s,h,:] . kv[b, idx_j, :]      for each kept j
    out   = sum_j e^{l_j} kv[b, idx_j, :] / (sum_j e^{l_j} + e^{sinks[h]})

Readings where the pages are silent: the single kv head serves as both key
and value (MQA over one latent head), so out has D features; an index
outside [0, K) is masked like -1 (the write-up pads out-of-range entries
with -1); a query with no kept index gets out = 0 (the sink alone); repeated
indices count once per occurrence (the indexer never repeats one). The
maximum subtracted for stability is max(max_j l_j, sinks[h]); it cancels.

Inputs are decoded to float64 first (q, kv as bf16 bit patterns, sinks as
float32); the dot products and the weighted sum of values are numpy fp64
matrix products.
"""
from __future__ import annotations

import numpy as np


def bf16_to_f64(bits: np.ndarray) -> np.ndarray:
    """bf16 bit patterns (uint16) to float64, exactly."""
    return (np.asarray(bits, np.uint16).astype(np.uint32) << 16).view(np.float32).astype(np.float64)


def sparse_mqa(q_bits: np.ndarray, kv_bits: np.ndarray, sinks: np.ndarray,
               topk_idxs: np.ndarray, sm_scale: float) -> np.ndarray:
    """out [B, S, H, D] float64 for q [B, S, H, D], kv [B, K, D] (bf16 bits),
    sinks [H] float32, topk_idxs [B, S, K_top] int32."""
    q = bf16_to_f64(q_bits)
    kv = bf16_to_f64(kv_bits)
    sinks = np.asarray(sinks, np.float32).astype(np.float64)
    idx = np.asarray(topk_idxs)
    B, S, H, D = q.shape
    K = kv.shape[1]
    out = np.zeros((B, S, H, D), np.float64)
    for b in range(B):
        for s in range(S):
            kept = [int(j) for j in idx[b, s] if 0 <= int(j) < K]
            if not kept:
                continue
            keys = kv[b, kept]                              # [n, D]
            for h in range(H):
                logits = sm_scale * (keys @ q[b, s, h])     # [n]
                m = max(float(logits.max()), float(sinks[h]))
                e = np.exp(logits - m)
                denom = float(e.sum()) + float(np.exp(sinks[h] - m))
                out[b, s, h] = (e @ keys) / denom
    return out
