"""Comparison helpers for the GPU parity tests (CUDA path vs fp64 oracle).

Acceptance rules:
 - scores: |gpu - oracle| <= tol * max_valid |oracle| on every slot of a row
   (tol 2e-2 for bf16 inputs, 6e-2 for fp8), masked slots bit-exact at the
   mask bound; a row whose valid oracle scores are all 0 must be exactly 0;
 - top-k, bit-exact: the GPU's set equals the oracle's selection applied to
   the GPU's own scores (same tie rule: lower slot first);
 - top-k vs the oracle's own selection: the symmetric difference may only
   hold slots whose oracle score is within tol * max_valid |oracle| of the
   oracle's k-th score.
"""
from __future__ import annotations

import numpy as np
import torch

import oracle

MB = float.fromhex("-0x1.FEp127")
TOL_BF16 = 2e-2
TOL_FP8 = 6e-2


def gpu_rows(P: oracle.Problem, dev_scores: torch.Tensor, rows):
    """Copy the listed score rows of the packed GPU buffer to the host."""
    out = []
    for t in rows:
        _, L, _, off = P.row_info(int(t))
        out.append(dev_scores[off:off + L].double().cpu().numpy())
    return out


def check_scores(P: oracle.Problem, rows, gpu, orc, tol):
    worst = 0.0
    for t, g, o in zip(rows, gpu, orc):
        _, L, last, _ = P.row_info(int(t))
        n = max(0, min(last + 1, L))
        assert np.all(g[n:] == MB), f"row {t}: masked slots not at the bound"
        assert np.all(o[n:] == MB)
        if n == 0:
            continue
        scale = np.abs(o[:n]).max()
        err = np.abs(g[:n] - o[:n]).max()
        if scale == 0.0:
            assert err == 0.0, f"row {t}: expected exact zeros"
            continue
        worst = max(worst, err / scale)
        assert err <= tol * scale, f"row {t}: rel err {err / scale:.3g} > {tol}"
    return worst


def check_topk(P: oracle.Problem, rows, gpu_topk, gpu_scores, orc_scores, k,
               tol):
    """gpu_topk: [len(rows), k] int array from the device."""
    exact = P.topk(rows, gpu_scores, k)
    ref = P.topk(rows, orc_scores, k)
    for i, t in enumerate(rows):
        g = np.sort(gpu_topk[i])
        assert np.array_equal(g, np.sort(exact[i])), \
            f"row {t}: top-k differs from the oracle's selection on GPU scores"
        _, L, last, _ = P.row_info(int(t))
        n = max(0, min(last + 1, L))
        sel = set(int(s) for s in ref[i] if s >= 0)
        diff = (set(int(s) for s in gpu_topk[i] if s >= 0) ^ sel)
        if diff:
            o = orc_scores[i]
            kth = min(o[s] for s in sel)
            scale = np.abs(o[:n]).max()
            for s in diff:
                assert abs(o[s] - kth) <= tol * scale, \
                    f"row {t}: slot {s} outside the tolerance band"
        assert (gpu_topk[i] == -1).sum() == k - min(k, n)
