"""The GPU parity checks are not vacuous (CPU): fed the oracle's own outputs
they pass, and fed outputs with a planted error they fail."""
import numpy as np
import pytest

import dsa_synth as syn
import oracle
from parity_util import TOL_BF16, check_scores, check_topk


@pytest.fixture(scope="module")
def case():
    wl = syn.Workload("h", syn.MODE_POSITIONS, T=4, H=4, D=128, index_topk=20, S=300,
                      pos_lo=50, pos_hi=300, w_scale=0.5, seed=9)
    inputs = syn.generate(wl)
    P = oracle.Problem(wl, inputs)
    rows = list(range(wl.T))
    orc = P.scores(rows)
    tk = P.topk(rows, orc, wl.index_topk)
    return wl, P, rows, orc, np.asarray(tk)


def _copy(rows):
    return [r.copy() for r in rows]


def test_exact_outputs_pass(case):
    wl, P, rows, orc, tk = case
    assert check_scores(P, rows, _copy(orc), orc, TOL_BF16) == 0.0
    check_topk(P, rows, tk.copy(), _copy(orc), orc, wl.index_topk, TOL_BF16)


def test_a_score_off_by_more_than_the_tolerance_fails(case):
    wl, P, rows, orc, tk = case
    bad = _copy(orc)
    _, L, last, _ = P.row_info(2)
    scale = np.abs(orc[2][:last + 1]).max()
    bad[2][last // 2] += 1.5 * TOL_BF16 * scale
    with pytest.raises(AssertionError):
        check_scores(P, rows, bad, orc, TOL_BF16)


def test_a_masked_slot_not_at_the_bound_fails(case):
    wl, P, rows, orc, tk = case
    bad = _copy(orc)
    _, L, last, _ = P.row_info(1)
    assert last + 1 < L
    bad[1][last + 1] = 0.0
    with pytest.raises(AssertionError):
        check_scores(P, rows, bad, orc, TOL_BF16)


def test_a_wrong_selected_slot_fails(case):
    wl, P, rows, orc, tk = case
    bad = tk.copy()
    _, L, last, _ = P.row_info(0)
    chosen = set(bad[0].tolist())
    outsider = next(s for s in range(last + 1) if s not in chosen)
    bad[0][0] = outsider
    with pytest.raises(AssertionError):
        check_topk(P, rows, bad, _copy(orc), orc, wl.index_topk, TOL_BF16)


def test_a_masked_slot_selected_or_missing_padding_fails(case):
    wl, P, rows, orc, tk = case
    _, L, last, _ = P.row_info(3)
    bad = tk.copy()
    bad[3][0] = last + 1                 # a masked slot
    with pytest.raises(AssertionError):
        check_topk(P, rows, bad, _copy(orc), orc, wl.index_topk, TOL_BF16)
    # a row with fewer valid slots than k must be padded with -1
    short = dict(syn.generate(wl), positions=np.array([4, 299, 299, 299], np.int32))
    Ps = oracle.Problem(wl, short)
    so = Ps.scores(rows)
    st = np.asarray(Ps.topk(rows, so, wl.index_topk))
    st_bad = st.copy()
    st_bad[0][st_bad[0] == -1] = 0      # padding replaced by a duplicate slot
    with pytest.raises(AssertionError):
        check_topk(Ps, rows, st_bad, _copy(so), so, wl.index_topk, TOL_BF16)
