"""bench.py's workload arithmetic on the CPU, checked against the oracle's
own row geometry (an independent statement of which slots are valid)."""
import os
import sys

import numpy as np
import pytest

import dsa_synth as syn
import oracle

sys.path.insert(0, os.path.dirname(os.path.dirname(os.path.abspath(__file__))))
import bench  # noqa: E402


def _cases():
    yield syn.Workload("pos", syn.MODE_POSITIONS, T=7, H=4, D=128, index_topk=8, S=300,
                       pos_lo=0, pos_hi=400, seed=1)
    yield syn.Workload("shared", syn.MODE_POSITIONS, T=9, H=4, D=128, index_topk=8, S=300,
                       shared_cache=True, pos_lo=0, pos_hi=300, seed=2)
    yield syn.Workload("causal", syn.MODE_CAUSAL, T=140, H=4, D=128, index_topk=8,
                       seqlens=(1, 7, 132), seed=3)
    yield syn.Workload("c4", syn.MODE_COMPRESSED, T=90, H=4, D=128, index_topk=8, S=30,
                       compress_ratio=4, query_start=3, seed=4)
    yield syn.Workload("paged", syn.MODE_POSITIONS, T=5, H=4, D=128, index_topk=8, S=500,
                       pos_lo=0, pos_hi=500, page_size=32, seed=5)


@pytest.mark.parametrize("wl", list(_cases()), ids=lambda w: w.name)
def test_valid_pairs_and_score_elements_match_the_oracle_geometry(wl):
    inputs = syn.generate(wl)
    P = oracle.Problem(wl, inputs)
    valid = elems = 0
    for t in range(wl.T):
        _, L, last, _ = P.row_info(t)
        valid += max(0, min(last + 1, L))
        elems += L
    assert bench.valid_pairs(wl, inputs) == valid
    assert bench.score_elems(wl) == elems


def test_algorithmic_bytes_and_flops_by_hand():
    """Shared cache, bf16: q 2*H*D per token, w 4*H per token, the keys up to
    the largest position once, the whole score rows, the index rows."""
    wl = syn.Workload("hand", syn.MODE_POSITIONS, T=3, H=2, D=128, index_topk=5, S=100,
                      shared_cache=True, pos_lo=0, pos_hi=100, seed=0)
    inputs = syn.generate(wl)
    inputs["positions"] = np.array([9, 49, 19], np.int32)
    flops, sbytes, tbytes = bench.algorithmic(wl, inputs)
    assert flops == 2 * 2 * 128 * (10 + 50 + 20)
    assert sbytes == 3 * 2 * 128 * 2 + 3 * 2 * 4 + 50 * 128 * 2 + 3 * 100 * 4
    assert tbytes == 3 * 5 * 4


def test_workload_config_names_every_mode():
    for wl in _cases():
        c = bench.workload_config(wl)
        assert c["workload"] == wl.name and c["T"] == wl.T
        assert c["mask"] in ("positions", "causal", "compressed")
    assert "paged" in bench.workload_config(list(_cases())[-1])["caches"]
    for name in syn.WORKLOADS:
        assert name in bench.DEFAULTS
