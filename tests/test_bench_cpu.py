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


def test_stratified_rows_cover_every_sequence_edge():
    """The CPU baseline's row sample of a packed causal batch: the first and
    last 16 rows of every sequence, seeded random rows, each row once, and
    the valid pairs of those rows (row i of a sequence sees i + 1 keys)."""
    wl = syn.Workload("c", syn.MODE_CAUSAL, T=5 + 40 + 100, H=4, D=128, index_topk=8,
                      seqlens=(5, 40, 100), seed=0)
    rows, pairs = bench.stratified_rows(wl, n_random=20)
    assert rows == sorted(set(rows))
    for a, L in ((0, 5), (5, 40), (45, 100)):
        edge = set(range(a, a + min(L, 16))) | set(range(a + max(0, L - 16), a + L))
        assert edge <= set(rows)
    assert all(0 <= r < wl.T for r in rows)
    P = oracle.Problem(wl, syn.generate(wl))
    want = 0
    for r in rows:
        _, L, last, _ = P.row_info(r)
        want += min(last + 1, L)
    assert pairs == want


def test_profiled_traffic_reads_only_a_current_summary(tmp_path, monkeypatch):
    """The `traffic` of a bench line comes from profiles/<kernel>_<workload>.md
    only when its src_hash is the sources' current hash."""
    monkeypatch.setattr(bench, "ROOT", str(tmp_path))
    (tmp_path / "profiles").mkdir()
    f = tmp_path / "profiles" / "score_kernel_w.md"
    f.write_text("# x\n\nsrc_hash: `abc123`\ndram_bytes_per_launch: `12345`\n")
    monkeypatch.setattr(bench, "source_hash", lambda: "abc123")
    assert bench.profiled_traffic("w") == 12345.0
    assert bench.profiled_traffic("missing") is None
    monkeypatch.setattr(bench, "source_hash", lambda: "def456")
    assert bench.profiled_traffic("w") is None
    g = tmp_path / "profiles" / "sparse_mqa_kernel_m.md"
    g.write_text("src_hash: `def456`\ndram_bytes_per_launch: `7`\n")
    assert bench.profiled_traffic("m", "sparse_mqa_kernel") == 7.0


def test_committed_profiles_name_their_sources_and_traffic():
    """Every committed summary states the source hash it was taken on and
    the DRAM bytes of one launch, in the form bench.py reads."""
    import re
    d = os.path.join(os.path.dirname(os.path.dirname(os.path.abspath(__file__))), "profiles")
    names = [n for n in os.listdir(d) if n.endswith(".md")]
    assert names
    for n in names:
        txt = open(os.path.join(d, n)).read()
        assert re.search(r"src_hash:\s*`[0-9a-f]{16}`", txt), n
        assert re.search(r"dram_bytes_per_launch:\s*`[0-9]+`", txt), n
        assert "--clock-control none" in txt, n
