"""The oracle's pins catch plausible mistakes (CPU).

Each case plants one mistake in a copy of the oracle's C source (a dropped
ReLU, an off-by-one mask, a wrong index, a wrong decoding constant, a
reversed tie rule, a wrong packed offset, a wrong compressed or paged
address, ...), builds the copy, and runs the pin tests against it: some pin
must fail. The sparse-MQA oracle (numpy) gets the same treatment against
its own pins. The copies live in the repository's unversioned _build
folder; the oracle in use is never touched.
"""
import os
import pathlib
import shutil
import subprocess
import sys
from concurrent.futures import ThreadPoolExecutor

import pytest

ROOT = pathlib.Path(__file__).resolve().parent.parent

# (what the mistake is, exact source text, its replacement)
MUTATIONS = [
    ("ReLU dropped", "double relu = x > 0.0 ? x : 0.0;", "double relu = x;"),
    ("|x| for ReLU", "double relu = x > 0.0 ? x : 0.0;", "double relu = x > 0.0 ? x : -x;"),
    ("mask exclusive of the position", "if (!(s <= last)) {", "if (!(s < last)) {"),
    ("causal mask off by one", "*last_valid = t - a;", "*last_valid = t - a - 1;"),
    ("key feature index shifted", "x += qrow[h * D + d] * krow[d];",
     "x += qrow[h * D + d] * krow[(d + 1) % D];"),
    ("head weight of head 0 for all", "I += (double)p->w[t * H + h] * relu;",
     "I += (double)p->w[t * H] * relu;"),
    ("wrong scale block", "scale[r * (D / ORC_MX_BLOCK) + d / ORC_MX_BLOCK]",
     "scale[r * (D / ORC_MX_BLOCK) + d % 4]"),
    ("e4m3 exponent bias 8", "mag = ldexp(1.0 + m / 8.0, e - 7);",
     "mag = ldexp(1.0 + m / 8.0, e - 8);"),
    ("e4m3 subnormal scale", "mag = ldexp((double)m, -9);", "mag = ldexp((double)m, -10);"),
    ("tie rule reversed", "return (x->s > y->s) - (x->s < y->s);",
     "return (x->s < y->s) - (x->s > y->s);"),
    ("padding 0 instead of -1", "out[j] = j < nvalid ? (int32_t)c[j].s : -1;",
     "out[j] = j < nvalid ? (int32_t)c[j].s : 0;"),
    ("packed causal offset", "*score_offset = base + (t - a) * L;",
     "*score_offset = base + (t - a) * (L + 1);"),
    ("compressed rule off by one", "(p->query_start + t + 1) / p->compress_ratio - 1;",
     "(p->query_start + t) / p->compress_ratio - 1;"),
    ("paged row within the page", "return page * p->page_size + s % p->page_size;",
     "return page * p->page_size + s / p->page_size;"),
]


# the sparse-MQA oracle (numpy), against its own pins
MQA_MUTATIONS = [
    ("sink left out", "denom = float(e.sum()) + float(np.exp(sinks[h] - m))",
     "denom = float(e.sum())"),
    ("sm_scale ignored", "logits = sm_scale * (keys @ q[b, s, h])", "logits = (keys @ q[b, s, h])"),
    ("negative indices kept", "if 0 <= int(j) < K]", "if int(j) < K]"),
    ("stability shift left out of the keys' terms", "e = np.exp(logits - m)",
     "e = np.exp(logits)"),
    ("first kept key dropped", "keys = kv[b, kept]", "keys = kv[b, kept[1:] or kept]"),
]


def _run_mutant(i, old, new, source="dsa_oracle.c", pins="test_oracle_pins.py"):
    d = ROOT / "_build" / "oracle_mutants" / f"{source}.{i}"
    shutil.rmtree(d, ignore_errors=True)
    d.mkdir(parents=True)
    for name in ("oracle", "dsa_synth"):
        shutil.copytree(ROOT / name, d / name,
                        ignore=shutil.ignore_patterns("*.so", "__pycache__"))
    (d / "tests").mkdir()
    for name in ("conftest.py", pins):
        shutil.copy(ROOT / "tests" / name, d / "tests" / name)
    shutil.copytree(ROOT / "tests" / "golden", d / "tests" / "golden")
    src = d / "oracle" / source
    text = src.read_text()
    assert text.count(old) == 1, f"mutation target not found once: {old}"
    src.write_text(text.replace(old, new))
    env = dict(os.environ, PYTHONPATH=str(d), OMP_NUM_THREADS="2")
    r = subprocess.run([sys.executable, "-m", "pytest", "-q", "-x", "-p", "no:cacheprovider",
                        f"tests/{pins}"], cwd=d, env=env,
                       capture_output=True, text=True, timeout=600)
    return r.returncode, r.stdout[-400:]


def test_every_planted_mistake_fails_a_pin():
    with ThreadPoolExecutor(max_workers=min(8, os.cpu_count() or 1)) as ex:
        results = list(ex.map(lambda a: _run_mutant(*a),
                              [(i, old, new) for i, (_, old, new) in enumerate(MUTATIONS)]))
    survivors = [what for (what, _, _), (rc, _) in zip(MUTATIONS, results) if rc == 0]
    assert not survivors, f"mistakes no pin catches: {survivors}"
    # a failing pin, not a broken build, must be what stops each mutant
    for (what, _, _), (rc, tail) in zip(MUTATIONS, results):
        assert rc == 1 and "failed" in tail, (what, rc, tail)


def test_every_planted_mistake_in_the_sparse_mqa_oracle_fails_a_pin():
    with ThreadPoolExecutor(max_workers=min(8, os.cpu_count() or 1)) as ex:
        results = list(ex.map(
            lambda a: _run_mutant(*a, source="sparse_mqa.py", pins="test_oracle_sparse_mqa.py"),
            [(i, old, new) for i, (_, old, new) in enumerate(MQA_MUTATIONS)]))
    survivors = [what for (what, _, _), (rc, _) in zip(MQA_MUTATIONS, results) if rc == 0]
    assert not survivors, f"mistakes no pin catches: {survivors}"
    for (what, _, _), (rc, tail) in zip(MQA_MUTATIONS, results):
        assert rc == 1 and "failed" in tail, (what, rc, tail)
