#!/usr/bin/env python
"""Benchmark of the lightning indexer (scores + top-k) on B200.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--workload NAME]
                    [--impl ours|reference]

One step = one dsa_indexer_forward (score kernel + top-k kernel; packed
causal batches also run the one-CTA check of cu_seqlens) over one batch of
the workload, inputs resident in HBM. The default workload is the largest:
the packed ragged prefill (4 sequences of 4096/16384/32768/65536 tokens).
The forward is the top-k-only call (scores = NULL): the score rows are
written to the caller's workspace, the index set is the result. Steps are
replayed from CUDA graphs over several copies of the inputs, rotated so that
the bytes touched between two uses of a copy exceed twice the L2; the K timed
steps are replayed R times (R >= 1, so that the timed windows add up to about
half a second) and the median window is reported. Prints ONE JSON line
(rank 0).

Metric: valid query.key pairs per second (score + top-k); `roofline` gives
the dominant kernel's achieved fraction of the measured peak, `path_roofline`
the whole step's. `e2e` repeats the measurement through the API with pinned
host buffers and the host<->device copies inside the timed region.
`cpu_baseline` is the fp64 oracle on a bounded sample, on the host cores.
Multi-GPU (torchrun): every rank runs its own copy of the workload (weak
scaling, no collective on the data path); time = max over ranks.
"""
from __future__ import annotations

import argparse
import dataclasses
import datetime
import hashlib
import json
import os
import re
import subprocess
import sys
import time

import numpy as np

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

import dsa_synth as syn  # noqa: E402

METRIC = "indexer query·key pairs/s (score+top-k) at 1 B200, % of roofline"
UNIT = "pairs/s"
DEFAULTS = {   # steps, warmup, graph length
    "tiny_decode": (100000, 5000, 500),
    "decode_batch": (60000, 3000, 240),
    "decode_batch_paged": (60000, 3000, 240),
    "long_decode_fp8": (6000, 300, 60),
    "long_decode_fp8_paged": (6000, 300, 60),
    "prefill_causal": (1500, 30, 30),
    "ragged_prefill": (20, 3, 1),
    "c4_prefill": (1500, 30, 30),
}
L2_BYTES = 126 * 2**20


# ---------------------------------------------------------------- workload math
def row_positions(wl, inputs):
    """Last valid slot of each row before clamping to the row (decode-style
    rows): the token's position, or the last fully pooled slot."""
    if wl.mode == syn.MODE_POSITIONS:
        return np.asarray(inputs["positions"], np.int64)
    t = np.arange(wl.T, dtype=np.int64)
    return (wl.query_start + t + 1) // wl.compress_ratio - 1


def valid_pairs(wl, inputs) -> int:
    if wl.mode != syn.MODE_CAUSAL:
        return int(np.clip(row_positions(wl, inputs) + 1, 0, wl.S).sum())
    return int(sum(L * (L + 1) // 2 for L in wl.seqlens))


def score_elems(wl) -> int:
    if wl.mode != syn.MODE_CAUSAL:
        return wl.T * wl.S
    return int(sum(L * L for L in wl.seqlens))


def algorithmic(wl, inputs):
    """(flops, score-kernel bytes, top-k bytes) per step.

    Bytes: q (+scales) + w + key slots that some token may attend to (+scales)
    + the score write; top-k: its index write. The top-k's read of the score
    rows is an implementation cost and is not counted."""
    pairs = valid_pairs(wl, inputs)
    elt = 1 if wl.dtype == syn.DTYPE_FP8 else 2
    slot_bytes = wl.D * elt + (wl.D // 32 if wl.dtype == syn.DTYPE_FP8 else 0)
    q_bytes = wl.T * wl.H * slot_bytes
    w_bytes = wl.T * wl.H * 4
    if wl.mode != syn.MODE_CAUSAL:
        p = np.clip(row_positions(wl, inputs) + 1, 0, wl.S)
        shared = wl.shared_cache or wl.mode == syn.MODE_COMPRESSED
        k_slots = int(p.max()) if shared else int(p.sum())
    else:
        k_slots = wl.T
    score_bytes = q_bytes + w_bytes + k_slots * slot_bytes + score_elems(wl) * 4
    topk_bytes = wl.T * wl.index_topk * 4
    flops = 2.0 * wl.H * wl.D * pairs
    return flops, score_bytes, topk_bytes


def peaks():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    try:
        m = json.load(open(path))
        return dict(hbm=float(m["hbm_gbs"]), bf16=float(m["bf16_tflops"]),
                    bf16_sust=float(m["bf16_tflops_sustained"]), src="measured")
    except Exception:
        return dict(hbm=6650.0, bf16=1590.0, bf16_sust=1400.0, src="fallback")


def source_hash() -> str:
    h = hashlib.sha256()
    cs = os.path.join(ROOT, "sparse_attention_lightning_tcgen05_b200", "csrc")
    for f in sorted(os.listdir(cs)):
        h.update(open(os.path.join(cs, f), "rb").read())
    return h.hexdigest()[:16]


def profiled_traffic(workload: str, kernel: str = "score_kernel"):
    """DRAM bytes per launch of `kernel` on `workload` from the committed ncu
    summary (profiles/<kernel>_<workload>.md), or None when the summary is
    absent or the kernel sources changed since it was taken."""
    path = os.path.join(ROOT, "profiles", f"{kernel}_{workload}.md")
    if not os.path.exists(path):
        return None
    txt = open(path).read()
    mh = re.search(r"src_hash:\s*`?([0-9a-f]+)", txt)
    mb = re.search(r"dram_bytes_per_launch:\s*`?([0-9.eE+]+)", txt)
    if not mh or not mb or mh.group(1) != source_hash():
        return None
    return float(mb.group(1))


# ---------------------------------------------------------------- ranks
def dist_env():
    return (int(os.environ.get("RANK", "0")), int(os.environ.get("WORLD_SIZE", "1")),
            int(os.environ.get("LOCAL_RANK", "0")))


def init_dist(world: int, backend: str):
    if world <= 1:
        return None
    import torch.distributed as dist
    dist.init_process_group(backend, timeout=datetime.timedelta(seconds=120))
    return dist


def barrier(dist, device=None):
    if dist is not None:
        if device is not None:
            dist.barrier(device_ids=[device.index])
        else:
            dist.barrier()


def max_over_ranks(dist, value: float, device) -> float:
    """Largest `value` over all ranks (every rank calls this, in order)."""
    if dist is None:
        return value
    import torch
    t = torch.tensor([value], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


# ---------------------------------------------------------------- clocks
class ClockSampler:
    """nvidia-smi samples of SM clock and throttle reasons while running."""
    FIELDS = ("index,clocks.sm,clocks.max.sm,power.draw,utilization.gpu,"
              "clocks_event_reasons.hw_slowdown,"
              "clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,"
              "clocks_event_reasons.sw_power_cap")

    def __init__(self, gpu_id: str):
        self.gpu = gpu_id           # "GPU-<uuid>" (immune to index remapping)
        self.proc = None

    def __enter__(self):
        try:
            self.proc = subprocess.Popen(
                ["nvidia-smi", "-i", str(self.gpu), "--query-gpu=" + self.FIELDS,
                 "--format=csv,noheader,nounits", "-lms", "100"],
                stdout=subprocess.PIPE, stderr=subprocess.DEVNULL, text=True)
        except OSError:
            self.proc = None
        time.sleep(0.3)
        return self

    def __exit__(self, *exc):
        self.out = ""
        if self.proc is not None:
            time.sleep(0.15)
            self.proc.terminate()
            try:
                self.out, _ = self.proc.communicate(timeout=5)
            except subprocess.TimeoutExpired:
                self.proc.kill()
                self.out, _ = self.proc.communicate()

    def summary(self):
        rows = []
        for line in (self.out or "").strip().splitlines():
            f = [x.strip() for x in line.split(",")]
            if len(f) < 9:
                continue
            try:
                rows.append(dict(sm=float(f[1]), smax=float(f[2]),
                                 util=float(f[4]) if f[4] not in ("", "[N/A]") else 0.0,
                                 hw=f[5], hwt=f[6], swt=f[7], pcap=f[8]))
            except ValueError:
                continue
        if not rows:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": [], "samples": 0}
        loaded = [r for r in rows if r["util"] > 0] or rows
        reasons = set()
        for r in loaded:
            for key, name in (("hw", "hw_slowdown"), ("hwt", "hw_thermal_slowdown"),
                              ("swt", "sw_thermal_slowdown"), ("pcap", "sw_power_cap")):
                if r[key].lower().startswith("active"):
                    reasons.add(name)
        return {"sm_mhz": float(np.median([r["sm"] for r in loaded])),
                "sm_max_mhz": max(r["smax"] for r in rows),
                "reasons": sorted(reasons), "samples": len(loaded)}


# ---------------------------------------------------------------- our arm
def build_sets(wl, inputs, nsets, device):
    from sparse_attention_lightning_tcgen05_b200.problem import DeviceProblem
    return [DeviceProblem.from_workload(wl, inputs, device=device, topk_only=True)
            for _ in range(nsets)]


def capture(fn_list, stream):
    import torch
    g = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g, stream=stream):
        for fn in fn_list:
            fn()
    return g


def time_graphs(graphs, reps, stream, windows=1):
    """Replay graphs[0] `reps` times then graphs[1:] once, `windows` times
    in a row, each window bracketed by its own CUDA events; device ms of
    every window."""
    import torch
    ev = [torch.cuda.Event(enable_timing=True) for _ in range(windows + 1)]
    with torch.cuda.stream(stream):
        ev[0].record(stream)
        for w in range(windows):
            for _ in range(reps):
                graphs[0].replay()
            for g in graphs[1:]:
                g.replay()
            ev[w + 1].record(stream)
    ev[-1].synchronize()
    ms = [ev[i].elapsed_time(ev[i + 1]) for i in range(windows)]
    return ms if windows > 1 else ms[0]


def step_graphs(sets, which, steps, glen, stream):
    """Graphs that run `steps` steps in total (a main graph of `glen` steps,
    replayed, and a remainder graph)."""
    n = len(sets)
    calls = {"forward": lambda p: p.forward, "score": lambda p: p.score,
             "topk": lambda p: p.run_topk}[which]
    glen = max(1, min(glen, steps))
    main = capture([calls(sets[i % n]) for i in range(glen)], stream)
    rem = steps % glen
    extra = [capture([calls(sets[i % n]) for i in range(rem)], stream)] if rem else []
    return [main] + extra, steps // glen


def run_ours(args, wl, dist, rank, world, device):
    import torch
    from sparse_attention_lightning_tcgen05_b200 import DSA_OK
    torch.cuda.set_device(device)
    inputs = syn.generate(wl, seed=wl.seed + rank)
    flops, sbytes, tbytes = algorithmic(wl, inputs)
    pairs = valid_pairs(wl, inputs)
    per_set = sbytes
    nsets = 1 if per_set > 2 * L2_BYTES else int(np.ceil(2 * L2_BYTES / per_set)) + 1
    nsets = min(nsets, 8)
    sets = build_sets(wl, inputs, nsets, device)
    steps, warmup = args.steps, args.warmup
    glen = DEFAULTS.get(wl.name.split("[")[0], (0, 0, 32))[2]
    glen = (max(1, glen // nsets)) * nsets if glen >= nsets else glen
    stream = torch.cuda.Stream(device=device)

    # eager warm-up: sets kernel attributes, checks the device status
    with torch.cuda.stream(stream):
        for p in sets:
            p.forward(stream)
    for p in sets:
        st = p.device_status(stream)
        if st != DSA_OK:
            raise RuntimeError(f"device status {st} after warm-up")

    fwd, fwd_reps = step_graphs(sets, "forward", steps, glen, stream)
    wg, wreps = step_graphs(sets, "forward", max(warmup, 1), glen, stream)
    w_ms = time_graphs(wg, wreps, stream)                   # W warm-up steps
    # windows of K steps: enough of them for about half a second in total
    # (the same count on every rank)
    est = w_ms / max(warmup, 1) * steps
    windows = int(min(50, max(1, np.ceil(500.0 / max(est, 1e-3)))))
    windows = int(max_over_ranks(dist, float(windows), device))

    torch.cuda.synchronize(device)
    barrier(dist, device)
    torch.cuda.synchronize(device)
    uuid = str(torch.cuda.get_device_properties(device).uuid)
    with ClockSampler(uuid if uuid.startswith("GPU-") else "GPU-" + uuid) as clk:
        ms_w = time_graphs(fwd, fwd_reps, stream, windows)  # R windows of K steps
    torch.cuda.synchronize(device)
    barrier(dist, device)
    ms_w = [ms_w] if windows == 1 else ms_w
    ms = float(np.median(ms_w))
    ms_max = max_over_ranks(dist, ms, device)

    # the two kernels alone, same rotation, for the roofline
    rsteps = max(glen, min(steps, 4 * glen))
    sg, sreps = step_graphs(sets, "score", rsteps, glen, stream)
    tg, treps = step_graphs(sets, "topk", rsteps, glen, stream)
    time_graphs(sg, sreps, stream)
    ms_score = time_graphs(sg, sreps, stream) / rsteps
    ms_topk = time_graphs(tg, treps, stream) / rsteps
    for p in sets:
        st = p.device_status(stream)
        if st != DSA_OK:
            raise RuntimeError(f"device status {st} after timing")

    e2e = run_e2e(args, wl, inputs, sets[0], pairs, stream, device, dist)
    del fwd, wg, sg, tg
    return dict(ms_step=ms_max / steps, ms_local=ms / steps, ms_score=ms_score,
                ms_topk=ms_topk, flops=flops, sbytes=sbytes, tbytes=tbytes,
                pairs=pairs, nsets=nsets, clocks=clk.summary(), e2e=e2e,
                windows=windows, ms_windows=[m / steps for m in ms_w])


def run_e2e(args, wl, inputs, p, pairs, stream, device, dist):
    """Through the API with pinned host buffers: per step the inputs go
    host->device, the top-k-only forward runs (the score rows stay in the
    device workspace, for the consumer), the index set comes back."""
    import torch

    def pinned(x):
        if x is None:
            return None
        a = np.ascontiguousarray(x)
        if a.dtype == np.uint16:
            a = a.view(np.int16)
        return torch.from_numpy(a).pin_memory()
    host = {k: pinned(inputs.get(k)) for k in ("q", "q_scale", "w", "k", "k_scale",
                                                "positions", "cu_seqlens", "block_table")}
    dev = {"q": p.q, "q_scale": p.q_scale, "w": p.w, "k": p.k_cache,
           "k_scale": p.k_scale, "positions": p.positions, "cu_seqlens": p.cu_seqlens,
           "block_table": p.block_table}
    out_t = torch.empty(p.topk.shape, dtype=p.topk.dtype).pin_memory()
    h2d = sum(v.numel() * v.element_size() for v in host.values() if v is not None)
    d2h = out_t.numel() * 4
    n = args.e2e_steps

    def step():
        for k, v in host.items():
            if v is not None:
                dev[k].copy_(v, non_blocking=True)
        p.forward(stream)
        out_t.copy_(p.topk, non_blocking=True)

    with torch.cuda.stream(stream):
        for _ in range(2):
            step()
        torch.cuda.synchronize(device)
        barrier(dist, device)
        start = torch.cuda.Event(enable_timing=True)
        end = torch.cuda.Event(enable_timing=True)
        start.record(stream)
        for _ in range(n):
            step()
        end.record(stream)
    end.synchronize()
    ms = max_over_ranks(dist, start.elapsed_time(end), device)
    world = dist.get_world_size() if dist is not None else 1
    return {"value": pairs * n * world / (ms / 1e3), "unit": UNIT,
            "h2d_bytes_per_step": int(h2d), "d2h_bytes_per_step": int(d2h),
            "steps": n}


# ---------------------------------------------------------------- the oracle
def oracle_sample_rows(wl, inputs, pair_budget: int, start: int = 0):
    """Query rows, taken round-robin from `start`, until the sample holds
    about `pair_budget` valid pairs (at least one row)."""
    if wl.mode != syn.MODE_CAUSAL:
        nv = np.clip(row_positions(wl, inputs) + 1, 0, wl.S)
    else:
        cu = wl.cu_seqlens().astype(np.int64)
        nv = np.empty(wl.T, np.int64)
        for i in range(len(wl.seqlens)):
            nv[cu[i]:cu[i + 1]] = np.arange(1, wl.seqlens[i] + 1)
    # spread the sample over the workload: a fixed stride through the rows
    stride = max(1, wl.T // 64) if wl.T > 64 else 1
    order = np.concatenate([np.arange(o, wl.T, stride) for o in range(stride)])
    order = np.roll(order, -start)
    rows, total = [], 0
    for t in order:
        rows.append(int(t))
        total += int(nv[t])
        if total >= pair_budget:
            break
    return rows, total


def time_oracle(wl, inputs, rows, nthreads):
    import oracle
    P = oracle.Problem(wl, inputs)
    t0 = time.perf_counter()
    sc = P.scores(rows, nthreads=nthreads)
    P.topk(rows, sc, wl.index_topk, nthreads=nthreads)
    return time.perf_counter() - t0


def stratified_rows(wl, seed=0, n_random=512):
    """Packed causal batches: the first and last 16 rows of every sequence
    plus n_random seeded random rows (each row once)."""
    cu = wl.cu_seqlens().astype(np.int64)
    rows = set()
    for i in range(len(wl.seqlens)):
        a, b = int(cu[i]), int(cu[i + 1])
        rows.update(range(a, min(b, a + 16)))
        rows.update(range(max(a, b - 16), b))
    rng = np.random.default_rng(seed)
    rows.update(int(r) for r in rng.integers(0, wl.T, n_random))
    rows = sorted(rows)
    nv = np.empty(wl.T, np.int64)
    for i in range(len(wl.seqlens)):
        nv[cu[i]:cu[i + 1]] = np.arange(1, wl.seqlens[i] + 1)
    return rows, int(nv[rows].sum())


def cpu_baseline(wl, inputs, budget_s=15.0):
    """The oracle, as it is, on a bounded sample of the workload: the
    stratified row sample for a packed batch of several sequences, else rows
    spread over the workload up to about budget_s of work."""
    cores = os.cpu_count() or 1
    if wl.mode == syn.MODE_CAUSAL and len(wl.seqlens) > 1:
        rows, pairs = stratified_rows(wl)
        dt = time_oracle(wl, inputs, rows, cores)
        return {"value": pairs / dt, "unit": UNIT, "cores": cores, "kind": "oracle",
                "sample": f"{len(rows)} of {wl.T} query rows of {wl.name} (the first and "
                          f"last 16 rows of each sequence and 512 seeded random rows; "
                          f"{pairs} valid pairs), fp64 scores + top-k, {dt:.2f} s"}
    rows, pairs = oracle_sample_rows(wl, inputs, 2000)
    dt = time_oracle(wl, inputs, rows, cores)
    rate = pairs / max(dt, 1e-9)
    target = int(min(valid_pairs(wl, inputs), max(pairs, rate * budget_s * 0.5)))
    rows, pairs = oracle_sample_rows(wl, inputs, target)
    dt = time_oracle(wl, inputs, rows, cores)
    return {"value": pairs / dt, "unit": UNIT, "cores": cores, "kind": "oracle",
            "sample": f"{len(rows)} of {wl.T} query rows of {wl.name} ({pairs} valid "
                      f"pairs), fp64 scores + top-k, {dt:.2f} s"}


def run_reference(args, wl):
    """The fp64 oracle as the reference arm: each step scores and selects a
    bounded sample of rows, sized so that the whole run takes a few minutes."""
    inputs = syn.generate(wl)
    cores = os.cpu_count() or 1
    rows, pairs = oracle_sample_rows(wl, inputs, 2000)
    dt = time_oracle(wl, inputs, rows, cores)
    rate = pairs / max(dt, 1e-9)
    per_step_s = max(0.002, 150.0 / (args.steps + args.warmup))
    budget = int(max(1, rate * per_step_s))
    for i in range(args.warmup):
        r, _ = oracle_sample_rows(wl, inputs, budget, start=i)
        time_oracle(wl, inputs, r, cores)
    total_pairs, total_s, nrows = 0, 0.0, 0
    for i in range(args.steps):
        r, pr = oracle_sample_rows(wl, inputs, budget, start=args.warmup + i)
        total_s += time_oracle(wl, inputs, r, cores)
        total_pairs += pr
        nrows += len(r)
    value = total_pairs / total_s
    sample = (f"each step: {nrows / args.steps:.1f} of {wl.T} query rows of {wl.name} "
              f"(~{total_pairs // args.steps} valid pairs), fp64 scores + top-k")
    return {"metric": METRIC, "value": value, "unit": UNIT, "impl": "reference",
            "n_gpus": args.gpus, "steps": args.steps, "warmup": args.warmup,
            "ms_per_step": 1e3 * total_s / args.steps, "higher_is_better": True,
            "scaling": "weak", "vs_baseline": None, "dtype": "f64",
            "data": "synthetic", "config": workload_config(wl),
            "cpu_baseline": {"value": value, "unit": UNIT, "cores": cores,
                             "kind": "oracle", "sample": sample},
            "e2e": {"value": value, "unit": UNIT, "h2d_bytes_per_step": 0,
                    "d2h_bytes_per_step": 0}}


def workload_config(wl, extra=None):
    c = {"workload": wl.name, "T": wl.T, "H": wl.H, "D": wl.D,
         "index_topk": wl.index_topk,
         "kv_dtype": "fp8_e4m3+e8m0/32" if wl.dtype == syn.DTYPE_FP8 else "bf16",
         "mask": {syn.MODE_POSITIONS: "positions", syn.MODE_CAUSAL: "causal",
                  syn.MODE_COMPRESSED: "compressed"}[wl.mode]}
    if wl.mode == syn.MODE_POSITIONS:
        c.update(S=wl.S, positions=f"U[{wl.pos_lo},{wl.pos_hi})",
                 caches="shared" if wl.shared_cache else (
                     f"one per token, paged ({wl.page_size}-slot pages)" if wl.paged
                     else "one per token"))
    elif wl.mode == syn.MODE_COMPRESSED:
        c.update(S=wl.S, compress_ratio=wl.compress_ratio, query_start=wl.query_start,
                 caches="one pooled cache")
    else:
        c.update(seqlens=list(wl.seqlens))
    if extra:
        c.update(extra)
    return c


# ---------------------------------------------------------------- sparse MQA
MQA_METRIC = "sparse-MQA (query token, kept key) pairs/s at 1 B200, % of roofline"
MQA_DEFAULTS = {"mqa_decode": (20000, 1000, 200), "mqa_prefill": (200, 10, 10)}


def mqa_algorithmic(wl, idx):
    """(flops, bytes, kept entries) per step. FLOPs: 2*H*D for the logits and
    2*H*D for the weighted sum, per kept entry. Bytes: q, the index rows, the
    output, and every kv row some token of its batch selects, once."""
    kept = (idx >= 0) & (idx < wl.K)
    n_kept = int(kept.sum())
    uniq = sum(int(np.unique(idx[b][kept[b]]).size) for b in range(wl.B))
    T = wl.B * wl.S
    nbytes = T * wl.H * wl.D * 2 * 2 + idx.size * 4 + uniq * wl.D * 2
    return 4.0 * wl.H * wl.D * n_kept, nbytes, n_kept


def run_mqa(args, wl):
    import torch
    import sparse_attention_lightning_tcgen05_b200 as m
    from oracle.sparse_mqa import sparse_mqa
    device = torch.device("cuda", 0)
    torch.cuda.set_device(device)
    inputs = syn.generate_mqa(wl)
    flops, nbytes, n_kept = mqa_algorithmic(wl, inputs["idx"])
    T = wl.B * wl.S
    desc = m.make_mqa_desc(wl.B, wl.S, wl.H, wl.K, wl.K_top, wl.sm_scale)
    nsets = 1 if nbytes > 2 * L2_BYTES else min(8, int(np.ceil(2 * L2_BYTES / nbytes)) + 1)
    ws_bytes = m.dsa_sparse_mqa_workspace_size(desc)
    sets = []
    for _ in range(nsets):
        sets.append(dict(
            q=torch.from_numpy(inputs["q"].view(np.int16)).to(device),
            kv=torch.from_numpy(inputs["kv"].view(np.int16)).to(device),
            sinks=torch.from_numpy(inputs["sinks"]).to(device),
            idx=torch.from_numpy(inputs["idx"]).to(device),
            out=torch.empty((wl.B, wl.S, wl.H, wl.D), dtype=torch.int16, device=device),
            ws=torch.zeros(ws_bytes, dtype=torch.uint8, device=device)))
    stream = torch.cuda.Stream(device=device)

    def call(st):
        return lambda: m.dsa_sparse_mqa_forward(desc, st["q"], st["kv"], st["sinks"], st["idx"],
                                                st["out"], st["ws"], ws_bytes, stream.cuda_stream)
    with torch.cuda.stream(stream):
        for st in sets:
            call(st)()
    for st in sets:
        assert m.dsa_indexer_get_error(st["ws"], stream.cuda_stream) == m.DSA_OK
    glen = MQA_DEFAULTS[wl.name][2]
    glen = max(nsets, glen // nsets * nsets)
    steps, warmup = args.steps, args.warmup

    def graphs(n):
        main = capture([call(sets[i % nsets]) for i in range(min(glen, n))], stream)
        rem = n % min(glen, n)
        extra = [capture([call(sets[i % nsets]) for i in range(rem)], stream)] if rem else []
        return [main] + extra, n // min(glen, n)
    wg, wr = graphs(warmup)
    w_ms = time_graphs(wg, wr, stream)
    fg, fr = graphs(steps)
    windows = int(min(50, max(1, np.ceil(500.0 / max(w_ms / warmup * steps, 1e-3)))))
    uuid = str(torch.cuda.get_device_properties(device).uuid)
    torch.cuda.synchronize(device)
    with ClockSampler(uuid if uuid.startswith("GPU-") else "GPU-" + uuid) as clk:
        ms_w = time_graphs(fg, fr, stream, windows)
    ms_w = [ms_w] if windows == 1 else ms_w
    ms = float(np.median(ms_w)) / steps
    pk = peaks()
    t_flops = flops / (pk["bf16"] * 1e12)
    t_bytes = nbytes / (pk["hbm"] * 1e9)
    bound = "tensor" if t_flops >= t_bytes else "hbm"
    if bound == "tensor":
        roof = {"bound": "tensor", "achieved": flops / (ms / 1e3) / 1e12, "peak": pk["bf16"],
                "unit": "TFLOP/s"}
    else:
        roof = {"bound": "hbm", "achieved": nbytes / (ms / 1e3) / 1e9, "peak": pk["hbm"],
                "unit": "GB/s"}
    roof.update(frac=roof["achieved"] / roof["peak"],
                traffic=profiled_traffic(wl.name, "sparse_mqa_kernel"), kernel="sparse_mqa_kernel",
                roofline_ms=max(t_flops, t_bytes) * 1e3,
                peak_source=f"{pk['src']} (MEASURED_PEAKS.json)")
    # the fp64 oracle on a bounded sample of tokens
    cores = os.cpu_count() or 1
    rng = np.random.default_rng(0)
    toks = sorted(set(int(x) for x in rng.integers(0, T, min(T, 8))))
    t0 = time.perf_counter()
    for tk in toks:
        b, s_ = divmod(tk, wl.S)
        sparse_mqa(inputs["q"][b:b + 1, s_:s_ + 1], inputs["kv"][b:b + 1], inputs["sinks"],
                   inputs["idx"][b:b + 1, s_:s_ + 1], wl.sm_scale)
    dt = time.perf_counter() - t0
    kept_t = sum(int(((inputs["idx"].reshape(T, -1)[tk] >= 0) &
                      (inputs["idx"].reshape(T, -1)[tk] < wl.K)).sum()) for tk in toks)
    return {"metric": MQA_METRIC, "value": n_kept / (ms / 1e3), "unit": "pairs/s", "n_gpus": 1,
            "steps": steps, "warmup": warmup, "ms_per_step": ms, "higher_is_better": True,
            "scaling": "weak", "vs_baseline": None, "dtype": "bf16", "data": "synthetic",
            "config": {"workload": wl.name, "B": wl.B, "S": wl.S, "H": wl.H, "D": wl.D,
                       "K": wl.K, "K_top": wl.K_top, "causal_index_rows": wl.causal},
            "timing": {"l2": f"{nsets} rotating input copies" if nsets > 1
                       else "inputs larger than L2", "windows": windows,
                       "ms_per_step_windows": [x / steps for x in ms_w]},
            "kept_pairs_per_step": n_kept, "tflops": flops / (ms / 1e3) / 1e12,
            "roofline": roof, "clocks": clk.summary(),
            "gpu_launches": (2 if ws_bytes > 256 else 1) * steps * windows,
            "cpu_baseline": {"value": kept_t / dt, "unit": "pairs/s", "cores": 1,
                             "kind": "oracle",
                             "sample": f"{len(toks)} of {T} tokens (numpy fp64), {dt:.2f} s"}}


# ---------------------------------------------------------------- the front end
PREP_METRIC = "indexer front end (q, k, w projections) tokens/s at 1 B200, % of roofline"
PREP_DEFAULTS = {"prepare_decode": (20000, 1000, 200), "prepare_prefill": (200, 10, 10)}


def prep_algorithmic(wl):
    """(flops, bytes) per step: the three projections' multiply-adds; the
    weights, the activations and the outputs (q, k rows, w) moved once."""
    T, H, D = wl.T, wl.H, wl.D
    flops = 2.0 * T * (H * D * wl.q_lora_rank + (D + H) * wl.hidden)
    weights = 2 * (H * D * wl.q_lora_rank + (D + H) * wl.hidden)
    acts = 2 * T * (wl.hidden + wl.q_lora_rank)
    outs = T * (H * D * 2 + H * 4 + D * 2)
    return flops, weights + acts + outs


def run_prepare(args, wl):
    import torch
    import sparse_attention_lightning_tcgen05_b200 as m
    from oracle.front_end import front_end
    device = torch.device("cuda", 0)
    torch.cuda.set_device(device)
    inputs = syn.generate_prepare(wl)
    flops, nbytes = prep_algorithmic(wl)
    desc = m.make_prepare_desc(wl.T, wl.H, wl.hidden, wl.q_lora_rank, wl.rope_dim,
                               w_scale=wl.w_scale)
    ws_bytes = m.dsa_indexer_prepare_workspace_size(desc)
    nsets = 1 if nbytes > 2 * L2_BYTES else min(8, int(np.ceil(2 * L2_BYTES / nbytes)) + 1)

    def dev(a):
        a = np.ascontiguousarray(a)
        return torch.from_numpy(a.view(np.int16) if a.dtype == np.uint16 else a).to(device)
    sets = []
    for _ in range(nsets):
        st = {k: dev(inputs[k]) for k in ("x", "qr", "wq_b", "wk", "wp", "gain", "bias",
                                          "cos", "sin")}
        st.update(q=torch.empty((wl.T, wl.H, wl.D), dtype=torch.int16, device=device),
                  w=torch.empty((wl.T, wl.H), dtype=torch.float32, device=device),
                  k=torch.empty((wl.T, wl.D), dtype=torch.int16, device=device),
                  ws=torch.zeros(ws_bytes, dtype=torch.uint8, device=device))
        sets.append(st)
    stream = torch.cuda.Stream(device=device)

    def call(st):
        return lambda: m.dsa_indexer_prepare(desc, st["x"], st["qr"], st["wq_b"], st["wk"],
                                             st["wp"], st["gain"], st["bias"], st["cos"],
                                             st["sin"], None, st["q"], st["w"], st["k"],
                                             st["ws"], ws_bytes, stream.cuda_stream)
    with torch.cuda.stream(stream):
        for st in sets:
            call(st)()
    for st in sets:
        assert m.dsa_indexer_get_error(st["ws"], stream.cuda_stream) == m.DSA_OK
    glen = PREP_DEFAULTS[wl.name][2]
    glen = max(nsets, glen // nsets * nsets)
    steps, warmup = args.steps, args.warmup

    def graphs(n):
        g = min(glen, n)
        main = capture([call(sets[i % nsets]) for i in range(g)], stream)
        rem = n % g
        extra = [capture([call(sets[i % nsets]) for i in range(rem)], stream)] if rem else []
        return [main] + extra, n // g
    wg, wr = graphs(warmup)
    w_ms = time_graphs(wg, wr, stream)
    fg, fr = graphs(steps)
    windows = int(min(50, max(1, np.ceil(500.0 / max(w_ms / warmup * steps, 1e-3)))))
    uuid = str(torch.cuda.get_device_properties(device).uuid)
    torch.cuda.synchronize(device)
    with ClockSampler(uuid if uuid.startswith("GPU-") else "GPU-" + uuid) as clk:
        ms_w = time_graphs(fg, fr, stream, windows)
    ms_w = [ms_w] if windows == 1 else ms_w
    ms = float(np.median(ms_w)) / steps
    pk = peaks()
    t_flops = flops / (pk["bf16"] * 1e12)
    t_bytes = nbytes / (pk["hbm"] * 1e9)
    if t_flops >= t_bytes:
        roof = {"bound": "tensor", "achieved": flops / (ms / 1e3) / 1e12, "peak": pk["bf16"],
                "unit": "TFLOP/s"}
    else:
        roof = {"bound": "hbm", "achieved": nbytes / (ms / 1e3) / 1e9, "peak": pk["hbm"],
                "unit": "GB/s"}
    roof.update(frac=roof["achieved"] / roof["peak"], traffic=None, kernel="prep_gemm_kernel",
                roofline_ms=max(t_flops, t_bytes) * 1e3,
                peak_source=f"{pk['src']} (MEASURED_PEAKS.json)")
    # the fp64 oracle on a bounded sample of tokens
    rows = list(range(min(wl.T, 4)))
    t0 = time.perf_counter()
    sub = {k: (v[rows] if k in ("x", "qr", "cos", "sin") else v) for k, v in inputs.items()}
    front_end(sub["x"], sub["qr"], sub["wq_b"], sub["wk"], sub["wp"], sub["gain"], sub["bias"],
              sub["cos"], sub["sin"], H=wl.H, D=wl.D, rope_dim=wl.rope_dim, eps=1e-6,
              w_scale=wl.w_scale)
    dt = time.perf_counter() - t0
    return {"metric": PREP_METRIC, "value": wl.T / (ms / 1e3), "unit": "tokens/s", "n_gpus": 1,
            "steps": steps, "warmup": warmup, "ms_per_step": ms, "higher_is_better": True,
            "scaling": "weak", "vs_baseline": None, "dtype": "bf16", "data": "synthetic",
            "config": {"workload": wl.name, "T": wl.T, "H": wl.H, "D": wl.D,
                       "hidden": wl.hidden, "q_lora_rank": wl.q_lora_rank,
                       "rope_dim": wl.rope_dim},
            "timing": {"l2": f"{nsets} rotating input copies" if nsets > 1
                       else "inputs larger than L2", "windows": windows,
                       "ms_per_step_windows": [x / steps for x in ms_w]},
            "tflops": flops / (ms / 1e3) / 1e12, "roofline": roof, "clocks": clk.summary(),
            "cpu_baseline": {"value": len(rows) / dt, "unit": "tokens/s",
                             "cores": os.cpu_count() or 1, "kind": "oracle",
                             "sample": f"{len(rows)} of {wl.T} tokens (numpy fp64 matmuls), "
                                       f"{dt:.2f} s"}}


# ---------------------------------------------------------------- main
def main(argv=None):
    ap = argparse.ArgumentParser(description=__doc__.split("\n")[0])
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=None)
    ap.add_argument("--warmup", type=int, default=None)
    ap.add_argument("--workload", default="ragged_prefill",
                    choices=sorted(syn.WORKLOADS) + sorted(syn.MQA_WORKLOADS) +
                    sorted(syn.PREPARE_WORKLOADS))
    ap.add_argument("--impl", default="ours", choices=["ours", "reference"])
    ap.add_argument("--e2e-steps", type=int, default=None,
                    help="end-to-end steps (default 20; 5 for the ragged prefill)")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--seqlens", default=None,
                    help="packed causal workloads: other sequence lengths, comma "
                         "separated (a smaller batch of the same kind, for profiling)")
    args = ap.parse_args(argv)
    if args.workload in syn.PREPARE_WORKLOADS:
        wl = syn.PREPARE_WORKLOADS[args.workload]
        d_steps, d_warm, _ = PREP_DEFAULTS[wl.name]
        args.steps = d_steps if args.steps is None else args.steps
        args.warmup = d_warm if args.warmup is None else args.warmup
        if args.impl == "reference":
            print(json.dumps({"impl": "reference", "unavailable": "the oracle arm covers the "
                              "indexer workloads only"}), flush=True)
            return 0
        print(json.dumps(run_prepare(args, wl)), flush=True)
        return 0
    if args.workload in syn.MQA_WORKLOADS:
        wl = syn.MQA_WORKLOADS[args.workload]
        d_steps, d_warm, _ = MQA_DEFAULTS[wl.name]
        args.steps = d_steps if args.steps is None else args.steps
        args.warmup = d_warm if args.warmup is None else args.warmup
        if args.impl == "reference":
            print(json.dumps({"impl": "reference", "unavailable": "the oracle arm covers the "
                              "indexer workloads only"}), flush=True)
            return 0
        print(json.dumps(run_mqa(args, wl)), flush=True)
        return 0
    wl = syn.WORKLOADS[args.workload]
    if args.seqlens:
        if wl.mode != syn.MODE_CAUSAL:
            ap.error("--seqlens needs a packed causal workload")
        lens = tuple(int(x) for x in args.seqlens.split(","))
        wl = dataclasses.replace(wl, name=f"{wl.name}[{args.seqlens}]", seqlens=lens,
                                 T=sum(lens))
    d_steps, d_warm, _ = DEFAULTS[args.workload]
    args.steps = d_steps if args.steps is None else args.steps
    args.warmup = d_warm if args.warmup is None else args.warmup
    if args.e2e_steps is None:
        args.e2e_steps = 5 if args.workload == "ragged_prefill" else 20
    if args.steps < 1 or args.warmup < 3:
        ap.error("need --steps >= 1 and --warmup >= 3")
    rank, world, local_rank = dist_env()

    if args.impl == "reference":
        if rank == 0:
            print(json.dumps(run_reference(args, wl)), flush=True)
        return 0

    import torch
    device = torch.device("cuda", local_rank)
    torch.cuda.set_device(device)
    dist = init_dist(world, "nccl")
    try:
        r = run_ours(args, wl, dist, rank, world, device)
    finally:
        if dist is not None:
            dist.destroy_process_group()
    if rank != 0:
        return 0
    pk = peaks()
    value = r["pairs"] * world / (r["ms_step"] / 1e3)
    tensor_bound = wl.mode != syn.MODE_POSITIONS or wl.shared_cache
    fp8_ratio = 2.0 if wl.dtype == syn.DTYPE_FP8 else 1.0
    # a launch of tens of ms runs under the power cap like the seconds-long
    # GEMM loop of the sustained figure; shorter launches meet the burst one
    sustained = r["ms_score"] > 5.0
    if tensor_bound:
        peak_t = (pk["bf16_sust"] if sustained else pk["bf16"]) * fp8_ratio
        achieved = r["flops"] / (r["ms_score"] / 1e3) / 1e12
        roof = {"bound": "tensor", "achieved": achieved, "peak": peak_t, "unit": "TFLOP/s",
                "frac": achieved / peak_t,
                "peak_kind": ("sustained bf16" if sustained else "burst bf16") +
                             (" x 2 (fp8, nominal ratio)" if fp8_ratio > 1 else ""),
                "frac_of_burst": achieved / (pk["bf16"] * fp8_ratio)}
    else:
        achieved = r["sbytes"] / (r["ms_score"] / 1e3) / 1e9
        roof = {"bound": "hbm", "achieved": achieved, "peak": pk["hbm"], "unit": "GB/s",
                "frac": achieved / pk["hbm"]}
    traffic = profiled_traffic(wl.name)
    roof.update(traffic=traffic, kernel="score_kernel",
                kernel_ms=r["ms_score"], peak_source=f"{pk['src']} (MEASURED_PEAKS.json)"
                if pk["src"] == "measured" else "fallback")
    t_roof = max(r["flops"] / ((pk["bf16_sust"] if sustained else pk["bf16"]) * fp8_ratio
                               * 1e12),
                 (r["sbytes"] + r["tbytes"]) / (pk["hbm"] * 1e9))
    out = {
        "metric": METRIC, "value": value, "unit": UNIT, "n_gpus": world,
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": r["ms_step"],
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None,
        "dtype": "fp8" if wl.dtype == syn.DTYPE_FP8 else "bf16", "data": "synthetic",
        "config": workload_config(wl),
        "timing": {
            "l2": (f"{r['nsets']} rotating input copies" if r["nsets"] > 1
                   else "inputs larger than L2"),
            "steps_from": "CUDA graphs of top-k-only forward calls (scores in the workspace)",
            "windows": r["windows"],
            "ms_per_step_windows": r["ms_windows"],
            "reported": "median window of K steps",
            "parallelism": f"{world} independent replicas" if world > 1 else "1 GPU"},
        "valid_pairs_per_step": r["pairs"],
        "tflops": r["flops"] * world / (r["ms_step"] / 1e3) / 1e12,
        "roofline": roof,
        "path_roofline": {"roofline_ms": t_roof * 1e3, "step_ms": r["ms_step"],
                          "frac": t_roof * 1e3 / r["ms_step"],
                          "score_ms": r["ms_score"], "topk_ms": r["ms_topk"]},
        "clocks": r["clocks"], "e2e": r["e2e"],
        "gpu_launches": (3 if wl.mode == syn.MODE_CAUSAL else 2) * args.steps * r["windows"],
    }
    if world == 1 and not args.no_cpu_baseline:
        out["cpu_baseline"] = cpu_baseline(wl, syn.generate(wl))
    print(json.dumps(out), flush=True)
    return 0


if __name__ == "__main__":
    sys.exit(main())
