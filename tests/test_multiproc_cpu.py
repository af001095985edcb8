"""The multi-rank plumbing of bench.py on the CPU (gloo, world size 2).

With N GPUs bench.py runs one independent replica of the workload per rank
(no collective on the data path); the ranks only meet in barriers and in one
all-reduce MAX of their device times, and rank 0 alone prints. These tests
run exactly those helpers, and the reference arm's rank-0-only rule, in two
CPU processes rendezvousing on 127.0.0.1.
"""
import json
import os
import socket
import subprocess
import sys

import torch.multiprocessing as mp

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def free_port() -> int:
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _rank_main(rank, world, port, out):
    os.environ.update(RANK=str(rank), WORLD_SIZE=str(world), LOCAL_RANK=str(rank),
                      MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    sys.path.insert(0, ROOT)
    import bench
    r, w, lr = bench.dist_env()
    dist = bench.init_dist(w, "gloo")
    try:
        bench.barrier(dist)
        # each rank "measured" a different time; every rank gets the largest
        got = bench.max_over_ranks(dist, 1.5 + rank, "cpu")
        bench.barrier(dist)
    finally:
        dist.destroy_process_group()
    out.put((r, w, lr, got))


def test_ranks_agree_on_the_max_device_time():
    world, port = 2, free_port()
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    procs = [ctx.Process(target=_rank_main, args=(r, world, port, q)) for r in range(world)]
    for p in procs:
        p.start()
    res = sorted(q.get(timeout=120) for _ in range(world))
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    assert [x[0] for x in res] == [0, 1]
    assert all(x[1] == world and x[2] == x[0] for x in res)
    assert all(x[3] == 1.5 + (world - 1) for x in res)


def test_single_rank_needs_no_process_group():
    sys.path.insert(0, ROOT)
    import bench
    assert bench.init_dist(1, "gloo") is None
    assert bench.max_over_ranks(None, 3.25, "cpu") == 3.25


def _reference_arm(rank, world):
    env = dict(os.environ, RANK=str(rank), WORLD_SIZE=str(world), LOCAL_RANK=str(rank),
               MASTER_ADDR="127.0.0.1", MASTER_PORT=str(free_port()))
    return subprocess.run(
        [sys.executable, os.path.join(ROOT, "bench.py"), "--impl", "reference", "--gpus",
         str(world), "--workload", "tiny_decode", "--steps", "3", "--warmup", "3"],
        env=env, capture_output=True, text=True, timeout=300, cwd=ROOT)


def test_reference_arm_prints_on_rank_zero_only():
    r1 = _reference_arm(1, 2)
    assert r1.returncode == 0, r1.stderr
    assert r1.stdout.strip() == ""
    r0 = _reference_arm(0, 2)
    assert r0.returncode == 0, r0.stderr
    line = json.loads(r0.stdout.strip().splitlines()[-1])
    assert line["impl"] == "reference" and line["n_gpus"] == 2
    assert line["value"] > 0 and line["cpu_baseline"]["kind"] == "oracle"
    assert line["e2e"]["h2d_bytes_per_step"] == 0
