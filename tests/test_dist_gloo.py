"""bench.py's multi-rank plumbing on CPU: world size 2 over gloo.

The decode path shards as independent replicas (one workload per GPU, no
data-path collective); the only collectives are the timing reductions, which
must give the max of the ranks' times and the sum of their bytes, and the
barriers around the timed region.  The reference arm runs on rank 0 only.
"""
import json
import multiprocessing as mp
import os
import socket
import subprocess
import sys

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _worker(rank, world, port, q):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), RANK=str(rank), WORLD_SIZE=str(world),
                      LOCAL_RANK=str(rank))
    sys.path.insert(0, ROOT)
    import bench

    try:
        dist = bench.init_dist(world, "gloo", rank)
        bench.barrier(dist)
        t_max = bench.max_over_ranks(10.0 * (rank + 1), dist)
        b_sum = bench.sum_over_ranks(1000.0 * (rank + 1), dist)
        bench.barrier(dist)
        q.put((rank, t_max, b_sum))
        dist.destroy_process_group()
    except Exception as e:  # report instead of hanging the parent
        q.put((rank, repr(e), None))


def test_timing_reductions_over_two_gloo_ranks():
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_worker, args=(r, 2, port, q)) for r in range(2)]
    for p in procs:
        p.start()
    results = sorted(q.get(timeout=120) for _ in range(2))
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    for rank, t_max, b_sum in results:
        assert t_max == 20.0, (rank, t_max)  # the slowest rank's time
        assert b_sum == 3000.0, (rank, b_sum)  # all ranks' bytes


def test_single_rank_needs_no_process_group():
    sys.path.insert(0, ROOT)
    import bench

    assert bench.init_dist(1, "gloo", 0) is None
    assert bench.max_over_ranks(3.5, None) == 3.5
    assert bench.sum_over_ranks(2.0, None) == 2.0


def _env(rank, world):
    env = dict(os.environ)
    env.update(RANK=str(rank), WORLD_SIZE=str(world), LOCAL_RANK=str(rank))
    return env


def test_reference_arm_prints_one_line_on_rank0_and_nothing_elsewhere():
    cmd = [sys.executable, os.path.join(ROOT, "bench.py"), "--impl", "reference", "--workload", "tiny",
           "--steps", "2", "--warmup", "1"]
    r0 = subprocess.run(cmd, capture_output=True, text=True, timeout=300, env=_env(0, 1))
    assert r0.returncode == 0, r0.stderr
    line = json.loads(r0.stdout.strip().splitlines()[-1])
    for key in ("metric", "value", "unit", "n_gpus", "steps", "warmup", "ms_per_step", "higher_is_better",
                "config", "impl", "cpu_baseline", "e2e"):
        assert key in line, key
    assert line["impl"] == "reference" and line["unit"] == "GB/s" and line["value"] > 0
    assert line["e2e"]["h2d_bytes_per_step"] == 0 and line["cpu_baseline"]["kind"] == "oracle"
    r1 = subprocess.run(cmd, capture_output=True, text=True, timeout=300, env=_env(1, 2))
    assert r1.returncode == 0 and r1.stdout.strip() == ""
