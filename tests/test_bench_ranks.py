"""bench.py's multi-GPU path (replicas: one decoder per rank, no data-path collective), on CPU.

Two gloo ranks stand in for two GPUs: every rank must receive the largest
per-rank time, the job throughput counts all ranks' tokens over that time,
and the reference arm prints on rank 0 only.
"""
import json
import os
import socket
import subprocess
import sys

import pytest
import torch.multiprocessing as mp

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _rank(rank, world, port, q):
    import datetime

    import torch.distributed as dist

    sys.path.insert(0, ROOT)
    import bench

    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    dist.init_process_group("gloo", rank=rank, world_size=world, timeout=datetime.timedelta(seconds=60))
    try:
        ms = bench.max_over_ranks(10.0 + 5.0 * rank, dist, device="cpu")  # rank 1 is the slower one
        q.put((rank, ms, bench.job_throughput(world, 100, ms / 1e3)))
        dist.barrier()
    finally:
        dist.destroy_process_group()


def test_max_over_ranks_and_job_throughput_gloo():
    world, port = 2, _free_port()
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    procs = [ctx.Process(target=_rank, args=(r, world, port, q)) for r in range(world)]
    for p in procs:
        p.start()
    for p in procs:
        p.join(120)
        assert p.exitcode == 0
    got = sorted(q.get(timeout=10) for _ in range(world))
    for rank, ms, value in got:
        assert ms == 15.0  # both ranks see the slowest rank's time
        assert value == pytest.approx(2 * 100 / 0.015)  # all ranks' tokens over the slowest time


def test_single_rank_needs_no_process_group():
    sys.path.insert(0, ROOT)
    import bench

    assert bench.max_over_ranks(3.5) == 3.5
    assert bench.job_throughput(1, 10, 0.5) == 20.0


def test_reference_arm_prints_on_rank_zero_only():
    env = dict(os.environ, RANK="1", WORLD_SIZE="2", LOCAL_RANK="1")
    out = subprocess.run([sys.executable, os.path.join(ROOT, "bench.py"), "--impl", "reference", "--workload",
                          "tiny_dense_f32", "--steps", "1", "--warmup", "3"],
                         capture_output=True, text=True, env=env, timeout=300)
    assert out.returncode == 0, out.stderr
    assert out.stdout.strip() == ""
    env.update(RANK="0", LOCAL_RANK="0")
    out = subprocess.run([sys.executable, os.path.join(ROOT, "bench.py"), "--impl", "reference", "--workload",
                          "tiny_dense_f32", "--steps", "1", "--warmup", "3", "--cpu-budget-s", "1"],
                         capture_output=True, text=True, env=env, timeout=300)
    assert out.returncode == 0, out.stderr
    line = json.loads(out.stdout.strip().splitlines()[-1])
    assert line["impl"] == "reference" and line["value"] > 0 and line["cpu_baseline"]["kind"] == "oracle"


def test_tpot_stats_nearest_rank():
    sys.path.insert(0, ROOT)
    import bench

    st = bench.tpot_stats([3.0, 1.0, 2.0] + [2.0] * 97)  # ms per step
    assert st["p50"] == 2000.0 and st["max"] == 3000.0 and st["steps"] == 100
    assert st["p99"] == 2000.0  # nearest rank of 99 % of 100 steps
    assert bench.tpot_stats([]) is None
