"""Host logic of the multi-rank bench path, on CPU with the gloo backend (world size 2).

Each rank runs its own replica of the workload (the path partitions by
sequence, so there is no data-path collective); the job's throughput is the
units all ranks processed divided by the slowest rank's time. These tests run
that aggregation and the reference arm's rank gating in two processes.
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


def _rank_main(rank, world, port, local_ms, q):
    import torch.distributed as dist
    sys.path.insert(0, ROOT)
    import bench
    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        value, max_ms = bench.job_throughput(local_ms[rank], world, 1.0e9, 10, 1e9, dist, "cpu")
        q.put((rank, value, max_ms))
    finally:
        dist.barrier()
        dist.destroy_process_group()


def test_job_throughput_takes_the_slowest_rank():
    world, port = 2, _free_port()
    local_ms = [40.0, 50.0]   # rank 1 is slower
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    procs = [ctx.Process(target=_rank_main, args=(r, world, port, local_ms, q)) for r in range(world)]
    for p in procs:
        p.start()
    for p in procs:
        p.join(timeout=120)
        assert p.exitcode == 0
    got = sorted(q.get(timeout=10) for _ in range(world))
    for rank, value, max_ms in got:
        assert max_ms == 50.0
        # 2 ranks x 1e9 units x 10 steps in 50 ms -> 4e11 units/s -> 400 in units of 1e9
        assert value == pytest.approx(400.0)


def test_job_throughput_single_rank():
    sys.path.insert(0, ROOT)
    import bench
    value, max_ms = bench.job_throughput(20.0, 1, 5.0e8, 4, 1e9)
    assert max_ms == 20.0
    assert value == pytest.approx(100.0)


def test_reference_arm_runs_on_rank_zero_only():
    # a non-zero rank of the reference arm prints nothing and exits 0
    env = dict(os.environ, RANK="1", WORLD_SIZE="2", LOCAL_RANK="1")
    r = subprocess.run([sys.executable, os.path.join(ROOT, "bench.py"), "--impl", "reference", "--workload",
                        "tiny_prefill_f32", "--steps", "1", "--warmup", "1"],
                       capture_output=True, text=True, env=env, timeout=300)
    assert r.returncode == 0
    assert r.stdout.strip() == ""


def test_reference_arm_line_on_rank_zero():
    env = dict(os.environ, RANK="0", WORLD_SIZE="1", LOCAL_RANK="0")
    r = subprocess.run([sys.executable, os.path.join(ROOT, "bench.py"), "--impl", "reference", "--workload",
                        "tiny_prefill_f32", "--steps", "1", "--warmup", "1"],
                       capture_output=True, text=True, env=env, timeout=300)
    assert r.returncode == 0, r.stderr[-2000:]
    line = json.loads([l for l in r.stdout.splitlines() if l.startswith("{")][-1])
    assert line["impl"] == "reference"
    assert line["value"] > 0 and line["unit"] == "TFLOP/s"
    assert line["cpu_baseline"]["kind"] == "oracle"
    assert line["e2e"]["h2d_bytes_per_step"] == 0
