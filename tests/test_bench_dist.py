"""The benchmark's multi-rank host path on CPU (gloo, world size 2): the
barrier, the max over ranks that defines the job's time, the weak-scaling
aggregate, and the reference arm launched the way the multi-GPU run launches
it (torchrun, one process per rank, rank 0 alone prints)."""

import json
import os
import socket
import subprocess
import sys

import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _worker(rank, world, port, out):
    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    sys.path.insert(0, ROOT)
    import datetime

    import bench
    dist.init_process_group("gloo", rank=rank, world_size=world, timeout=datetime.timedelta(seconds=60))
    try:
        local_ms = 2.0 + rank  # rank 1 is the slow one
        bench.rank_barrier(world)
        job_ms = bench.dist_max(local_ms, world, torch.device("cpu"))
        rate = bench.weak_scaling_rate(world, 1000, 10, job_ms)
        out.put((rank, job_ms, rate))
        bench.rank_barrier(world)
    finally:
        dist.destroy_process_group()


def test_max_over_ranks_and_weak_scaling_on_gloo():
    world = 2
    ctx = mp.get_context("spawn")
    out = ctx.Queue()
    port = _free_port()  # both ranks rendezvous on it
    procs = [ctx.Process(target=_worker, args=(r, world, port, out)) for r in range(world)]
    for p in procs:
        p.start()
    for p in procs:
        p.join(120)
        assert p.exitcode == 0
    results = sorted(out.get(timeout=10) for _ in range(world))
    for rank, job_ms, rate in results:
        assert job_ms == 3.0  # the slowest rank's time
        assert rate == pytest.approx(world * 1000 * 10 / 3.0e-3)


def test_single_rank_helpers_need_no_process_group():
    sys.path.insert(0, ROOT)
    import bench
    bench.rank_barrier(1)
    assert bench.dist_max(4.5, 1, torch.device("cpu")) == 4.5
    assert bench.weak_scaling_rate(1, 10, 5, 1000.0) == pytest.approx(50.0)


def test_reference_arm_under_torchrun_two_ranks():
    port = _free_port()
    cmd = [sys.executable, "-m", "torch.distributed.run", "--nnodes=1", "--nproc-per-node", "2",
           "--master-addr", "127.0.0.1", "--master-port", str(port),
           os.path.join(ROOT, "bench.py"), "--impl", "reference", "--gpus", "2", "--steps", "1", "--warmup", "3"]
    res = subprocess.run(cmd, capture_output=True, text=True, timeout=600, cwd=ROOT)
    assert res.returncode == 0, res.stderr[-2000:]
    lines = [ln for ln in res.stdout.splitlines() if ln.startswith("{")]
    assert len(lines) == 1, res.stdout
    rec = json.loads(lines[0])
    assert rec["impl"] == "reference"
    assert rec["n_gpus"] == 2 and rec["steps"] == 1 and rec["warmup"] == 3
    assert rec["value"] > 0 and rec["unit"] == "TFLOP/s"
    assert rec["e2e"]["h2d_bytes_per_step"] == 0
    assert rec["cpu_baseline"]["kind"] == "oracle"
