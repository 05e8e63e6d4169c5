"""The multi-process (N > 1) host path of bench.py, on CPU with the gloo backend.

Each rank of a weak-scaling run is an independent replica; the only collectives are
the barriers around the timed region and the max over ranks of the measured time.
These tests run two ranks as processes and check that every rank agrees on the max,
that the whole-job value counts the work of all ranks over the slowest rank's time,
and that the reference arm prints exactly one line, from rank 0, under torchrun.
"""
import json
import os
import socket
import subprocess
import sys

import pytest
import torch
import torch.multiprocessing as mp

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
sys.path.insert(0, ROOT)

import bench  # noqa: E402


def free_port() -> int:
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _rank_main(rank, world, port, local_ms, queue):
    os.environ.update({"MASTER_ADDR": "127.0.0.1", "MASTER_PORT": str(port),
                       "RANK": str(rank), "WORLD_SIZE": str(world), "LOCAL_RANK": str(rank)})
    w, r, _ = bench.dist_env()
    dist = bench.init_dist(w, backend="gloo")
    try:
        bench.barrier(dist)
        ms = bench.max_over_ranks(local_ms[r], dist, torch.device("cpu"))
        bench.barrier(dist)
        # 1e12 FLOPs per rank per step, 10 steps
        value = bench.job_throughput(1e12, 10, w, ms, 1e12)
        queue.put((r, w, ms, value))
    finally:
        dist.destroy_process_group()


def test_two_ranks_agree_on_the_slowest_time_and_count_all_work():
    world = 2
    local_ms = [40.0, 50.0]          # rank 1 is the slower one
    ctx = mp.get_context("spawn")
    queue = ctx.Queue()
    port = free_port()
    procs = [ctx.Process(target=_rank_main, args=(r, world, port, local_ms, queue)) for r in range(world)]
    for p in procs:
        p.start()
    for p in procs:
        p.join(timeout=120)
        assert p.exitcode == 0
    got = sorted(queue.get(timeout=10) for _ in range(world))
    for r, (rank, w, ms, value) in enumerate(got):
        assert rank == r and w == world
        assert ms == 50.0
        # 2 ranks x 10 steps x 1 TFLOP in 50 ms
        assert value == pytest.approx(2 * 10 * 1.0 / 0.050)


def test_single_process_needs_no_process_group():
    assert bench.init_dist(1) is None
    assert bench.max_over_ranks(3.5, None, torch.device("cpu")) == 3.5
    bench.barrier(None)
    assert bench.job_throughput(2e9, 4, 1, 8.0, 1e9) == pytest.approx(2 * 4 / 0.008)


def test_reference_arm_under_torchrun_prints_one_line_from_rank_zero():
    port = free_port()
    cmd = [sys.executable, "-m", "torch.distributed.run", "--nnodes=1", "--nproc-per-node", "2",
           "--master-addr", "127.0.0.1", "--master-port", str(port), os.path.join(ROOT, "bench.py"),
           "--impl", "reference", "--workload", "tiny", "--gpus", "2", "--steps", "3", "--warmup", "3"]
    out = subprocess.run(cmd, capture_output=True, text=True, timeout=300, cwd=ROOT)
    assert out.returncode == 0, out.stderr[-2000:]
    lines = [ln for ln in out.stdout.splitlines() if ln.startswith("{")]
    assert len(lines) == 1
    rec = json.loads(lines[0])
    assert rec["impl"] == "reference"
    assert rec["n_gpus"] == 2
    assert rec["cpu_baseline"]["kind"] == "oracle"
    assert rec["e2e"]["h2d_bytes_per_step"] == 0 and rec["e2e"]["d2h_bytes_per_step"] == 0
