"""The multi-process path of bench.py (one process per GPU under torchrun), on CPU.

Two gloo ranks rendezvous through the same environment torchrun provides, take the
slowest rank's time and compute the whole-job throughput the way the CUDA arm does; the
reference arm's non-zero ranks exit without work or output. No GPU is used.
"""
from __future__ import annotations

import os
import socket
import subprocess
import sys

import pytest
import torch
import torch.multiprocessing as mp

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _free_port() -> int:
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _rank_main(rank: int, world: int, port: int, out):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), RANK=str(rank),
                      WORLD_SIZE=str(world), LOCAL_RANK=str(rank))
    sys.path.insert(0, ROOT)
    import bench
    dist, r, w = bench._dist(backend="gloo")
    try:
        dist.barrier()
        ms = bench._max_over_ranks(dist, 10.0 + 3.0 * r, torch.device("cpu"))   # rank 1 is slower
        value = bench._job_tflops(w, 2.0e12, ms)
        dist.barrier()
        out.put((r, w, ms, value))
    finally:
        dist.destroy_process_group()


def test_two_ranks_take_the_slowest_time_and_sum_the_work():
    ctx = mp.get_context("spawn")
    out = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_rank_main, args=(r, 2, port, out)) for r in range(2)]
    for p in procs:
        p.start()
    results = [out.get(timeout=120) for _ in procs]
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    results.sort()
    assert [r[0] for r in results] == [0, 1] and all(r[1] == 2 for r in results)
    for _, _, ms, value in results:
        assert ms == pytest.approx(13.0)                       # max over ranks
        assert value == pytest.approx(2 * 2.0e12 / 13.0e-3 / 1e12)   # both replicas' work / slowest time


def test_single_process_needs_no_group():
    sys.path.insert(0, ROOT)
    import bench
    assert bench._max_over_ranks(None, 4.5, torch.device("cpu")) == 4.5
    assert bench._job_tflops(1, 1.0e12, 1000.0) == pytest.approx(1.0)


def test_reference_arm_runs_on_rank_zero_only():
    env = dict(os.environ, RANK="1", WORLD_SIZE="2", LOCAL_RANK="1", MASTER_ADDR="127.0.0.1", MASTER_PORT="1")
    r = subprocess.run([sys.executable, os.path.join(ROOT, "bench.py"), "--impl", "reference", "--gpus", "2",
                        "--steps", "1", "--warmup", "0"], env=env, capture_output=True, text=True, timeout=300)
    assert r.returncode == 0, r.stderr[-2000:]
    assert r.stdout.strip() == ""
