"""bench.py's multi-rank plumbing on CPU with two gloo ranks: the barrier,
the max-over-ranks timing and the whole-job aggregate of N replicas, and the
reference arm's rule that only rank 0 runs and prints."""
import argparse
import datetime
import multiprocessing as mp
import os
import socket

import pytest

import bench


def _free_port() -> int:
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _worker(rank, world, port, q):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), RANK=str(rank), WORLD_SIZE=str(world))
    import torch.distributed as dist
    dist.init_process_group("gloo", rank=rank, world_size=world, timeout=datetime.timedelta(seconds=60))
    try:
        bench.barrier(world)
        ms = bench.max_over_ranks(1.5 * (rank + 1), world)   # rank r took 1.5 (r + 1) ms
        q.put((rank, ms, bench.whole_job_tflops(3.0e12, world, ms)))
        bench.barrier(world)
    finally:
        dist.destroy_process_group()


def test_two_ranks_max_timing_and_aggregate():
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_worker, args=(r, 2, port, q)) for r in range(2)]
    for p in procs:
        p.start()
    for p in procs:
        p.join(timeout=120)
    for p in procs:
        if p.is_alive():
            p.kill()
    assert [p.exitcode for p in procs] == [0, 0]
    got = sorted(q.get(timeout=5) for _ in range(2))
    for rank, ms, tflops in got:
        assert ms == 3.0                       # the slowest rank's time, on every rank
        assert tflops == pytest.approx(2 * 3.0e12 / 3.0e-3 / 1e12)   # both replicas' work over it


def test_single_rank_needs_no_process_group():
    assert bench.max_over_ranks(2.5, 1) == 2.5
    assert bench.whole_job_tflops(1e12, 1, 1.0) == pytest.approx(1000.0)


def test_reference_arm_runs_on_rank_zero_only(monkeypatch, capsys):
    monkeypatch.setenv("RANK", "1")
    monkeypatch.setenv("WORLD_SIZE", "2")
    args = argparse.Namespace(gpus=2, steps=2, warmup=1, impl="reference")
    assert bench.run_reference(args) == 0
    assert capsys.readouterr().out == ""
