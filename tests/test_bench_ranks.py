"""Multi-process plumbing of bench.py on CPU (gloo, world size 2).

The path does not shard: with N processes every rank runs an independent
replica, the step time is the maximum over ranks and the reported throughput
is the work of all ranks over that time.  These tests cover that host logic
without a GPU.
"""
import os
import socket
import sys

import pytest
import torch.distributed as dist
import torch.multiprocessing as mp

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _worker(rank, world, port, out):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), RANK=str(rank), WORLD_SIZE=str(world))
    sys.path.insert(0, ROOT)
    import argparse
    import contextlib
    import io

    import bench

    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        ms = bench.max_over_ranks(10.0 + 5.0 * rank, "cpu")
        thr = bench.job_throughput(1000.0, world, ms)
        # the reference arm runs on rank 0 only: the other ranks return without work or output
        buf = io.StringIO()
        if rank != 0:
            with contextlib.redirect_stdout(buf):
                bench.run_reference(argparse.Namespace(workload="tiny", steps=1, warmup=3, ref_seconds=0.1))
        dist.barrier()
        out[rank] = (ms, thr, buf.getvalue())
    finally:
        dist.destroy_process_group()


def test_max_over_ranks_and_job_throughput_gloo():
    world = 2
    mgr = mp.get_context("spawn").Manager()
    out = mgr.dict()
    mp.start_processes(_worker, args=(world, _free_port(), out), nprocs=world, join=True, start_method="spawn")
    slowest = 10.0 + 5.0 * (world - 1)
    for r in range(world):
        ms, thr, printed = out[r]
        assert ms == pytest.approx(slowest)
        assert thr == pytest.approx(1000.0 * world / (slowest * 1e-3))
        if r != 0:
            assert printed == ""


def test_single_process_helpers():
    import bench
    assert bench.max_over_ranks(3.25, "cpu") == 3.25
    assert bench.job_throughput(500.0, 1, 2.0) == pytest.approx(250000.0)


def test_traffic_is_null_for_another_kernel_source(monkeypatch):
    import bench
    monkeypatch.setitem(bench.ATTN_TRAFFIC, "bytes_per_launch", 123)
    monkeypatch.setitem(bench.ATTN_TRAFFIC, "kernel_source_sha256", "0" * 64)
    assert bench.attn_traffic(bench.ATTN_TRAFFIC["workload"]) is None
    monkeypatch.setitem(bench.ATTN_TRAFFIC, "kernel_source_sha256", bench.kernel_source_sha256())
    assert bench.attn_traffic(bench.ATTN_TRAFFIC["workload"]) == 123
    assert bench.attn_traffic("another") is None
