"""Head sharding plumbing on CPU: the head partition and the all-gather of the ranks'
output blocks (gloo, 2 ranks).  The attention itself is covered on the GPU by
tests/test_gpu_sharding.py."""
import os
import socket
import sys

import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)

from head_wise_dynamic_b200.sharding import gather_heads, head_range  # noqa: E402


def test_head_range_partitions_the_heads():
    for H, world in [(16, 1), (16, 2), (16, 4), (16, 8), (4, 4)]:
        seen = []
        for r in range(world):
            h0, h1 = head_range(H, world, r)
            assert h1 - h0 == H // world
            seen += list(range(h0, h1))
        assert seen == list(range(H))
    with pytest.raises(ValueError):
        head_range(16, 3, 0)
    with pytest.raises(ValueError):
        head_range(16, 2, 2)


def test_gather_without_process_group_copies():
    local = torch.arange(24, dtype=torch.float32).reshape(2, 3, 4)
    full = torch.zeros_like(local)
    gather_heads(local, full)
    assert torch.equal(full, local)


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _worker(rank, world, port, out):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), RANK=str(rank), WORLD_SIZE=str(world))
    sys.path.insert(0, ROOT)
    from head_wise_dynamic_b200.sharding import gather_heads as gh, head_range as hr
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        H, N = 8, 5
        h0, h1 = hr(H, world, rank)
        # every rank's block holds its own head indices: the gather must put them in head order
        local = torch.arange(h0, h1, dtype=torch.float32).reshape(-1, 1, 1).repeat(1, N, 4) + 0.5
        full = torch.zeros((H, N, 4))
        gh(local, full)
        out[rank] = full.clone()
    finally:
        dist.destroy_process_group()


def test_gather_heads_gloo_two_ranks():
    world = 2
    mgr = mp.get_context("spawn").Manager()
    out = mgr.dict()
    mp.start_processes(_worker, args=(world, _free_port(), out), nprocs=world, join=True, start_method="spawn")
    want = torch.arange(8, dtype=torch.float32).reshape(8, 1, 1).repeat(1, 5, 4) + 0.5
    for r in range(world):
        assert torch.equal(out[r], want)
