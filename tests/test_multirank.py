"""The multi-GPU path is replicas only (no exchange step): each rank runs its own decode and bench.py
combines the ranks' measurements. These CPU tests run that combination with world_size 2 over gloo:
the job time is the slowest rank's, bytes and tokens add up."""
import os
import socket
import sys

import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _free_port() -> int:
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _rank(rank: int, world: int, port: int, out):
    sys.path.insert(0, ROOT)
    import bench

    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        ms = [12.5, 20.25][rank]
        got = bench.reduce_over_ranks(dist, "cpu", ms, 1000.0 * (rank + 1), 8.0)
        single = bench.reduce_over_ranks(dist, "cpu", ms)
        out[rank] = (got, single)
    finally:
        dist.destroy_process_group()


def test_reduce_over_ranks_world2():
    port = _free_port()
    mgr = mp.get_context("spawn").Manager()
    out = mgr.dict()
    mp.start_processes(_rank, args=(2, port, out), nprocs=2, join=True, start_method="spawn")
    for rank in (0, 1):
        got, single = out[rank]
        assert got == (20.25, 3000.0, 16.0)  # max time, summed bytes and tokens, identical on every rank
        assert single == (20.25,)


def test_reduce_over_ranks_without_group():
    sys.path.insert(0, ROOT)
    import bench

    assert bench.reduce_over_ranks(None, "cpu", 3.0, 4.0, 5.0) == (3.0, 4.0, 5.0)
