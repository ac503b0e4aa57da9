"""Multi-rank logic of bench.py on CPU: two gloo ranks, no GPU.

Each replica runs the same work; the job's time is the slowest rank's and its
throughput counts the units of every rank.
"""
import os
import socket

import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp

import bench


def _free_port() -> int:
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _worker(rank, world, port, out):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        ms = 1.5 + rank  # rank 1 is the slow one
        ms_max = bench.max_over_ranks(dist, ms, torch.device("cpu"))
        dist.barrier()
        out[rank] = (ms_max, bench.job_rate(100.0, world, ms_max))
    finally:
        dist.destroy_process_group()


def test_max_over_ranks_gloo_two_ranks():
    world = 2
    mgr = mp.get_context("spawn").Manager()
    out = mgr.dict()
    mp.start_processes(_worker, args=(world, _free_port(), out), nprocs=world, join=True, start_method="spawn")
    assert sorted(out.keys()) == [0, 1]
    for r in range(world):
        ms_max, rate = out[r]
        assert ms_max == 2.5
        assert rate == pytest.approx(100.0 * world / 2.5e-3)


def test_single_process_identity():
    assert bench.max_over_ranks(None, 3.25, None) == 3.25
    assert bench.job_rate(64, 1, 2.0) == pytest.approx(32000.0)
