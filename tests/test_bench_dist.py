"""The multi-rank parts of bench.py on CPU: two gloo ranks, max-over-ranks
timing and whole-job aggregation (no GPU)."""
import os
import socket

import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp

import bench


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _rank(rank, world, port, out):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        ms = [3.0, 5.0][rank]  # the slower rank decides
        m = bench.reduce_max(ms, world, "cpu")
        bench.barrier(world)
        out[rank] = m
    finally:
        dist.destroy_process_group()


def test_two_rank_max_and_aggregate():
    world = 2
    out = mp.Manager().dict()
    mp.spawn(_rank, args=(world, _free_port(), out), nprocs=world, join=True)
    assert out[0] == out[1] == 5.0
    # each rank did its own 1e12-FLOP step; the job's rate uses the slowest rank
    assert bench.whole_job_tflops(1e12, world, 5.0) == pytest.approx(400.0)
    assert bench.whole_job_tflops(1e12, 1, 5.0) == pytest.approx(200.0)
