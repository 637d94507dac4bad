"""The multi-rank host logic of bench.py, on CPU ranks (gloo, world size 2).

Under torchrun every rank runs its own replica of the step (weak scaling, no
collective in the data path); the job time is the slowest rank's time and the
job throughput counts every rank's bytes.  These tests run two gloo ranks as
processes on the host and check both rules.
"""
import os
import socket
import sys

import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
sys.path.insert(0, ROOT)

import bench  # noqa: E402


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _rank_main(rank, world, port, out):
    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        local_ms = 10.0 + 5.0 * rank          # rank 1 is the slow one
        job_ms = bench.max_over_ranks(local_ms, dist)
        dist.barrier()
        out[rank] = job_ms
    finally:
        dist.destroy_process_group()


def test_job_time_is_the_max_over_ranks():
    world = 2
    port = _free_port()
    out = mp.get_context("spawn").Manager().dict()
    mp.start_processes(_rank_main, args=(world, port, out), nprocs=world, start_method="spawn", join=True)
    assert dict(out) == {0: 15.0, 1: 15.0}


def test_single_process_job_time_is_local():
    assert bench.max_over_ranks(12.5, None) == 12.5


@pytest.mark.parametrize("world", [1, 2, 4, 8])
def test_job_throughput_counts_every_rank(world):
    # 1 GB per rank per step in 1 ms -> 1000 GB/s per rank
    assert bench.job_throughput(1e9, world, 1.0) == pytest.approx(1000.0 * world)
