"""The multi-GPU bench path on CPU: two gloo ranks check the job-time and
whole-job-rate rules bench.py applies under torchrun (the layer does not shard,
so every rank runs its own replica and the slowest rank's time is the job's)."""
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


def _rank(rank: int, world: int, port: int, out):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), RANK=str(rank), WORLD_SIZE=str(world))
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        ms = 10.0 + 5.0 * rank  # rank 1 is the slow one
        job_ms = bench.max_over_ranks(ms, torch.device("cpu"))
        out[rank] = (job_ms, bench.whole_job_rate(2.0, world, job_ms * 1e-3))
        dist.barrier()
    finally:
        dist.destroy_process_group()


def test_two_rank_job_time_and_rate():
    world = 2
    out = mp.Manager().dict()
    mp.spawn(_rank, args=(world, _free_port(), out), nprocs=world, join=True)
    for r in range(world):
        job_ms, rate = out[r]
        assert job_ms == pytest.approx(15.0)                   # max over ranks, on every rank
        assert rate == pytest.approx(2.0 * world / 15e-3)      # replicas' work / slowest time
