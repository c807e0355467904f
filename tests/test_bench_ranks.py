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


def _dp_rank(rank: int, world: int, port: int, out):
    """Each rank: the oracle's adapter gradients on its token shard, then the same
    sum-all-reduce bench.py applies to its dA/dB bucket."""
    import numpy as np
    from bit_nf4_quantised_codebook_b200 import inputs
    from oracle import linear, nf4

    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), RANK=str(rank), WORLD_SIZE=str(world))
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        case = inputs.LinearCase("dp", M=64, N=128, K=192, r=16, alpha=16.0, w_std=0.02, a_std=0.05,
                                 b_std=0.05, seed=9)
        what = nf4.dequantize_nf4(nf4.quantize_nf4(case.W()))
        X, dY = case.X(), case.dY()
        sl = slice(rank * case.M // world, (rank + 1) * case.M // world)  # this rank's token shard
        g = linear.backward(X[sl], dY[sl], what, case.A(), case.B(), case.s)
        bucket = torch.tensor(np.concatenate([g["dA"].ravel(), g["dB"].ravel()]))
        dist.all_reduce(bucket)
        full = linear.backward(X, dY, what, case.A(), case.B(), case.s)
        out[rank] = (bucket.numpy(), np.concatenate([full["dA"].ravel(), full["dB"].ravel()]))
        dist.barrier()
    finally:
        dist.destroy_process_group()


def test_data_parallel_adapter_gradients_sum_over_shards():
    """The exchange step of the data-parallel bench: summing the shards' dA/dB gives
    the whole batch's gradients (they are sums over tokens)."""
    world = 2
    out = mp.Manager().dict()
    mp.spawn(_dp_rank, args=(world, _free_port(), out), nprocs=world, join=True)
    for r in range(world):
        got, full = out[r]
        assert got.shape == full.shape
        assert abs(got - full).max() <= 1e-12 * max(1.0, abs(full).max())
