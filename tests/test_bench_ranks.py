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
    """Each rank: the oracle's adapter gradients of two linears on its token shard,
    written into bench.py's gradient bucket and summed by its all-reduce helper."""
    import numpy as np
    from bit_nf4_quantised_codebook_b200 import inputs
    from oracle import linear, nf4

    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), RANK=str(rank), WORLD_SIZE=str(world))
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        cases = [inputs.LinearCase("dp0", M=64, N=128, K=192, r=16, alpha=16.0, w_std=0.02, a_std=0.05,
                                   b_std=0.05, seed=9),
                 inputs.LinearCase("dp1", M=64, N=64, K=256, r=16, alpha=32.0, w_std=0.02, a_std=0.05,
                                   b_std=0.05, seed=19)]
        bucket, views = bench.grad_bucket([(c.K, c.r, c.N) for c in cases], torch.device("cpu"))
        want = []
        for c, (dA, dB) in zip(cases, views):
            what = nf4.dequantize_nf4(nf4.quantize_nf4(c.W()))
            X, dY = c.X(), c.dY()
            sl = slice(rank * c.M // world, (rank + 1) * c.M // world)  # this rank's token shard
            g = linear.backward(X[sl], dY[sl], what, c.A(), c.B(), c.s)
            dA.copy_(torch.from_numpy(g["dA"]))
            dB.copy_(torch.from_numpy(g["dB"]))
            full = linear.backward(X, dY, what, c.A(), c.B(), c.s)
            want.append((full["dA"], full["dB"]))
        bench.allreduce_grads(bucket)
        out[rank] = ([(dA.numpy().copy(), dB.numpy().copy()) for dA, dB in views], want)
        dist.barrier()
    finally:
        dist.destroy_process_group()


def test_data_parallel_adapter_gradients_sum_over_shards():
    """The exchange step of the data-parallel bench: bench.py's bucket of every
    linear's dA/dB, summed by its all-reduce helper, holds the whole batch's
    gradients (they are sums over tokens)."""
    world = 2
    out = mp.Manager().dict()
    mp.spawn(_dp_rank, args=(world, _free_port(), out), nprocs=world, join=True)
    for r in range(world):
        got, want = out[r]
        for (ga, gb), (wa, wb) in zip(got, want):
            assert ga.shape == wa.shape and gb.shape == wb.shape
            for g, w in ((ga, wa), (gb, wb)):
                assert abs(g - w).max() <= 1e-5 * max(1.0, abs(w).max())


def test_shards_differ_by_rank():
    """Every rank's X and dY come from their own seeds; rank 0 keeps the configuration's."""
    from bit_nf4_quantised_codebook_b200 import inputs
    c = inputs.LinearCase("dp", M=8, N=64, K=64, r=8, alpha=16.0, w_std=0.02, a_std=0.05, b_std=0.05, seed=3)
    c0, c1 = bench.shard_case(c, 0), bench.shard_case(c, 1)
    assert c0 is c
    assert bench.tensor_key("X", c1) != bench.tensor_key("X", c0)
    assert bench.tensor_key("dY", c1) != bench.tensor_key("dY", c0)
    assert (c1.M, c1.N, c1.K, c1.r, c1.s) == (c.M, c.N, c.K, c.r, c.s)
