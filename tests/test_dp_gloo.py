"""The data-parallel path's host logic on CPU: two gloo ranks.

Each rank computes the adapter gradients of its own token shard with the oracle;
after the all-reduce both hold the full-batch gradient (sum over shards), and the
reported time is the slowest rank's.
"""
import os

import numpy as np
import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp

from diffusion_dit_b200 import dp


def _worker(rank, world, port, q):
    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        from oracle import fourtune_oracle as ora
        from tests.test_oracle_layer import _tiny_layer
        x, dy, layer = _tiny_layer(M=64, K=64, N=48, r_s=2, r=4, alpha=8.0)
        lo, hi = dp.token_shard(64, world, rank, multiple=16)
        res = ora.linear_bwd(x[lo:hi].contiguous(), dy[lo:hi].contiguous(), layer)
        da = torch.from_numpy(res.da.copy())
        db = torch.from_numpy(res.db.copy())
        dp.allreduce_adapter_grads(da, db)
        slow = dp.max_over_ranks(1.0 + rank, torch.device("cpu"))
        q.put((rank, da.numpy(), db.numpy(), slow))
    finally:
        dist.barrier()
        dist.destroy_process_group()


def test_two_rank_adapter_gradient_allreduce():
    world = 2
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = 29500 + (os.getpid() % 1000)
    procs = [ctx.Process(target=_worker, args=(r, world, port, q)) for r in range(world)]
    for p in procs:
        p.start()
    out = [q.get(timeout=120) for _ in range(world)]
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    from oracle import fourtune_oracle as ora
    from tests.test_oracle_layer import _tiny_layer
    x, dy, layer = _tiny_layer(M=64, K=64, N=48, r_s=2, r=4, alpha=8.0)
    full = ora.linear_bwd(x, dy, layer)
    for rank, da, db, slow in out:
        assert np.allclose(da, full.da, rtol=1e-12, atol=1e-14)
        assert np.allclose(db, full.db, rtol=1e-12, atol=1e-14)
        assert slow == 2.0


@pytest.mark.parametrize("m,world", [(4608, 8), (9216, 3), (256, 2), (1280, 7)])
def test_token_shards_cover_the_batch(m, world):
    spans = [dp.token_shard(m, world, r) for r in range(world)]
    assert spans[0][0] == 0 and spans[-1][1] == m
    for (a, b), (c, d) in zip(spans, spans[1:]):
        assert b == c and (b - a) % 128 == 0
    sizes = [b - a for a, b in spans]
    assert max(sizes) - min(sizes) <= 128


@pytest.mark.parametrize("world", [1, 2, 3, 4, 8])
def test_strong_scaling_shards_of_the_single_stream_batch(world):
    # bench.py --scaling strong: each rank takes a token shard of the 9216-token batch in
    # multiples of the pair GEMM's 256 rows, and the shards cover the batch once
    m = 9216
    spans = [dp.token_shard(m, world, r, multiple=256) for r in range(world)]
    assert spans[0][0] == 0 and spans[-1][1] == m
    for (a, b), (c, d) in zip(spans, spans[1:]):
        assert b == c
    assert all((b - a) % 256 == 0 and b > a for a, b in spans)
