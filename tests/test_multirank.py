"""The multi-GPU path shards tokens across ranks with no data-path exchange.
On CPU with two gloo ranks: the oracle evaluated on each rank's token shard
and gathered equals the single-process evaluation, and the bench's timing
reduction takes the maximum over ranks."""
import os
import socket

import numpy as np
import torch
import torch.distributed as dist
import torch.multiprocessing as mp

import bench
from oracle import moe_oracle as mo

T, D, KS, N, K, I = 24, 16, 1, 8, 2, 6


def layer():
    rng = np.random.default_rng(1)
    experts = [(rng.normal(size=(I, D)) * 0.3, rng.normal(size=(I, D)) * 0.3,
                rng.normal(size=(D, I)) * 0.3) for _ in range(KS + N)]
    return rng.normal(size=(T, D)), rng.normal(size=(N, D)) * 0.3, rng.normal(size=N) * 0.05, \
        experts


def run(x, w_r, b, experts):
    return mo.moe_forward(x, w_r, b, lambda e: experts[e], n_shared=KS, gate="sigmoid", top_k=K,
                          n_group=2, topk_group=1, renorm=True, route_scale=2.5)["h"]


def _rank(rank, world, port, out):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=world)
    x, w_r, b, experts = layer()
    lo, hi = bench.token_shard(T, rank, world)
    h = torch.from_numpy(run(x[lo:hi], w_r, b, experts))
    parts = [torch.zeros(bench.token_shard(T, r, world)[1] - bench.token_shard(T, r, world)[0], D,
                         dtype=torch.float64) for r in range(world)]
    dist.all_gather(parts, h)
    t = bench.max_over_ranks(float(rank + 1) * 1.5, "cpu")
    if rank == 0:
        out.put((torch.cat(parts).numpy(), t))
    dist.barrier()
    dist.destroy_process_group()


def free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def test_two_gloo_ranks_shard_tokens_exactly():
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = free_port()
    procs = [ctx.Process(target=_rank, args=(r, 2, port, q)) for r in range(2)]
    for p in procs:
        p.start()
    gathered, tmax = q.get(timeout=120)
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    x, w_r, b, experts = layer()
    # token independence: shards evaluate to the whole batch (up to BLAS blocking order)
    np.testing.assert_allclose(gathered, run(x, w_r, b, experts), rtol=1e-12, atol=1e-12)
    assert tmax == 3.0


def test_token_shards_cover_batch():
    for world in (1, 2, 3, 8):
        spans = [bench.token_shard(1001, r, world) for r in range(world)]
        assert spans[0][0] == 0 and spans[-1][1] == 1001
        assert all(a[1] == b[0] for a, b in zip(spans, spans[1:]))
