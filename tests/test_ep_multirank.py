"""Expert parallelism across ranks on the CPU (gloo, world 2 and 4).

Each rank routes its own token shard, plans the dispatch with the product's
host logic (forward_moe_route_b200/ep.py), exchanges the row counts, the rows
and their gate weights through the product's torch.distributed transport,
evaluates the experts it holds on the rows it received, returns them, and
combines.  The routing and the expert arithmetic on each rank are the fp64
oracle's (this test has no GPU; on a GPU the same plan and transport drive
moe_dispatch_rows, moe_expert_ffn and moe_combine_rows, tested in
tests/test_gpu_ep.py).  The gathered outputs must equal the single-process
oracle's layer; per-expert row counts must add up exactly; with redundant
copies of the hottest experts the busiest rank processes fewer rows.
"""
import os
import socket

import numpy as np
import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp

import bench
from forward_moe_route_b200 import ep
from oracle import moe_oracle as mo

T, D, KS, N, K, I = 60, 16, 1, 8, 2, 6


def layer():
    rng = np.random.default_rng(7)
    experts = [(rng.normal(size=(I, D)) * 0.3, rng.normal(size=(I, D)) * 0.3,
                rng.normal(size=(D, I)) * 0.3) for _ in range(KS + N)]
    w_r = rng.normal(size=(N, D)) * 0.3
    w_r[:2] *= 2.5                                 # two hot experts
    return rng.normal(size=(T, D)), w_r, rng.normal(size=N) * 0.05, experts


def route(x, w_r, b):
    return mo.route(x, w_r, b, gate="sigmoid", top_k=K, n_group=2, topk_group=1, renorm=True,
                    route_scale=2.5)


def _rank(rank, world, port, n_redundant, out):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=world)
    x_all, w_r, b, experts = layer()
    lo, hi = bench.token_shard(T, rank, world)
    x = x_all[lo:hi]
    r = route(x, w_r, b)
    counts, offsets, perm_src, slot_of = mo.permutation(r["idx"], N)
    replicas = {}
    if n_redundant:
        loads = torch.tensor(counts, dtype=torch.int64)   # a copy: the reduce is in place
        dist.all_reduce(loads)                    # global per-expert load
        replicas = ep.choose_replicas(loads.numpy(), world, n_redundant)
    pl = ep.Placement(N, world, replicas)
    plan = ep.dispatch_plan(pl, counts, offsets, slot_of)
    tr = ep.Transport()
    recv_counts = tr.counts(plan.send_counts)
    n_slots = len(pl.slots(rank))
    recv_splits = [int(v) for v in recv_counts[:, :n_slots].sum(axis=1)]
    # send buffer in the plan's order (what moe_dispatch_rows writes on a GPU)
    R = len(slot_of)
    x_send = np.zeros((R, D))
    w_send = np.zeros(R)
    x_send[plan.row_of] = np.repeat(x, K, axis=0)
    w_send[plan.row_of] = r["w"].reshape(-1)
    x_recv = tr.all_to_all(torch.from_numpy(x_send), plan.send_splits, recv_splits).numpy()
    w_recv = tr.all_to_all(torch.from_numpy(w_send), plan.send_splits, recv_splits).numpy()
    rp = ep.receive_plan(pl, rank, recv_counts)
    assert rp.recv_splits == recv_splits
    y_recv = np.zeros_like(x_recv)
    for row0, rows, slot, out0 in rp.groups:
        j = pl.slots(rank)[slot]
        wg, wu, wd = experts[KS + j]
        y_recv[out0:out0 + rows] = w_recv[row0:row0 + rows, None] * \
            mo.swiglu_ffn(x_recv[row0:row0 + rows], wg, wu, wd)
    y_back = tr.all_to_all(torch.from_numpy(y_recv), recv_splits, plan.send_splits).numpy()
    # combine (what moe_combine_rows does on a GPU): residual, shared, then the K rows
    h = x.copy()
    for s in range(KS):
        h += mo.swiglu_ffn(x, *experts[s])
    for k in range(K):
        h += y_back[plan.row_of[np.arange(hi - lo) * K + k]]
    # gather outputs and per-slot loads on rank 0
    parts = [torch.zeros(bench.token_shard(T, q, world)[1] - bench.token_shard(T, q, world)[0], D,
                         dtype=torch.float64) for q in range(world)]
    dist.all_gather(parts, torch.from_numpy(h))
    slot_load = torch.zeros(world, pl.max_slots, dtype=torch.int64)
    slot_load[rank, :n_slots] = torch.as_tensor(rp.slot_rows)
    dist.all_reduce(slot_load)
    if rank == 0:
        out.put((torch.cat(parts).numpy(), slot_load.numpy(), {j: v for j, v in replicas.items()}))
    dist.barrier()
    dist.destroy_process_group()


def free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


@pytest.mark.parametrize("world,n_redundant", [(2, 0), (4, 0), (4, 2)])
def test_expert_parallel_layer_equals_single_process(world, n_redundant):
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = free_port()
    procs = [ctx.Process(target=_rank, args=(r, world, port, n_redundant, q))
             for r in range(world)]
    for p in procs:
        p.start()
    h, slot_load, replicas = q.get(timeout=180)
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    x, w_r, b, experts = layer()
    ref = route(x, w_r, b)
    want = mo.moe_forward(x, w_r, b, lambda e: experts[e], n_shared=KS, gate="sigmoid",
                          top_k=K, n_group=2, topk_group=1, renorm=True, route_scale=2.5)["h"]
    np.testing.assert_allclose(h, want, rtol=1e-12, atol=1e-12)
    # every expert's rows, summed over its holders, equal its global count exactly
    pl = ep.Placement(N, world, replicas)
    counts = np.bincount(ref["idx"].reshape(-1), minlength=N)
    got = np.zeros(N, np.int64)
    for r in range(world):
        for s, j in enumerate(pl.slots(r)):
            got[j] += slot_load[r, s]
    assert np.array_equal(got, counts)
    if n_redundant:
        plain = ep.Placement(N, world)
        per_rank_plain = [sum(counts[j] for j in plain.slots(r)) for r in range(world)]
        assert slot_load.sum(axis=1).max() < max(per_rank_plain)
