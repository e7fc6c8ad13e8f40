"""Expert parallelism through the CUDA path, with W ranks emulated on one GPU.

Each emulated rank owns a shard of the batch and the experts of its
placement (forward_moe_route_b200/ep.py).  The phases run rank by rank --
dispatch (moe_route, moe_permute maps, moe_dispatch_rows), expert compute
(moe_expert_ffn on the received rows), combine (moe_expert_ffn for the shared
experts, moe_combine_rows) -- and the all-to-all between them is a plain
exchange of device tensors here (on several GPUs it is torch.distributed).
No kernel waits on another rank.

The expert rows are computed by the same GEMMs with the same operands, the
gate weights are the same fp32 values and the combine adds in the same order,
so the gathered outputs must equal moe_forward over the whole batch bit for
bit, with and without redundant copies of the hottest experts.
"""
import dataclasses

import numpy as np
import pytest
import torch

import bench
import forward_moe_route_b200 as moe
from forward_moe_route_b200 import ep
from synth import recipes

pytestmark = pytest.mark.gpu


def emulate(cfg, inp, pl):
    W = pl.world
    shards = [bench.token_shard(cfg.T, r, W) for r in range(W)]
    descs, steps, xs = [], [], []
    for r, (lo, hi) in enumerate(shards):
        c = dataclasses.replace(cfg, T=hi - lo)
        d = moe.desc_from_config(c)
        x = inp["x"][lo:hi].contiguous()
        descs.append(d)
        xs.append(x)
        steps.append(ep.ep_dispatch(d, pl, r, x, inp["w_r"], inp["bias"]))
    # exchange: counts, then rows and weights
    send_counts = np.stack([s.plan.send_counts for s in steps])          # [src, dst, slot]
    recv_counts = [send_counts[:, q, :] for q in range(W)]               # [src, slot]

    def a2a(bufs, splits):
        """bufs[s] split by splits[s] -> per destination the concatenation over sources."""
        parts = [torch.split(b, sp) for b, sp in zip(bufs, splits)]
        return [torch.cat([parts[s][q] for s in range(W)]) for q in range(W)]

    send_splits = [s.plan.send_splits for s in steps]
    x_recv = a2a([s.x_send for s in steps], send_splits)
    w_recv = a2a([s.w_send for s in steps], send_splits)
    fp8 = cfg.dtype == "e4m3"
    s_recv = a2a([s.s_send for s in steps], send_splits) if fp8 else [None] * W
    full = (inp["w_gu"], inp["w_down"]) + ((inp["w_gu_scale"], inp["w_down_scale"]) if fp8 else ())
    weights = [ep.local_weights(pl, r, cfg.n_shared, *full) for r in range(W)]
    scales = [wt[2:] if fp8 else (None, None) for wt in weights]
    ys = [ep.ep_compute(descs[r], pl, steps[r], recv_counts[r], x_recv[r], w_recv[r],
                        *weights[r][:2], s_recv[r], *scales[r]) for r in range(W)]
    recv_splits = [s.recv.recv_splits for s in steps]
    y_back = a2a(ys, recv_splits)
    hs = [ep.ep_combine(descs[r], steps[r], xs[r], None, y_back[r], *weights[r][:2], *scales[r])
          for r in range(W)]
    loads = [int(sum(s.recv.recv_splits)) for s in steps]
    return torch.cat(hs), loads


def reference(cfg, inp):
    desc = moe.desc_from_config(cfg)
    ws = moe.workspace(desc)
    h = torch.empty(cfg.T, cfg.d, dtype=torch.bfloat16, device="cuda")
    counts = torch.empty(cfg.n_routed, dtype=torch.int32, device="cuda")
    moe.moe_forward(desc, inp["x"], None, inp["w_r"], inp["bias"], inp["w_gu"],
                    inp.get("w_gu_scale"), inp["w_down"], inp.get("w_down_scale"), h, None,
                    counts, ws)
    return h, counts.cpu().numpy()


def fp8_inputs(cfg):
    """The layer's inputs with the expert weights quantised 128x128 to E4M3."""
    inp = recipes.device_inputs(cfg)
    E, I, d = cfg.n_experts, cfg.inter, cfg.d
    gq = torch.empty(E, 2 * I, d, dtype=torch.uint8, device="cuda")
    gs = torch.empty(E, 2 * I // 128, d // 128, dtype=torch.float32, device="cuda")
    dq = torch.empty(E, d, I, dtype=torch.uint8, device="cuda")
    ds = torch.empty(E, d // 128, I // 128, dtype=torch.float32, device="cuda")
    moe.moe_quantize_fp8_blockwise(inp["w_gu"], 2 * I, d, E, gq, gs)
    moe.moe_quantize_fp8_blockwise(inp["w_down"], d, I, E, dq, ds)
    inp.update(w_gu=gq, w_gu_scale=gs, w_down=dq, w_down_scale=ds)
    return inp


CFG = dataclasses.replace(
    recipes.small_variant(recipes.CONFIGS["v3_bf16"], T=777, d=512, inter=256, n_routed=32),
    n_group=4, topk_group=2)


@pytest.mark.parametrize("world,n_redundant", [(1, 0), (2, 0), (4, 0), (4, 4)])
def test_emulated_expert_parallel_equals_single_gpu(world, n_redundant):
    moe.moe_last_device_status()
    inp = recipes.device_inputs(CFG)
    h_ref, counts = reference(CFG, inp)
    replicas = ep.choose_replicas(counts, world, n_redundant) if n_redundant else {}
    pl = ep.Placement(CFG.n_routed, world, replicas)
    h, loads = emulate(CFG, inp, pl)
    assert moe.moe_last_device_status() == moe.OK
    assert torch.equal(h, h_ref), \
        f"max |diff| {float((h.float() - h_ref.float()).abs().max()):.3e}"
    assert sum(loads) == CFG.T * CFG.top_k
    print(f"W={world} redundant={n_redundant}: rows per rank {loads}")


def emulate_peer(cfg, inp, pl):
    """The peer-memory exchange with W ranks emulated on one GPU: each rank's
    dispatch kernel stores straight into the other ranks' receive buffers and
    each rank's down projection straight into the senders' return buffers
    (local addresses here; CUDA IPC mappings of other GPUs' memory on a
    node).  Phases run rank by rank, all dispatches before any expert phase."""
    W = pl.world
    shards = [bench.token_shard(cfg.T, r, W) for r in range(W)]
    descs, steps, xs = [], [], []
    for r, (lo, hi) in enumerate(shards):
        c = dataclasses.replace(cfg, T=hi - lo)
        d = moe.desc_from_config(c)
        x = inp["x"][lo:hi].contiguous()
        descs.append(d)
        xs.append(x)
        steps.append(ep.ep_dispatch(d, pl, r, x, inp["w_r"], inp["bias"], build_send=False))
    M = np.stack([s.plan.send_counts for s in steps])                    # [src, dst, slot]
    cap = int(M.sum(axis=(0, 2)).max())
    exs = [ep.PeerExchange(descs[r], pl, r, cap, "cuda", torch.bfloat16) for r in range(W)]
    ep.PeerExchange.link(exs)
    for r in range(W):
        ep.peer_dispatch(descs[r], exs[r], steps[r], xs[r], M)
    fp8 = cfg.dtype == "e4m3"
    full = (inp["w_gu"], inp["w_down"]) + ((inp["w_gu_scale"], inp["w_down_scale"]) if fp8 else ())
    weights = [ep.local_weights(pl, r, cfg.n_shared, *full) for r in range(W)]
    loads = [ep.peer_compute(descs[r], exs[r], steps[r], M, *weights[r]) for r in range(W)]
    hs = [ep.peer_combine(descs[r], exs[r], steps[r], xs[r], None, *weights[r])
          for r in range(W)]
    return torch.cat(hs), loads


@pytest.mark.parametrize("world,n_redundant", [(1, 0), (2, 0), (4, 0), (4, 4)])
def test_emulated_peer_exchange_equals_single_gpu(world, n_redundant):
    moe.moe_last_device_status()
    inp = recipes.device_inputs(CFG)
    h_ref, counts = reference(CFG, inp)
    replicas = ep.choose_replicas(counts, world, n_redundant) if n_redundant else {}
    pl = ep.Placement(CFG.n_routed, world, replicas)
    h, loads = emulate_peer(CFG, inp, pl)
    assert moe.moe_last_device_status() == moe.OK
    assert torch.equal(h, h_ref), \
        f"max |diff| {float((h.float() - h_ref.float()).abs().max()):.3e}"
    assert sum(loads) == CFG.T * CFG.top_k
    print(f"peer W={world} redundant={n_redundant}: rows per rank {loads}")


CFG_FP8 = dataclasses.replace(CFG, dtype="e4m3", name="v3_fp8-ep")


@pytest.mark.parametrize("world,n_redundant,peer", [(1, 0, False), (4, 0, False), (4, 4, False),
                                                    (2, 0, True), (4, 4, True)])
def test_emulated_fp8_expert_parallel_equals_single_gpu(world, n_redundant, peer):
    """§3.6's FP8 dispatch: rows travel as 1x128 E4M3 codes with their scales,
    expert outputs come back in bf16; equal to the FP8 moe_forward bit for bit."""
    moe.moe_last_device_status()
    inp = fp8_inputs(CFG_FP8)
    h_ref, counts = reference(CFG_FP8, inp)
    replicas = ep.choose_replicas(counts, world, n_redundant) if n_redundant else {}
    pl = ep.Placement(CFG_FP8.n_routed, world, replicas)
    h, loads = (emulate_peer if peer else emulate)(CFG_FP8, inp, pl)
    assert moe.moe_last_device_status() == moe.OK
    assert torch.equal(h, h_ref), \
        f"max |diff| {float((h.float() - h_ref.float()).abs().max()):.3e}"
    assert sum(loads) == CFG_FP8.T * CFG_FP8.top_k
