"""GPU parity of the gating step alone (moe_route) over the shapes the
selection kernel handles: softmax and sigmoid gating, groups of 8, 16, 24
and 64 experts, K above 8, more than 256 experts, a ragged T, and more
tokens than one wave of blocks.  Indices must match the oracle bit-exactly
outside near-ties, counts exactly, weights within 1e-5, and a second call
must give the same bits.
"""
import dataclasses

import numpy as np
import pytest
import torch

import forward_moe_route_b200 as moe
from synth import recipes

from gpu_layer import HostLayer, check_routing

pytestmark = pytest.mark.gpu

V3 = recipes.CONFIGS["v3_bf16"]
DS = recipes.CONFIGS["dsmoe16b_bf16"]


def case(base, **kw):
    return dataclasses.replace(base, name="gating", inter=128, **kw)


CASES = {
    # sigmoid + bias with groups of 16, 64 and 8 experts
    "groups16": case(V3, T=777, d=256, n_routed=128, n_group=8, topk_group=4, top_k=8),
    "groups64": case(V3, T=512, d=384, n_routed=256, n_group=4, topk_group=2, top_k=8),
    "groups8": case(V3, T=300, d=256, n_routed=64, n_group=8, topk_group=3, top_k=6),
    # softmax without groups, N not a multiple of 64
    "softmax160": case(DS, T=1000, d=256, n_routed=160, top_k=6),
    # many tokens
    "many_tiles": case(V3, T=20000, d=128, n_routed=64, n_group=8, topk_group=4, top_k=8),
    # K > 8, N > 256, groups of 24
    "k10": case(DS, T=500, d=256, n_routed=64, top_k=10),
    "n320": case(DS, T=400, d=256, n_routed=320, top_k=6),
    "groups24": case(V3, T=350, d=256, n_routed=96, n_group=4, topk_group=2, top_k=6),
}


@pytest.mark.parametrize("name", list(CASES))
def test_gating_parity(name):
    cfg = CASES[name]
    moe.moe_last_device_status()
    inp = recipes.device_inputs(cfg)
    desc = moe.desc_from_config(cfg)
    ws = moe.workspace(desc)
    idx = torch.full((cfg.T, cfg.top_k), -7, dtype=torch.int32, device="cuda")
    w = torch.full((cfg.T, cfg.top_k), float("nan"), dtype=torch.float32, device="cuda")
    counts = torch.full((cfg.n_routed,), -7, dtype=torch.int32, device="cuda")
    moe.moe_route(desc, inp["x"], inp["w_r"], inp["bias"], idx, w, counts, ws)
    assert moe.moe_last_device_status() == moe.OK
    ref = HostLayer(cfg).route()
    ties = check_routing(cfg, ref, idx.cpu().numpy().astype(np.int64),
                         w.cpu().numpy().astype(np.float64), counts.cpu().numpy())
    print(f"{name}: near-ties {len(ties)} of {cfg.T}")
    # a second call gives the same bits
    idx2, w2, c2 = torch.empty_like(idx), torch.empty_like(w), torch.empty_like(counts)
    moe.moe_route(desc, inp["x"], inp["w_r"], inp["bias"], idx2, w2, c2, ws)
    assert torch.equal(idx, idx2) and torch.equal(w, w2) and torch.equal(counts, c2)
