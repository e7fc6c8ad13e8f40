"""GPU parity of the load-balancing rows: affinities for every expert, the
f_i / P_i statistics per sequence, and the auxiliary-loss-free bias update,
against the oracle."""
import numpy as np
import pytest
import torch

import forward_moe_route_b200 as moe
from oracle import moe_oracle as mo
from synth import recipes

from gpu_layer import HostLayer

pytestmark = pytest.mark.gpu

C = recipes.CONFIGS
CASES = {
    "tiny_f32": C["tiny_f32"],
    "dsmoe_small": recipes.small_variant(C["dsmoe16b_bf16"], T=1000, d=256, inter=192),
    "v3_small": recipes.small_variant(C["v3_bf16"], T=900, d=512, inter=256),
}


def route_on_gpu(cfg, inp, bias=None):
    desc = moe.desc_from_config(cfg)
    ws = moe.workspace(desc)
    idx = torch.empty(cfg.T, cfg.top_k, dtype=torch.int32, device="cuda")
    w = torch.empty(cfg.T, cfg.top_k, dtype=torch.float32, device="cuda")
    counts = torch.empty(cfg.n_routed, dtype=torch.int32, device="cuda")
    moe.moe_route(desc, inp["x"], inp["w_r"], inp["bias"] if bias is None else bias, idx, w,
                  counts, ws)
    return desc, ws, idx, counts


@pytest.mark.parametrize("name", list(CASES))
def test_affinities_and_stats(name):
    cfg = CASES[name]
    moe.moe_last_device_status()
    inp = recipes.device_inputs(cfg)
    desc, ws, idx, counts = route_on_gpu(cfg, inp)
    s = torch.empty(cfg.T, cfg.n_routed, dtype=torch.float32, device="cuda")
    moe.moe_route_affinities(desc, inp["x"], inp["w_r"], s, ws)
    host = HostLayer(cfg)
    ref = host.route()
    s_gpu = s.double().cpu().numpy()
    assert np.max(np.abs(s_gpu - ref["s"])) <= 1e-5
    g_idx = idx.cpu().numpy().astype(np.int64)
    for L in sorted({cfg.T, cfg.T // 4 if cfg.T % 4 == 0 else cfg.T, 1}):
        S = cfg.T // L
        f = torch.empty(S, cfg.n_routed, dtype=torch.float32, device="cuda")
        P = torch.empty_like(f)
        moe.moe_balance_stats(desc, s, idx, L, f, P)
        f_ref, P_ref = mo.balance_stats(s_gpu, g_idx, L)
        np.testing.assert_allclose(f.cpu().numpy(), f_ref, rtol=1e-6, atol=0)
        np.testing.assert_allclose(P.cpu().numpy(), P_ref, rtol=1e-5, atol=1e-9)
    assert moe.moe_last_device_status() == moe.OK


def test_bias_update_bit_exact_and_balancing():
    cfg = CASES["v3_small"]
    inp = recipes.device_inputs(cfg)
    bias = inp["bias"].clone()
    desc = moe.desc_from_config(cfg)
    first = None
    for step in range(40):
        _, _, _, counts = route_on_gpu(cfg, inp, bias)
        c = counts.cpu().numpy()
        if first is None:
            first = c.max()
        want = mo.bias_update(bias.cpu().numpy(), c, 0.01)
        moe.moe_bias_update(desc, counts, bias, 0.01)
        assert np.array_equal(bias.cpu().numpy(), want), f"step {step}"
    assert c.max() < first
    assert moe.moe_last_device_status() == moe.OK
