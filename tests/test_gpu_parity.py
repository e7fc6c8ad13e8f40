"""GPU parity: the CUDA path through the C ABI against the fp64 oracle, element
by element, on seeded inputs that span several tiles with ragged tails.

Bars: expert indices, counts, offsets and the permutation bit-exact (near-tie
tokens, whose K-th/(K+1)-th key gap or group gap is below 1e-5, are excluded
from the index check and counted, and the oracle is fed the GPU's selection
for them); gate weights within 1e-5; outputs within max-abs-relative 2e-2
(fp32 and bf16 layers) on h, and on the MoE part h - x_res.  The MoE part is
taken from the expert slots before the residual is added (the sum of a
token's y_slots rows): after the residual a bf16 h carries a rounding error of
up to 2^-9 |h|, which for |x_res| >> |MoE part| alone exceeds 2e-2 of the MoE
part, so the residual would mask nothing but it would hide the MoE error.
"""
import dataclasses

import numpy as np
import pytest
import torch

import forward_moe_route_b200 as moe
from oracle import moe_oracle as mo
from synth import recipes

from gpu_layer import (TOL, HostLayer, check_routing, f64, oracle_outputs, run_forward,
                       run_stages)

pytestmark = pytest.mark.gpu

C = recipes.CONFIGS


def small_cases():
    return {
        # the tiny fp32 layer exactly as specified
        "tiny_f32": C["tiny_f32"],
        # fp32 with a ragged T, d not a multiple of 64 and I = 96 (32-wide tiles)
        "f32_ragged": dataclasses.replace(C["tiny_f32"], name="f32_ragged", T=333, d=96, inter=96),
        # 16B-shaped gating, reduced widths: I = 192 -> 64-wide H tiles
        "dsmoe_small": recipes.small_variant(C["dsmoe16b_bf16"], T=1000, d=256, inter=192),
        # V2-shaped gating (160 routed, 2 shared), d = 320 -> 64-wide output tiles
        "v2_small": dataclasses.replace(
            recipes.small_variant(C["v2_bf16_zipf"], T=700, d=320, inter=128), zipf=False),
        # V3-shaped gating: sigmoid + bias, 8 groups / top-4, renorm x 2.5
        "v3_small": recipes.small_variant(C["v3_bf16"], T=900, d=512, inter=256),
        "v3_T1": recipes.small_variant(C["v3_bf16"], T=1, d=256, inter=128),
        "v3_T129": recipes.small_variant(C["v3_bf16"], T=129, d=256, inter=128),
        # long K: 64 k-blocks per tile
        "v3_d4096": recipes.small_variant(C["v3_bf16"], T=300, d=4096, inter=128),
    }


CASES = small_cases()


@pytest.fixture(autouse=True)
def _clean_status():
    moe.moe_last_device_status()
    yield


@pytest.mark.parametrize("name", list(CASES))
def test_layer_parity(name):
    cfg = CASES[name]
    inp = recipes.device_inputs(cfg)
    g = run_stages(cfg, inp)
    assert g["status"] == moe.OK, moe.moe_status_string(g["status"])
    host = HostLayer(cfg)
    ref = host.route()
    g_idx = g["idx"].cpu().numpy().astype(np.int64)
    ties = check_routing(cfg, ref, g_idx, g["w"].cpu().numpy().astype(np.float64),
                         g["counts"].cpu().numpy())
    # permutation of the GPU's selection, bit-exact
    counts, offsets, perm_src, slot_of = mo.permutation(g_idx, cfg.n_routed)
    assert np.array_equal(g["offsets"].cpu().numpy(), offsets)
    assert np.array_equal(g["perm_src"].cpu().numpy(), perm_src)
    assert np.array_equal(g["slot_of"].cpu().numpy(), slot_of.reshape(-1))
    # gathered rows are byte copies of their source rows
    xp = g["x_perm"][:cfg.T * cfg.top_k]
    assert torch.equal(xp, inp["x"][torch.as_tensor(perm_src, device="cuda")])
    # outputs
    out = oracle_outputs(host, ref, g_idx, None)
    got = f64(g["h"][:cfg.T])
    err = mo.max_abs_rel(got, out["h"])
    moe_part = f64(g["y"][:cfg.T]).sum(axis=1)
    err_d = mo.max_abs_rel(moe_part, out["delta"])
    print(f"{name}: max-abs-rel h {err:.3e}, MoE part {err_d:.3e}, near-ties {len(ties)}")
    assert err <= TOL[cfg.dtype] and err_d <= TOL[cfg.dtype]


@pytest.mark.parametrize("name", ["tiny_f32", "v3_small", "dsmoe_small"])
def test_forward_equals_stages_and_is_deterministic(name):
    cfg = CASES[name]
    inp = recipes.device_inputs(cfg)
    g = run_stages(cfg, inp)
    h1, idx1, c1, st1 = run_forward(cfg, inp)
    h2, idx2, c2, st2 = run_forward(cfg, inp)
    assert st1 == moe.OK and st2 == moe.OK
    assert torch.equal(h1, g["h"][:cfg.T]) and torch.equal(idx1, g["idx"])
    assert torch.equal(h1, h2) and torch.equal(idx1, idx2) and torch.equal(c1, c2)


def test_residual_is_separate_input():
    # With a zero residual, h is the MoE part alone; with another residual r,
    # h is r plus that part.
    cfg = CASES["v3_small"]
    inp = recipes.device_inputs(cfg)
    desc = moe.desc_from_config(cfg)
    ws = moe.workspace(desc)
    host = HostLayer(cfg)
    ref = host.route()
    zero = torch.zeros_like(inp["x"])
    h = torch.empty_like(inp["x"])
    idx = torch.empty(cfg.T, cfg.top_k, dtype=torch.int32, device="cuda")
    moe.moe_forward(desc, inp["x"], zero, inp["w_r"], inp["bias"], inp["w_gu"], None,
                    inp["w_down"], None, h, idx, None, ws)
    assert moe.moe_last_device_status() == moe.OK
    g_idx = idx.cpu().numpy().astype(np.int64)
    out = oracle_outputs(host, ref, g_idx, None)
    assert mo.max_abs_rel(f64(h), out["delta"]) <= TOL["bf16"]
    r = (inp["x"].float() * 0.5 + 1.0).to(torch.bfloat16)
    moe.moe_forward(desc, inp["x"], r, inp["w_r"], inp["bias"], inp["w_gu"], None,
                    inp["w_down"], None, h, None, None, ws)
    assert mo.max_abs_rel(f64(h), f64(r) + out["delta"]) <= TOL["bf16"]


def test_empty_input():
    cfg = dataclasses.replace(CASES["v3_small"], T=0)
    desc = moe.desc_from_config(cfg)
    ws = moe.workspace(desc)
    counts = torch.full((cfg.n_routed,), 5, dtype=torch.int32, device="cuda")
    x = torch.empty(1, cfg.d, dtype=torch.bfloat16, device="cuda")
    inp = recipes.device_inputs(dataclasses.replace(cfg, T=1))
    moe.moe_forward(desc, x, None, inp["w_r"], inp["bias"], inp["w_gu"], None, inp["w_down"],
                    None, x, None, counts, ws)
    assert moe.moe_last_device_status() == moe.OK
    assert int(counts.sum()) == 0


def test_all_tokens_to_the_same_experts():
    # A large bias on experts 40..47 (all in group 1) sends every token there:
    # those experts hold T rows each, every other routed expert is empty.
    cfg = recipes.small_variant(C["v3_bf16"], T=300, d=256, inter=128)
    inp = recipes.device_inputs(cfg)
    inp["bias"][40:48] += 10.0
    g = run_stages(cfg, inp)
    assert g["status"] == moe.OK
    counts = g["counts"].cpu().numpy()
    assert counts[40:48].tolist() == [cfg.T] * 8 and counts.sum() == cfg.T * 8
    host = HostLayer(cfg)
    host.bias = inp["bias"].double().cpu().numpy()
    ref = host.route()
    g_idx = g["idx"].cpu().numpy().astype(np.int64)
    check_routing(cfg, ref, g_idx, g["w"].cpu().numpy().astype(np.float64), counts)
    out = oracle_outputs(host, ref, g_idx, None)
    got = f64(g["h"][:cfg.T])
    assert mo.max_abs_rel(got, out["h"]) <= TOL["bf16"]
    assert mo.max_abs_rel(f64(g["y"][:cfg.T]).sum(axis=1), out["delta"]) <= TOL["bf16"]


def test_corrupt_counts_are_detected():
    cfg = CASES["dsmoe_small"]
    inp = recipes.device_inputs(cfg)
    desc = moe.desc_from_config(cfg)
    ws = moe.workspace(desc)
    T, K, N = cfg.T, cfg.top_k, cfg.n_routed
    idx = torch.empty(T, K, dtype=torch.int32, device="cuda")
    w = torch.empty(T, K, dtype=torch.float32, device="cuda")
    counts = torch.empty(N, dtype=torch.int32, device="cuda")
    moe.moe_route(desc, inp["x"], inp["w_r"], None, idx, w, counts, ws)
    assert moe.moe_last_device_status() == moe.OK
    counts[3] += 1
    offsets = torch.empty(N + 1, dtype=torch.int32, device="cuda")
    ps = torch.empty(T * K, dtype=torch.int32, device="cuda")
    so = torch.empty(T * K, dtype=torch.int32, device="cuda")
    xp = torch.empty(T * K, cfg.d, dtype=torch.bfloat16, device="cuda")
    moe.moe_permute(desc, inp["x"], idx, counts, offsets, ps, so, xp, None, ws)
    assert moe.moe_last_device_status() == moe.ERR_DEVICE_CHECK
    # an expert index outside [0, N) is reported, and nothing is written out of range
    counts[3] -= 1
    idx[5, 0] = N + 3
    moe.moe_permute(desc, inp["x"], idx, counts, offsets, ps, so, xp, None, ws)
    assert moe.moe_last_device_status() == moe.ERR_DEVICE_CHECK
    assert moe.moe_last_device_status() == moe.OK


def test_bounded_wait_reports_timeout_and_context_survives():
    moe.moe_selftest_bounded_wait(2000)
    assert moe.moe_last_device_status() == moe.ERR_TIMEOUT
    assert moe.moe_last_device_status() == moe.OK
    cfg = CASES["tiny_f32"]
    inp = recipes.device_inputs(cfg)
    _, _, _, st = run_forward(cfg, inp)
    assert st == moe.OK
