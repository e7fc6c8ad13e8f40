"""GPU parity of the FP8 E4M3 layer (1x128 activation tiles, 128x128 weight
blocks, fp32 scales, promotion every 128 elements) against the oracle.

Bit-exact: the weight codes and block scales of moe_quantize_fp8_blockwise,
and the activation codes and tile scales moe_permute writes (both sides take
the same fp32 decisions: amax, amax/448, v * (448/amax), E4M3 rounding).
Within max-abs-relative 6e-2: h and the MoE part, against the oracle's
emulation of the FP8 layer (E4M3 operands, exact block products, H held in
fp32 and requantised per 1x128 tile).
"""
import dataclasses

import numpy as np
import pytest
import torch

import forward_moe_route_b200 as moe
from oracle import fp8 as of8
from oracle import moe_oracle as mo
from synth import recipes

from gpu_layer import TOL, HostLayer, check_routing, f64, run_forward, run_stages

pytestmark = pytest.mark.gpu

PLAIN_TOL = 2.0 ** -3

C = recipes.CONFIGS


def e4m3_values(t):
    return t.view(torch.float8_e4m3fn).double().cpu().numpy()


def quantize_weights(cfg, inp):
    E, I, d = cfg.n_experts, cfg.inter, cfg.d
    gq = torch.empty(E, 2 * I, d, dtype=torch.uint8, device="cuda")
    gs = torch.empty(E, 2 * I // 128, d // 128, dtype=torch.float32, device="cuda")
    dq = torch.empty(E, d, I, dtype=torch.uint8, device="cuda")
    ds = torch.empty(E, d // 128, I // 128, dtype=torch.float32, device="cuda")
    moe.moe_quantize_fp8_blockwise(inp["w_gu"], 2 * I, d, E, gq, gs)
    moe.moe_quantize_fp8_blockwise(inp["w_down"], d, I, E, dq, ds)
    return gq, gs, dq, ds


class Fp8Host(HostLayer):
    """Host layer whose experts are the oracle's own 128x128 quantisation."""

    def expert(self, e):
        if e not in self._experts:
            wg, wu, wd = recipes.host_expert(self.cfg, e)
            gu = np.concatenate([wg, wu]).astype(np.float32)
            qg, sg = of8.quantize_weight_128x128(gu)
            qd, sd = of8.quantize_weight_128x128(wd.astype(np.float32))
            guh = of8.dequant_weight(qg, sg)
            I = self.cfg.inter
            self._experts[e] = (guh[:I], guh[I:], of8.dequant_weight(qd, sd))
        return self._experts[e]


CASES = {
    "v3_fp8_small": recipes.small_variant(C["v3_fp8"], T=600, d=512, inter=256),
    "v3_fp8_ragged": recipes.small_variant(C["v3_fp8"], T=257, d=768, inter=384),
    "v3_fp8_T1": recipes.small_variant(C["v3_fp8"], T=1, d=256, inter=128),
}


@pytest.mark.parametrize("name", list(CASES))
def test_fp8_layer_parity(name):
    cfg = CASES[name]
    moe.moe_last_device_status()
    inp = recipes.device_inputs(cfg)
    host = Fp8Host(cfg)
    if cfg.T > 5:
        inp["x"][5, 128:256] = 0          # one all-zero activation tile
        host.x[5, 128:256] = 0.0
    gq, gs, dq, ds = quantize_weights(cfg, inp)
    # weight codes and scales, bit-exact, for a few experts
    I, d = cfg.inter, cfg.d
    for e in (0, 1, cfg.n_experts - 1):
        wg, wu, wd = recipes.host_expert(cfg, e)
        qg, sg = of8.quantize_weight_128x128(np.concatenate([wg, wu]).astype(np.float32))
        qd, sd = of8.quantize_weight_128x128(wd.astype(np.float32))
        assert np.array_equal(e4m3_values(gq[e]), qg)
        assert np.array_equal(gs[e].cpu().numpy(), sg)
        assert np.array_equal(e4m3_values(dq[e]), qd)
        assert np.array_equal(ds[e].cpu().numpy(), sd)
    qinp = dict(inp, w_gu=gq, w_gu_scale=gs, w_down=dq, w_down_scale=ds)
    g = run_stages(cfg, qinp)
    assert g["status"] == moe.OK, moe.moe_status_string(g["status"])
    ref = host.route()
    g_idx = g["idx"].cpu().numpy().astype(np.int64)
    ties = check_routing(cfg, ref, g_idx, g["w"].cpu().numpy().astype(np.float64),
                         g["counts"].cpu().numpy())
    _, offsets, perm_src, _ = mo.permutation(g_idx, cfg.n_routed)
    assert np.array_equal(g["offsets"].cpu().numpy(), offsets)
    # activation codes and scales, bit-exact: routed rows then the token-order copy
    q, s = of8.quantize_act_1x128(host.x.astype(np.float32))
    R = cfg.T * cfg.top_k
    xq = e4m3_values(g["x_perm"][:R + cfg.T])
    xs = g["x_perm_scale"][:R + cfg.T].cpu().numpy()
    assert np.array_equal(xq[:R], q[perm_src]) and np.array_equal(xq[R:], q)
    assert np.array_equal(xs[:R], s[perm_src]) and np.array_equal(xs[R:], s)
    # outputs against the emulating oracle
    x_hat = of8.dequant_act(q, s)
    w = mo.gate_weights(ref["s"], g_idx, cfg.renorm, cfg.route_scale)
    h_ref, delta_ref = mo.layer_output(x_hat, host.x, g_idx, w, cfg.n_shared, host.expert,
                                       ffn=of8.fp8_swiglu_ffn)
    got = f64(g["h"][:cfg.T])
    err = mo.max_abs_rel(got, h_ref)
    err_d = mo.max_abs_rel(f64(g["y"][:cfg.T]).sum(axis=1), delta_ref)
    # for context: distance to the unquantised fp64 layer
    exact = mo.layer_output(host.x, host.x, g_idx, w, cfg.n_shared,
                            lambda e: recipes.host_expert(cfg, e))[1]
    err_exact = mo.max_abs_rel(f64(g["y"][:cfg.T]).sum(axis=1), exact)
    print(f"{name}: h {err:.3e}, MoE part {err_d:.3e} (vs unquantised {err_exact:.3e}), "
          f"near-ties {len(ties)}")
    assert err <= TOL["e4m3"] and err_d <= TOL["e4m3"]
    # The quantisation error itself, against the unquantised fp64 layer: a
    # separate, looser gate (twice E4M3's relative rounding step 2^-4); the
    # 6e-2 bound above applies to the oracle's emulation of the FP8 recipe.
    assert err_exact <= PLAIN_TOL, f"distance to the unquantised layer {err_exact:.3e}"


def test_fp8_forward_equals_stages_and_is_deterministic():
    cfg = CASES["v3_fp8_small"]
    moe.moe_last_device_status()
    inp = recipes.device_inputs(cfg)
    gq, gs, dq, ds = quantize_weights(cfg, inp)
    qinp = dict(inp, w_gu=gq, w_gu_scale=gs, w_down=dq, w_down_scale=ds)
    g = run_stages(cfg, qinp)
    h1, idx1, _, st1 = run_forward(cfg, qinp)
    h2, _, _, st2 = run_forward(cfg, qinp)
    assert st1 == moe.OK and st2 == moe.OK
    assert torch.equal(h1, g["h"][:cfg.T]) and torch.equal(h1, h2)
    assert torch.equal(idx1, g["idx"])
