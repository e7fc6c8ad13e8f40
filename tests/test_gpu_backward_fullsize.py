"""Parity of the layer backward at the full V3 size (T = 16384, d = 7168,
I = 2048, 1 + 256 experts, top-8), in the configuration `bench.py --backward`
times: moe_backward for the bf16 layer, moe_backward_fp8 for the E4M3 layer.

The whole backward oracle does not finish at this size, so outputs are
checked where the oracle can compute them one by one:
  * dx of sampled tokens: dx is separable by token (routing, the expert rows,
    the FP8 row tiles and the gate backward are all per token), so each
    sampled token's dx is the oracle's backward of a one-token batch with the
    GPU's selection;
  * dW_gate, dW_up, dW_down of sampled routed experts (the least-, a median-
    and the most-loaded one): the oracle's expert backward over all of the
    expert's rows, in token order (the FP8 weight-gradient tiles run over
    these rows).
Tolerances as at the small sizes: 2e-2 for the bf16 backward; for the FP8
backward 2e-2 of the oracle's FP8 emulation with bf16 intermediates and 2^-3
of the exact backward.
"""
import numpy as np
import pytest
import torch

import forward_moe_route_b200 as moe
import synth
from oracle import fp8 as of8
from oracle import fp8_backward as fb
from oracle import moe_backward as mb
from oracle import moe_oracle as mo
from synth import recipes

from gpu_layer import f64

pytestmark = pytest.mark.gpu

C = recipes.CONFIGS
TID_DH = 6


def upstream(cfg):
    v = synth.host_normal(cfg.T * cfg.d, 1.0, cfg.seed, TID_DH).reshape(cfg.T, cfg.d)
    dh = torch.from_numpy(v).to(torch.bfloat16)
    return dh, dh.double().numpy()


def gpu_route(cfg, inp):
    desc = moe.desc_from_config(cfg)
    ws = moe.workspace(desc)
    idx = torch.empty(cfg.T, cfg.top_k, dtype=torch.int32, device="cuda")
    w = torch.empty(cfg.T, cfg.top_k, dtype=torch.float32, device="cuda")
    counts = torch.empty(cfg.n_routed, dtype=torch.int32, device="cuda")
    moe.moe_route(desc, inp["x"], inp["w_r"], inp["bias"], idx, w, counts, ws)
    return idx.cpu().numpy().astype(np.int64), counts.cpu().numpy()


def samples(cfg, g_idx, counts, n_tokens):
    toks = sorted({int(i * cfg.T // n_tokens) for i in range(n_tokens)} | {cfg.T - 1})
    nonzero = np.nonzero(counts)[0]
    least = int(nonzero[np.argmin(counts[nonzero])])
    median = int(nonzero[np.argsort(counts[nonzero])[len(nonzero) // 2]])
    most = int(np.argmax(counts))
    return np.array(toks), sorted({least, median, most})


def check(cfg, dx, dw_gu, dw_down, g_idx, counts, expert, n_tokens, backward_rows,
          one_token, tol, label):
    """dx rows and sampled experts' weight gradients against the oracle."""
    x = recipes.host_x(cfg)
    w_r = recipes.host_router(cfg)
    bias = recipes.host_bias(cfg)
    _, dh64 = upstream(cfg)
    toks, experts = samples(cfg, g_idx, counts, n_tokens)
    kw = dict(n_shared=cfg.n_shared, gate=cfg.gate, top_k=cfg.top_k, n_group=cfg.n_group,
              topk_group=cfg.topk_group, renorm=cfg.renorm, route_scale=cfg.route_scale)
    want = np.stack([one_token(x[t:t + 1], w_r, bias, expert, dh64[t:t + 1],
                               idx_override=g_idx[t:t + 1], **kw)["dx"][0] for t in toks])
    err_dx = mo.max_abs_rel(f64(dx)[toks], want)
    s = mo.affinity(mo.router_logits(x, w_r), cfg.gate)
    g_all = mo.gate_weights(s, g_idx, cfg.renorm, cfg.route_scale)
    errs = {"dx": err_dx}
    for j in experts:
        t_sel, k_sel = np.nonzero(g_idx == j)
        e = cfg.n_shared + j
        wg, wu, wd = expert(e)
        dwg, dwu, dwd = backward_rows(x[t_sel], dh64[t_sel], g_all[t_sel, k_sel], wg, wu, wd)
        errs[f"dw_gu[{e}] ({len(t_sel)} rows)"] = mo.max_abs_rel(
            f64(dw_gu[e]), np.concatenate([dwg, dwu]))
        errs[f"dw_down[{e}]"] = mo.max_abs_rel(f64(dw_down[e]), dwd)
    print(f"{cfg.name} {label}: {len(toks)} tokens, " +
          ", ".join(f"{k} {v:.2e}" for k, v in errs.items()))
    for k, v in errs.items():
        assert v <= tol, f"{k}: max-abs-rel {v:.3e} above {tol}"


def test_v3_bf16_backward_full():
    cfg = C["v3_bf16"]
    inp = recipes.device_inputs(cfg, "cuda")
    dh, _ = upstream(cfg)
    desc = moe.desc_from_config(cfg)
    E, I, d, N = cfg.n_experts, cfg.inter, cfg.d, cfg.n_routed
    dx = torch.empty(cfg.T, d, dtype=torch.bfloat16, device="cuda")
    dwr = torch.empty(N, d, dtype=torch.float32, device="cuda")
    dwgu = torch.empty(E, 2 * I, d, dtype=torch.float32, device="cuda")
    dwd = torch.empty(E, d, I, dtype=torch.float32, device="cuda")
    moe.moe_backward(desc, inp["x"], inp["w_r"], inp["bias"], inp["w_gu"], inp["w_down"],
                     dh.cuda(), dx, dwr, dwgu, dwd, moe.backward_workspace(desc))
    assert moe.moe_last_device_status() == moe.OK
    g_idx, counts = gpu_route(cfg, inp)
    del inp
    cache = {}

    def expert(e):
        if e not in cache:
            cache[e] = recipes.host_expert(cfg, e)
        return cache[e]

    def rows(u, dh_rows, g, wg, wu, wd):
        _, _, dwg, dwu, dwd = mb.expert_backward(u, g[:, None] * dh_rows, wg, wu, wd)
        return dwg, dwu, dwd

    check(cfg, dx, dwgu, dwd, g_idx, counts, expert, 8, rows, mb.moe_backward, 2e-2, "bf16")


def test_v3_fp8_backward_full():
    cfg = C["v3_fp8"]
    inp = recipes.device_inputs(cfg, "cuda")
    dh, _ = upstream(cfg)
    desc = moe.desc_from_config(cfg)
    E, I, d, N = cfg.n_experts, cfg.inter, cfg.d, cfg.n_routed

    W = moe.fp8_backward_weights(inp["w_gu"], inp["w_down"])
    bf = dict(dtype=torch.bfloat16, device="cuda")
    dx = torch.empty(cfg.T, d, **bf)
    dwr = torch.empty(N, d, **bf)
    dwgu = torch.empty(E, 2 * I, d, **bf)
    dwd = torch.empty(E, d, I, **bf)
    moe.moe_backward_fp8(desc, inp["x"], inp["w_r"], inp["bias"], *W, dh.cuda(), dx, dwr, dwgu,
                         dwd, moe.backward_fp8_workspace(desc))
    assert moe.moe_last_device_status() == moe.OK
    g_idx, counts = gpu_route(cfg, inp)
    del inp, W
    cache = {}

    def expert(e):
        if e not in cache:
            wg, wu, wd = recipes.host_expert(cfg, e)
            qg, sg = of8.quantize_weight_128x128(np.concatenate([wg, wu]).astype(np.float32))
            qd, sd = of8.quantize_weight_128x128(wd.astype(np.float32))
            gu = of8.dequant_weight(qg, sg)
            cache[e] = (gu[:I], gu[I:], of8.dequant_weight(qd, sd))
        return cache[e]

    def rows_emu(u, dh_rows, g, wg, wu, wd):
        _, _, dwg, dwu, dwd = fb.expert_backward_fp8(u, dh_rows, g, wg, wu, wd, "bf16")
        return dwg, dwu, dwd

    def one_emu(*args, **kw):
        return fb.moe_backward_fp8(*args, intermediates="bf16", **kw)

    check(cfg, dx, dwgu, dwd, g_idx, counts, expert, 4, rows_emu, one_emu, 2e-2,
          "FP8 vs emulation (bf16 intermediates)")

    def rows_exact(u, dh_rows, g, wg, wu, wd):
        _, _, dwg, dwu, dwd = mb.expert_backward(u, g[:, None] * dh_rows, wg, wu, wd)
        return dwg, dwu, dwd

    check(cfg, dx, dwgu, dwd, g_idx, counts, expert, 4, rows_exact, mb.moe_backward,
          2.0 ** -3, "FP8 vs exact")
