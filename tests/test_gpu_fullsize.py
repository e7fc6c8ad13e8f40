"""Parity at the full sizes of the 16B-, V2- (skewed load), V3- and V3-FP8-shaped
layers, through moe_forward in the launch configuration the bench times.

Routing is checked on every token (indices bit-exact except near-ties,
counts, offsets and the permutation); outputs on a token sample the oracle
can evaluate one by one: min(T, 256) strided tokens, up to 64 tokens of the
most- and of the least-loaded expert, and the last row of the experts with
the most ragged last GEMM tile.  The MoE part is checked from a second forward with a
zero residual.
"""
import numpy as np
import pytest
import torch

import forward_moe_route_b200 as moe
from oracle import fp8 as of8
from oracle import moe_oracle as mo
from synth import recipes

from gpu_layer import TOL, HostLayer, check_routing, f64

pytestmark = pytest.mark.gpu

C = recipes.CONFIGS


def zipf_offsets(cfg):
    if not cfg.zipf:
        return None
    import os
    path = os.path.join(os.path.dirname(__file__), "golden",
                        f"zipf_offsets_{cfg.name.split('@')[0]}.txt")
    return np.loadtxt(path, dtype=np.float64)


def forward(cfg, inp, x_res=None, want_perm=False):
    desc = moe.desc_from_config(cfg)
    ws = moe.workspace(desc)
    h = torch.empty(cfg.T, cfg.d, dtype=torch.bfloat16, device="cuda")
    idx = torch.empty(cfg.T, cfg.top_k, dtype=torch.int32, device="cuda")
    counts = torch.empty(cfg.n_routed, dtype=torch.int32, device="cuda")
    moe.moe_forward(desc, inp["x"], x_res, inp["w_r"], inp["bias"], inp["w_gu"],
                    inp.get("w_gu_scale"), inp["w_down"], inp.get("w_down_scale"), h, idx, counts,
                    ws)
    st = moe.moe_last_device_status()
    assert st == moe.OK, moe.moe_status_string(st)
    perm = None
    if want_perm:
        T, K, N = cfg.T, cfg.top_k, cfg.n_routed
        offsets = torch.empty(N + 1, dtype=torch.int32, device="cuda")
        ps = torch.empty(T * K, dtype=torch.int32, device="cuda")
        so = torch.empty(T * K, dtype=torch.int32, device="cuda")
        fp8 = cfg.dtype == "e4m3"
        xp = torch.empty(T * K + (T if fp8 else 0), cfg.d,
                         dtype=torch.uint8 if fp8 else torch.bfloat16, device="cuda")
        xs = torch.empty(xp.shape[0], cfg.d // 128, dtype=torch.float32,
                         device="cuda") if fp8 else None
        moe.moe_permute(desc, inp["x"], idx, counts, offsets, ps, so, xp, xs, ws)
        perm = (offsets.cpu().numpy(), ps.cpu().numpy(), so.cpu().numpy())
    del ws
    return h, idx, counts, perm


def sample_tokens(cfg, g_idx, counts, offsets, perm_src, n_strided, n_extra=64, n_ragged=8):
    """S = min(T, n_strided) strided tokens, up to n_extra tokens of the most- and
    of the least-loaded (non-empty) expert, and the token holding the last row
    of the n_ragged experts whose last 32-token GEMM tile is the most ragged
    (fewest rows in it), so every kind of tile edge is sampled."""
    S = min(cfg.T, n_strided)
    toks = set(int(i * cfg.T // S) for i in range(S))
    for e in (int(np.argmax(counts)), int(np.argmin(np.where(counts > 0, counts, 1 << 30)))):
        rows = np.nonzero(np.any(g_idx == e, axis=1))[0]
        toks.update(int(t) for t in rows[:n_extra])
    tail = np.where(counts > 0, (counts - 1) % 32, 1 << 30)
    for e in np.argsort(tail, kind="stable")[:n_ragged]:
        if counts[e] > 0:
            toks.add(int(perm_src[offsets[e + 1] - 1]))
    return np.array(sorted(toks))


def check_layer(cfg, n_strided):
    offs = zipf_offsets(cfg)
    inp = recipes.device_inputs(cfg, "cuda", offs)
    h, idx, counts, perm = forward(cfg, inp, want_perm=True)
    h_moe, _, _, _ = forward(cfg, inp, x_res=torch.zeros_like(inp["x"]))
    host = HostLayer(cfg, offs)
    ref = host.route()
    g_idx = idx.cpu().numpy().astype(np.int64)
    g_counts = counts.cpu().numpy()
    # counts and weights need the GPU's topk_w, which moe_forward keeps internal:
    # re-run routing through moe_route on the same inputs (same kernels)
    desc = moe.desc_from_config(cfg)
    ws = moe.workspace(desc)
    idx2 = torch.empty_like(idx)
    w2 = torch.empty(cfg.T, cfg.top_k, dtype=torch.float32, device="cuda")
    c2 = torch.empty_like(counts)
    moe.moe_route(desc, inp["x"], inp["w_r"], inp["bias"], idx2, w2, c2, ws)
    assert torch.equal(idx2, idx) and torch.equal(c2, counts)
    # the router logits sit at the start of the workspace: report their error
    lg = ws[:cfg.T * cfg.n_routed * 4].view(torch.float32).view(cfg.T, cfg.n_routed)
    lerr = np.abs(lg.double().cpu().numpy() - ref["logits"])
    bad = np.nonzero(np.any(g_idx != ref["idx"], axis=1))[0]
    print(f"{cfg.name}: router logits max abs err {lerr.max():.3e} (max |l| "
          f"{np.abs(ref['logits']).max():.2f}); tokens selecting differently {len(bad)}: "
          f"kgap {ref['kgap'][bad][:8]}, ggap {ref['ggap'][bad][:8]}")
    del ws
    ties = check_routing(cfg, ref, g_idx, w2.cpu().numpy().astype(np.float64), g_counts)
    _, offsets, perm_src, slot_of = mo.permutation(g_idx, cfg.n_routed)
    assert np.array_equal(perm[0], offsets)
    assert np.array_equal(perm[1], perm_src) and np.array_equal(perm[2], slot_of)
    toks = sample_tokens(cfg, g_idx, g_counts, offsets, perm_src, n_strided)
    w_used = mo.gate_weights(ref["s"], g_idx, cfg.renorm, cfg.route_scale)
    xs = host.x[toks]
    h_ref, d_ref = mo.layer_output(xs, xs, g_idx[toks], w_used[toks], cfg.n_shared,
                                   lambda e: recipes.host_expert(cfg, e))
    err = mo.max_abs_rel(f64(h)[toks], h_ref)
    err_d = mo.max_abs_rel(f64(h_moe)[toks], d_ref)
    print(f"{cfg.name}: {len(toks)} sampled tokens, h {err:.3e}, MoE part {err_d:.3e}, "
          f"near-ties {len(ties)} of {cfg.T}, max/mean load {g_counts.max() / g_counts.mean():.2f}")
    assert err <= TOL["bf16"] and err_d <= TOL["bf16"]


def test_dsmoe16b_full():
    check_layer(C["dsmoe16b_bf16"], 256)


def test_v2_zipf_full():
    cfg = C["v2_bf16_zipf"]
    check_layer(cfg, 256)


def test_v3_bf16_full():
    check_layer(C["v3_bf16"], 256)


def fp8_expert(cfg, e):
    """Expert e as the FP8 layer sees it: the oracle's 128x128 quantisation."""
    wg, wu, wd = recipes.host_expert(cfg, e)
    qg, sg = of8.quantize_weight_128x128(np.concatenate([wg, wu]).astype(np.float32))
    qd, sd = of8.quantize_weight_128x128(wd.astype(np.float32))
    gu = of8.dequant_weight(qg, sg)
    return gu[:cfg.inter], gu[cfg.inter:], of8.dequant_weight(qd, sd)


def test_v3_fp8_sweep_full():
    """The FP8 layer at T = 256, 2048, 16384 and 65536.  The weights are the
    same at every T, so the GPU layers run first and keep their sampled rows;
    then one pass over the experts prepares each expert once (a thread pool,
    the contributions summed in expert order) for all four samples."""
    from concurrent.futures import ThreadPoolExecutor
    samples = []
    for T in recipes.FP8_SWEEP_T:
        cfg = C["v3_fp8"].with_T(T)
        inp = recipes.device_inputs(cfg, "cuda")
        E, I, d = cfg.n_experts, cfg.inter, cfg.d
        gq = torch.empty(E, 2 * I, d, dtype=torch.uint8, device="cuda")
        gs = torch.empty(E, 2 * I // 128, d // 128, dtype=torch.float32, device="cuda")
        dq = torch.empty(E, d, I, dtype=torch.uint8, device="cuda")
        ds = torch.empty(E, d // 128, I // 128, dtype=torch.float32, device="cuda")
        moe.moe_quantize_fp8_blockwise(inp["w_gu"], 2 * I, d, E, gq, gs)
        moe.moe_quantize_fp8_blockwise(inp["w_down"], d, I, E, dq, ds)
        inp.update(w_gu=gq, w_gu_scale=gs, w_down=dq, w_down_scale=ds)
        torch.cuda.synchronize()
        h, idx, counts, perm = forward(cfg, inp, want_perm=True)
        h_moe, _, _, _ = forward(cfg, inp, x_res=torch.zeros_like(inp["x"]))
        host = HostLayer(cfg)
        ref = host.route()
        g_idx = idx.cpu().numpy().astype(np.int64)
        g_counts = counts.cpu().numpy()
        desc = moe.desc_from_config(cfg)
        ws = moe.workspace(desc)
        w2 = torch.empty(cfg.T, cfg.top_k, dtype=torch.float32, device="cuda")
        moe.moe_route(desc, inp["x"], inp["w_r"], inp["bias"], torch.empty_like(idx), w2,
                      torch.empty_like(counts), ws)
        ties = check_routing(cfg, ref, g_idx, w2.cpu().numpy().astype(np.float64), g_counts)
        _, offsets, perm_src, slot_of = mo.permutation(g_idx, cfg.n_routed)
        assert np.array_equal(perm[0], offsets)
        assert np.array_equal(perm[1], perm_src) and np.array_equal(perm[2], slot_of)
        toks = sample_tokens(cfg, g_idx, g_counts, offsets, perm_src, 256)
        xs = host.x[toks]
        q, sc = of8.quantize_act_1x128(xs.astype(np.float32))
        samples.append(dict(cfg=cfg, toks=toks, xs=xs, xq=of8.dequant_act(q, sc),
                            idx=g_idx[toks],
                            w=mo.gate_weights(ref["s"], g_idx, cfg.renorm, cfg.route_scale)[toks],
                            h=f64(h)[toks], h_moe=f64(h_moe)[toks], ties=len(ties)))
        del inp, gq, dq, ws, h, h_moe
        torch.cuda.empty_cache()
    cfg0 = samples[0]["cfg"]
    Ks = cfg0.n_shared
    needed = sorted(set(range(Ks)) | {Ks + int(j) for sm in samples for j in np.unique(sm["idx"])})

    def contributions(e):
        """(FP8-emulated, unquantised) MoE-part contributions of expert e to each sample."""
        wq = fp8_expert(cfg0, e)
        wp = recipes.host_expert(cfg0, e)
        out = []
        for sm in samples:
            if e < Ks:
                rows, g = np.arange(len(sm["toks"])), np.ones(len(sm["toks"]))
            else:
                rows, ks = np.nonzero(sm["idx"] == e - Ks)
                g = sm["w"][rows, ks]
            if len(rows) == 0:
                out.append(None)
                continue
            cq = g[:, None] * of8.fp8_swiglu_ffn(sm["xq"][rows], *wq)
            cp = g[:, None] * mo.swiglu_ffn(sm["xs"][rows], *wp)
            out.append((rows, cq, cp))
        return e, out

    acc_q = [np.zeros_like(sm["xs"]) for sm in samples]
    acc_p = [np.zeros_like(sm["xs"]) for sm in samples]
    with ThreadPoolExecutor(max_workers=6) as pool:
        results = dict(pool.map(contributions, needed))
    for e in needed:                          # fixed summation order
        for i, r in enumerate(results[e]):
            if r is not None:
                rows, cq, cp = r
                acc_q[i][rows] += cq
                acc_p[i][rows] += cp
    for i, sm in enumerate(samples):
        err = mo.max_abs_rel(sm["h"], sm["xs"] + acc_q[i])
        err_d = mo.max_abs_rel(sm["h_moe"], acc_q[i])
        err_plain = mo.max_abs_rel(sm["h_moe"], acc_p[i])
        print(f"{sm['cfg'].name}: {len(sm['toks'])} sampled tokens, h {err:.3e}, MoE part "
              f"{err_d:.3e}, vs the unquantised layer {err_plain:.3e}, near-ties {sm['ties']}")
        assert err <= TOL["e4m3"] and err_d <= TOL["e4m3"]
        assert err_plain <= 2.0 ** -3
