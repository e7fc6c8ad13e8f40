"""Shared helpers of the GPU parity tests: run the layer through the C ABI
stage by stage, and evaluate the fp64 oracle on the same synthetic inputs."""
import numpy as np
import torch

import forward_moe_route_b200 as moe
from oracle import moe_oracle as mo
from synth import recipes

TOL = {"f32": 2e-2, "bf16": 2e-2, "e4m3": 6e-2}
W_ATOL = 1e-5  # gate weights: fp32 GPU vs fp64 oracle


def act_dtype(cfg):
    return torch.float32 if cfg.dtype == "f32" else torch.bfloat16


def run_stages(cfg, inp, zipf_offsets=None):
    """moe_route -> moe_permute -> moe_grouped_swiglu -> moe_combine; returns host copies."""
    T, N, K, d, Ks = cfg.T, cfg.n_routed, cfg.top_k, cfg.d, cfg.n_shared
    R = T * K
    dev = "cuda"
    desc = moe.desc_from_config(cfg)
    ws = moe.workspace(desc)
    i32 = dict(dtype=torch.int32, device=dev)
    idx = torch.full((T, K), -7, **i32)
    w = torch.full((T, K), float("nan"), dtype=torch.float32, device=dev)
    counts = torch.full((N,), -7, **i32)
    moe.moe_route(desc, inp["x"], inp["w_r"], inp["bias"], idx, w, counts, ws)
    offsets = torch.full((N + 1,), -7, **i32)
    perm_src = torch.full((max(R, 1),), -7, **i32)
    slot_of = torch.full((max(R, 1),), -7, **i32)
    fp8 = cfg.dtype == "e4m3"
    xrows = R + (T if fp8 else 0)
    x_perm = torch.empty(max(xrows, 1), d, dtype=torch.uint8 if fp8 else act_dtype(cfg),
                         device=dev)
    x_perm_scale = torch.empty(max(xrows, 1), d // 128, dtype=torch.float32,
                               device=dev) if fp8 else None
    moe.moe_permute(desc, inp["x"], idx, counts, offsets, perm_src, slot_of, x_perm,
                    x_perm_scale, ws)
    y = torch.empty(max(T, 1), K + Ks, d, dtype=act_dtype(cfg), device=dev)
    moe.moe_grouped_swiglu(desc, inp["x"], x_perm, x_perm_scale, offsets, perm_src, slot_of, w,
                           inp["w_gu"], inp.get("w_gu_scale"), inp["w_down"],
                           inp.get("w_down_scale"), y, ws)
    h = torch.empty(max(T, 1), d, dtype=act_dtype(cfg), device=dev)
    moe.moe_combine(desc, inp["x"], y, h)
    status = moe.moe_last_device_status()
    out = {"status": status, "idx": idx, "w": w, "counts": counts, "offsets": offsets,
           "perm_src": perm_src[:R], "slot_of": slot_of[:R], "x_perm": x_perm, "y": y, "h": h,
           "x_perm_scale": x_perm_scale}
    return out


def run_forward(cfg, inp, ws=None):
    desc = moe.desc_from_config(cfg)
    ws = moe.workspace(desc) if ws is None else ws
    h = torch.empty(max(cfg.T, 1), cfg.d, dtype=act_dtype(cfg), device="cuda")
    idx = torch.empty(max(cfg.T, 1), cfg.top_k, dtype=torch.int32, device="cuda")
    counts = torch.empty(cfg.n_routed, dtype=torch.int32, device="cuda")
    moe.moe_forward(desc, inp["x"], None, inp["w_r"], inp["bias"], inp["w_gu"],
                    inp.get("w_gu_scale"), inp["w_down"], inp.get("w_down_scale"), h, idx, counts,
                    ws)
    return h, idx, counts, moe.moe_last_device_status()


def f64(t):
    return t.double().cpu().numpy()


class HostLayer:
    """The layer's inputs on the host (float64, exactly the stored values)."""

    def __init__(self, cfg, zipf_offsets=None):
        self.cfg = cfg
        self.x = recipes.host_x(cfg)
        self.w_r = recipes.host_router(cfg, zipf_offsets)
        self.bias = recipes.host_bias(cfg)
        self._experts = {}

    def expert(self, e):
        if e not in self._experts:
            self._experts[e] = recipes.host_expert(self.cfg, e)
        return self._experts[e]

    def route(self):
        c = self.cfg
        return mo.route(self.x, self.w_r, self.bias, gate=c.gate, top_k=c.top_k,
                        n_group=c.n_group, topk_group=c.topk_group, renorm=c.renorm,
                        route_scale=c.route_scale)


def check_routing(cfg, ref, g_idx, g_w, g_counts):
    """Indices bit-exact except near-ties; counts from the GPU's own indices;
    weights within W_ATOL of the oracle's weights for the GPU's selection.

    Outside near-ties the selected set is unique and must match.  Its order is
    unique too, except where two selected keys lie within the tie bound of
    each other: keys equal in the kernel's fp32 go to the lower index, which
    the fp64 oracle may order the other way.  There the order must only be
    valid (non-increasing oracle keys up to the bound)."""
    ties = mo.near_tie_tokens(ref["kgap"], ref["ggap"])
    keep = np.setdiff1d(np.arange(cfg.T), ties)
    ref_idx = ref["idx"]
    K = ref_idx.shape[1]
    o_keys = np.take_along_axis(ref["key"], ref_idx, axis=1)
    if K > 1:
        inner = np.min(o_keys[:, :-1] - o_keys[:, 1:], axis=1) < mo.NEAR_TIE
    else:
        inner = np.zeros(cfg.T, bool)
    order_free = keep[inner[keep]]
    exact = keep[~inner[keep]]
    assert np.array_equal(g_idx[exact], ref_idx[exact]), \
        f"{np.sum(np.any(g_idx[exact] != ref_idx[exact], axis=1))} tokens select differently"
    if len(order_free):
        assert np.array_equal(np.sort(g_idx[order_free], axis=1),
                              np.sort(ref_idx[order_free], axis=1))
        g_keys = np.take_along_axis(ref["key"][order_free], g_idx[order_free], axis=1)
        assert np.all(g_keys[:, :-1] >= g_keys[:, 1:] - mo.NEAR_TIE)
    assert np.array_equal(g_counts, np.bincount(g_idx.reshape(-1), minlength=cfg.n_routed))
    if len(ties) == 0:
        assert np.array_equal(g_counts, np.bincount(ref["idx"].reshape(-1),
                                                    minlength=cfg.n_routed))
    w_ref = mo.gate_weights(ref["s"], g_idx, cfg.renorm, cfg.route_scale)
    assert np.max(np.abs(g_w - w_ref)) <= W_ATOL
    return ties


def oracle_outputs(host, ref, g_idx, tokens):
    c = host.cfg
    ties = mo.near_tie_tokens(ref["kgap"], ref["ggap"])
    return mo.moe_forward(host.x, host.w_r, host.bias, host.expert, n_shared=c.n_shared,
                          gate=c.gate, top_k=c.top_k, n_group=c.n_group,
                          topk_group=c.topk_group, renorm=c.renorm, route_scale=c.route_scale,
                          tokens=tokens, idx_override={int(t): g_idx[t] for t in ties})
