"""GPU parity of the layer backward (moe_backward) against the fp64 backward
oracle (oracle/moe_backward.py, itself pinned to central differences of the
forward oracle in tests/test_oracle_backward.py).

Every gradient is compared as a whole tensor with the max-abs-relative measure
of the forward tests: dx (through the experts and the router), dW_r, and the
three matrices of every expert (zeros for experts no token reaches).  The
bound 2e-2 is the bf16 one of the forward: the operands x, dh, the weights and
the backward's intermediates (a, b, g z, da, db, dl) are bf16, products
accumulate in fp32.  Both sides use the GPU's selection (checked against the
oracle's first, bit-exact outside near-ties), since no gradient flows through
the choice of experts.
"""
import dataclasses

import numpy as np
import pytest
import torch

import forward_moe_route_b200 as moe
import synth
from oracle import moe_backward as mb
from oracle import moe_oracle as mo
from synth import recipes

from gpu_layer import HostLayer, check_routing, f64

pytestmark = pytest.mark.gpu

TOL = 2e-2
TID_DH = 6          # tensor id of the upstream gradient in the seeded generator

C = recipes.CONFIGS
CASES = {
    # V3-like: sigmoid + selection bias, 4 groups / top-2 groups, renorm x 2.5;
    # T spans several 128-row tiles with a ragged tail
    "v3_small": dataclasses.replace(
        recipes.small_variant(C["v3_bf16"], T=300, d=512, inter=256, n_routed=32),
        n_group=4, topk_group=2),
    # 16B-like: softmax without renorm, 2 shared experts, d and I not multiples of 256
    "dsmoe16b_small": recipes.small_variant(C["dsmoe16b_bf16"], T=257, d=320, inter=192,
                                            n_routed=16),
    # reduced V3 shape: full d = 7168 and I = 2048 (the K loops and feature
    # tiles of the V3 layer), 16 routed experts, 512 tokens
    "v3_reduced": dataclasses.replace(
        recipes.small_variant(C["v3_bf16"], T=512, d=7168, inter=2048, n_routed=16),
        n_group=8, topk_group=4),
    # a single token: most experts get no row, their weight gradients must be zero
    "v3_T1": dataclasses.replace(
        recipes.small_variant(C["v3_bf16"], T=1, d=256, inter=128, n_routed=32),
        n_group=4, topk_group=2),
}


def upstream(cfg):
    v = synth.host_normal(cfg.T * cfg.d, 1.0, cfg.seed, TID_DH).reshape(cfg.T, cfg.d)
    dh = torch.from_numpy(v).to(torch.bfloat16)
    return dh.cuda(), dh.double().numpy()


def forward_save(cfg, inp):
    """moe_forward_save of the layer: (h, ab_saved, status)."""
    desc = moe.desc_from_config(cfg)
    ws = moe.workspace(desc)
    h = torch.empty(cfg.T, cfg.d, dtype=torch.bfloat16, device="cuda")
    ab = torch.full((cfg.T * (cfg.top_k + cfg.n_shared), 2 * cfg.inter), float("nan"),
                    dtype=torch.bfloat16, device="cuda")
    assert ab.numel() * 2 == moe.moe_saved_ab_bytes(desc)
    moe.moe_forward_save(desc, inp["x"], None, inp["w_r"], inp["bias"], inp["w_gu"],
                         inp["w_down"], h, None, None, ab, ws)
    return h, ab, moe.moe_last_device_status()


def run_backward(cfg, inp, dh, ab_saved=None):
    """moe_backward, or moe_backward_saved when the forward's a | b are given."""
    desc = moe.desc_from_config(cfg)
    ws = moe.backward_workspace(desc)
    E, I, d, N = cfg.n_experts, cfg.inter, cfg.d, cfg.n_routed
    dx = torch.full((cfg.T, d), float("nan"), dtype=torch.bfloat16, device="cuda")
    dwr = torch.full((N, d), float("nan"), dtype=torch.float32, device="cuda")
    dwgu = torch.full((E, 2 * I, d), float("nan"), dtype=torch.float32, device="cuda")
    dwd = torch.full((E, d, I), float("nan"), dtype=torch.float32, device="cuda")
    if ab_saved is None:
        moe.moe_backward(desc, inp["x"], inp["w_r"], inp["bias"], inp["w_gu"], inp["w_down"], dh,
                         dx, dwr, dwgu, dwd, ws)
    else:
        moe.moe_backward_saved(desc, inp["x"], inp["w_r"], inp["bias"], inp["w_gu"],
                               inp["w_down"], dh, ab_saved, dx, dwr, dwgu, dwd, ws)
    st = moe.moe_last_device_status()
    return dx, dwr, dwgu, dwd, st


@pytest.mark.parametrize("saved", [False, True], ids=["recompute", "saved"])
@pytest.mark.parametrize("name", list(CASES))
def test_backward_parity(name, saved):
    """Both backward forms against the oracle: recomputing a | b from x, and
    reading the a | b that moe_forward_save kept."""
    cfg = CASES[name]
    moe.moe_last_device_status()
    inp = recipes.device_inputs(cfg)
    dh, dh64 = upstream(cfg)
    ab = None
    if saved:
        _, ab, st = forward_save(cfg, inp)
        assert st == moe.OK, moe.moe_status_string(st)
    dx, dwr, dwgu, dwd, st = run_backward(cfg, inp, dh, ab)
    assert st == moe.OK, moe.moe_status_string(st)
    # the selection the backward used: the forward's routing of the same inputs
    desc = moe.desc_from_config(cfg)
    ws = moe.workspace(desc)
    idx = torch.empty(cfg.T, cfg.top_k, dtype=torch.int32, device="cuda")
    w = torch.empty(cfg.T, cfg.top_k, dtype=torch.float32, device="cuda")
    counts = torch.empty(cfg.n_routed, dtype=torch.int32, device="cuda")
    moe.moe_route(desc, inp["x"], inp["w_r"], inp["bias"], idx, w, counts, ws)
    host = HostLayer(cfg)
    ref_route = host.route()
    g_idx = idx.cpu().numpy().astype(np.int64)
    check_routing(cfg, ref_route, g_idx, w.cpu().numpy().astype(np.float64),
                  counts.cpu().numpy())
    ref = mb.moe_backward(host.x, host.w_r, host.bias, host.expert, dh64, n_shared=cfg.n_shared,
                          gate=cfg.gate, top_k=cfg.top_k, n_group=cfg.n_group,
                          topk_group=cfg.topk_group, renorm=cfg.renorm,
                          route_scale=cfg.route_scale, idx_override=g_idx)
    E, I = cfg.n_experts, cfg.inter

    def whole_tensor_err(got_of, ref_of):
        """max |got - ref| / max |ref| over all experts, one expert at a time."""
        num = den = 0.0
        for e in range(E):
            got = f64(got_of(e))
            want = ref_of(e) if e in ref["experts"] else np.zeros_like(got)
            num = max(num, float(np.max(np.abs(got - want))))
            den = max(den, float(np.max(np.abs(want))))
        return num / den

    errs = {
        "dx": mo.max_abs_rel(f64(dx), ref["dx"]),
        "dw_router": mo.max_abs_rel(f64(dwr), ref["dw_r"]),
        "dw_gu": whole_tensor_err(lambda e: dwgu[e],
                                  lambda e: np.concatenate(ref["experts"][e][:2])),
        "dw_down": whole_tensor_err(lambda e: dwd[e], lambda e: ref["experts"][e][2]),
    }
    print(f"{name}: " + ", ".join(f"{k} {v:.2e}" for k, v in errs.items()))
    # experts that no token reaches get exactly zero weight gradients
    untouched = [cfg.n_shared + j for j in range(cfg.n_routed) if not np.any(g_idx == j)]
    if untouched:
        assert torch.count_nonzero(dwgu[untouched]) == 0
        assert torch.count_nonzero(dwd[untouched]) == 0
    for k, v in errs.items():
        assert v <= TOL, f"{k}: max-abs-rel {v:.3e} above {TOL}"


def test_backward_is_deterministic():
    cfg = CASES["v3_small"]
    inp = recipes.device_inputs(cfg)
    dh, _ = upstream(cfg)
    a = run_backward(cfg, inp, dh)
    b = run_backward(cfg, inp, dh)
    assert a[4] == moe.OK and b[4] == moe.OK
    for x, y in zip(a[:4], b[:4]):
        assert torch.equal(x, y)


@pytest.mark.parametrize("name", ["v3_small", "dsmoe16b_small", "v3_T1"])
def test_backward_bf16_weight_gradients(name):
    """moe_backward_bf16_grads (weight gradients kept in BF16, as §3.6 keeps
    them): the same fp32 accumulators rounded to nearest even, so each bf16
    gradient equals the fp32 call's gradient cast to bf16 bit for bit, and dx
    is unchanged."""
    cfg = CASES[name]
    moe.moe_last_device_status()
    inp = recipes.device_inputs(cfg)
    dh, _ = upstream(cfg)
    dx, dwr, dwgu, dwd, st = run_backward(cfg, inp, dh)
    assert st == moe.OK
    desc = moe.desc_from_config(cfg)
    ws = moe.backward_workspace(desc)
    E, I, d, N = cfg.n_experts, cfg.inter, cfg.d, cfg.n_routed
    bf = dict(dtype=torch.bfloat16, device="cuda")
    dx2 = torch.full((cfg.T, d), float("nan"), **bf)
    dwr2 = torch.full((N, d), float("nan"), **bf)
    dwgu2 = torch.full((E, 2 * I, d), float("nan"), **bf)
    dwd2 = torch.full((E, d, I), float("nan"), **bf)
    moe.moe_backward_bf16_grads(desc, inp["x"], inp["w_r"], inp["bias"], inp["w_gu"],
                                inp["w_down"], dh, dx2, dwr2, dwgu2, dwd2, ws)
    assert moe.moe_last_device_status() == moe.OK
    assert torch.equal(dx2, dx)
    for got, ref in ((dwr2, dwr), (dwgu2, dwgu), (dwd2, dwd)):
        assert torch.equal(got, ref.to(torch.bfloat16))


@pytest.mark.parametrize("name", ["v3_small", "dsmoe16b_small", "v3_T1"])
def test_forward_save(name):
    """moe_forward_save: h is moe_forward's bit for bit, and ab_saved holds the
    pre-activations a = u W_gate^T, b = u W_up^T of every routed pair in the
    permuted row order (moe_permute's slot_of), then every shared expert's T
    rows, within bf16 rounding of the fp64 oracle."""
    cfg = CASES[name]
    moe.moe_last_device_status()
    inp = recipes.device_inputs(cfg)
    h_save, ab, st = forward_save(cfg, inp)
    assert st == moe.OK, moe.moe_status_string(st)
    desc = moe.desc_from_config(cfg)
    ws = moe.workspace(desc)
    h = torch.empty_like(h_save)
    moe.moe_forward(desc, inp["x"], None, inp["w_r"], inp["bias"], inp["w_gu"], None,
                    inp["w_down"], None, h, None, None, ws)
    assert moe.moe_last_device_status() == moe.OK
    assert torch.equal(h, h_save)
    # the row order: the permutation of the GPU's own routing
    T, K, Ks, I = cfg.T, cfg.top_k, cfg.n_shared, cfg.inter
    idx = torch.empty(T, K, dtype=torch.int32, device="cuda")
    w = torch.empty(T, K, dtype=torch.float32, device="cuda")
    counts = torch.empty(cfg.n_routed, dtype=torch.int32, device="cuda")
    moe.moe_route(desc, inp["x"], inp["w_r"], inp["bias"], idx, w, counts, ws)
    offsets = torch.empty(cfg.n_routed + 1, dtype=torch.int32, device="cuda")
    perm_src = torch.empty(T * K, dtype=torch.int32, device="cuda")
    slot_of = torch.empty(T * K, dtype=torch.int32, device="cuda")
    x_perm = torch.empty(T * K, cfg.d, dtype=torch.bfloat16, device="cuda")
    moe.moe_permute(desc, inp["x"], idx, counts, offsets, perm_src, slot_of, x_perm, None, ws)
    assert moe.moe_last_device_status() == moe.OK
    host = HostLayer(cfg)
    g_idx = idx.cpu().numpy().astype(np.int64)
    slots = slot_of.cpu().numpy().astype(np.int64)
    got = f64(ab)
    assert not np.isnan(got).any()
    num = den = 0.0
    flat = g_idx.reshape(-1)
    for j in np.unique(flat):
        pairs = np.nonzero(flat == j)[0]
        wg, wu, _ = host.expert(Ks + int(j))
        xt = host.x[pairs // K]
        want = np.concatenate([xt @ wg.T, xt @ wu.T], axis=1)
        num = max(num, float(np.max(np.abs(got[slots[pairs]] - want))))
        den = max(den, float(np.max(np.abs(want))))
    for s_ in range(Ks):
        wg, wu, _ = host.expert(s_)
        want = np.concatenate([host.x @ wg.T, host.x @ wu.T], axis=1)
        rows = got[T * K + s_ * T: T * K + (s_ + 1) * T]
        num = max(num, float(np.max(np.abs(rows - want))))
        den = max(den, float(np.max(np.abs(want))))
    assert num / den <= 1e-2, f"saved a | b: max-abs-rel {num / den:.3e}"


@pytest.mark.parametrize("name", ["v3_small", "v3_T1"])
def test_backward_saved_matches_recompute(name):
    """moe_backward_saved against moe_backward on the same inputs: both read
    bf16 pre-activations of the same products (kept by the forward or
    recomputed), so the gradients agree to bf16 rounding; the bf16-gradient
    form of the saved call rounds the same accumulators."""
    cfg = CASES[name]
    moe.moe_last_device_status()
    inp = recipes.device_inputs(cfg)
    dh, _ = upstream(cfg)
    _, ab, st = forward_save(cfg, inp)
    assert st == moe.OK
    ref = run_backward(cfg, inp, dh)
    got = run_backward(cfg, inp, dh, ab)
    assert ref[4] == moe.OK and got[4] == moe.OK
    for a, b in zip(got[:4], ref[:4]):
        a64, b64 = f64(a), f64(b)
        den = max(float(np.max(np.abs(b64))), 1e-30)
        assert float(np.max(np.abs(a64 - b64))) / den <= 1e-2
    desc = moe.desc_from_config(cfg)
    ws = moe.backward_workspace(desc)
    E, I, d, N = cfg.n_experts, cfg.inter, cfg.d, cfg.n_routed
    bf = dict(dtype=torch.bfloat16, device="cuda")
    dx2 = torch.full((cfg.T, d), float("nan"), **bf)
    dwr2 = torch.full((N, d), float("nan"), **bf)
    dwgu2 = torch.full((E, 2 * I, d), float("nan"), **bf)
    dwd2 = torch.full((E, d, I), float("nan"), **bf)
    moe.moe_backward_saved(desc, inp["x"], inp["w_r"], inp["bias"], inp["w_gu"], inp["w_down"],
                           dh, ab, dx2, dwr2, dwgu2, dwd2, ws, bf16_grads=True)
    assert moe.moe_last_device_status() == moe.OK
    assert torch.equal(dx2, got[0])
    for a, b in ((dwr2, got[1]), (dwgu2, got[2]), (dwd2, got[3])):
        assert torch.equal(a, b.to(torch.bfloat16))
