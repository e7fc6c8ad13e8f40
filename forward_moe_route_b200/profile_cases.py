"""Launch every kernel of the library on small cases, for a profiler.

    python -m forward_moe_route_b200.profile_cases [--only route]

Each case runs twice (the second launch of each kernel is the warm one) and
keeps a few GB on the device at most, so a per-kernel profiler capture of the
whole run ends in minutes:
  route     routing and permutation at the V3 shape (T = 16384, d = 7168,
            N = 256, top-8, 8 groups / top-4) with narrow experts (I = 128)
  v3        the V3-shaped bf16 layer (d = 7168, I = 2048) with 32 routed
            experts and T = 4096: forward, balance statistics, bias update,
            the expert-parallel entry points on one rank
  fp8       the same layer with E4M3 experts
  tiny      the tiny fp32 layer (tf32 GEMMs, fp32 router)
  backward  the V3-shaped layer with 8 routed experts, T = 2048
  ep        the v3 case's layer (bf16, then E4M3) over two expert-parallel
            ranks emulated on one GPU, exchanging over peer memory (local
            addresses): peer dispatch, expert GEMMs with per-group output
            addresses, the FP8 dispatch and row quantisation
  backward_bf16  the backward case with bf16 weight gradients
  backward_saved the backward case reading the pre-activations the forward kept
  backward_fp8   the backward case's shape as an E4M3 layer, FP8 GEMMs
Inputs come from the seeded synthetic generator (synth/).
"""
import argparse
import dataclasses

import torch

import forward_moe_route_b200 as moe
from forward_moe_route_b200 import ep
from synth import recipes

C = recipes.CONFIGS


def _forward(cfg, inp):
    desc = moe.desc_from_config(cfg)
    ws = moe.workspace(desc)
    h = torch.empty(cfg.T, cfg.d, dtype=inp["x"].dtype, device="cuda")
    moe.moe_forward(desc, inp["x"], None, inp["w_r"], inp["bias"], inp["w_gu"],
                    inp.get("w_gu_scale"), inp["w_down"], inp.get("w_down_scale"), h, None, None,
                    ws)
    return desc, ws


def case_route():
    cfg = recipes.small_variant(C["v3_bf16"], T=16384, d=7168, inter=128)
    inp = recipes.device_inputs(cfg)
    desc = moe.desc_from_config(cfg)
    ws = moe.workspace(desc)
    T, K, N = cfg.T, cfg.top_k, cfg.n_routed
    idx = torch.empty(T, K, dtype=torch.int32, device="cuda")
    w = torch.empty(T, K, dtype=torch.float32, device="cuda")
    counts = torch.empty(N, dtype=torch.int32, device="cuda")
    offsets = torch.empty(N + 1, dtype=torch.int32, device="cuda")
    ps = torch.empty(T * K, dtype=torch.int32, device="cuda")
    so = torch.empty(T * K, dtype=torch.int32, device="cuda")
    xp = torch.empty(T * K, cfg.d, dtype=torch.bfloat16, device="cuda")
    for _ in range(2):
        moe.moe_route(desc, inp["x"], inp["w_r"], inp["bias"], idx, w, counts, ws)
        moe.moe_permute(desc, inp["x"], idx, counts, offsets, ps, so, xp, None, ws)
    torch.cuda.synchronize()


def case_v3():
    cfg = dataclasses.replace(
        recipes.small_variant(C["v3_bf16"], T=4096, d=7168, inter=2048, n_routed=32),
        n_group=8, topk_group=4)
    inp = recipes.device_inputs(cfg)
    for _ in range(2):
        desc, ws = _forward(cfg, inp)
    s_out = torch.empty(cfg.T, cfg.n_routed, dtype=torch.float32, device="cuda")
    idx = torch.empty(cfg.T, cfg.top_k, dtype=torch.int32, device="cuda")
    w = torch.empty(cfg.T, cfg.top_k, dtype=torch.float32, device="cuda")
    counts = torch.empty(cfg.n_routed, dtype=torch.int32, device="cuda")
    f = torch.empty(cfg.T // 1024, cfg.n_routed, dtype=torch.float32, device="cuda")
    p = torch.empty_like(f)
    for _ in range(2):
        moe.moe_route(desc, inp["x"], inp["w_r"], inp["bias"], idx, w, counts, ws)
        moe.moe_route_affinities(desc, inp["x"], inp["w_r"], s_out, ws)
        moe.moe_balance_stats(desc, s_out, idx, 1024, f, p)
        moe.moe_bias_update(desc, counts, inp["bias"], 0.001)
    pl = ep.Placement(cfg.n_routed, 1)
    for _ in range(2):
        st = ep.ep_dispatch(desc, pl, 0, inp["x"], inp["w_r"], inp["bias"], ws)
        y = ep.ep_compute(desc, pl, st, st.plan.send_counts, st.x_send, st.w_send, inp["w_gu"],
                          inp["w_down"])
        ep.ep_combine(desc, st, inp["x"], None, y, inp["w_gu"], inp["w_down"])
    torch.cuda.synchronize()


def case_fp8():
    cfg = dataclasses.replace(
        recipes.small_variant(C["v3_fp8"], T=4096, d=7168, inter=2048, n_routed=32),
        n_group=8, topk_group=4)
    inp = recipes.device_inputs(cfg)
    E, I, d = cfg.n_experts, cfg.inter, cfg.d
    gq = torch.empty(E, 2 * I, d, dtype=torch.uint8, device="cuda")
    gs = torch.empty(E, 2 * I // 128, d // 128, dtype=torch.float32, device="cuda")
    dq = torch.empty(E, d, I, dtype=torch.uint8, device="cuda")
    ds = torch.empty(E, d // 128, I // 128, dtype=torch.float32, device="cuda")
    moe.moe_quantize_fp8_blockwise(inp["w_gu"], 2 * I, d, E, gq, gs)
    moe.moe_quantize_fp8_blockwise(inp["w_down"], d, I, E, dq, ds)
    inp.update(w_gu=gq, w_gu_scale=gs, w_down=dq, w_down_scale=ds)
    for _ in range(2):
        _forward(cfg, inp)
    torch.cuda.synchronize()


def case_tiny():
    cfg = C["tiny_f32"]
    inp = recipes.device_inputs(cfg)
    for _ in range(2):
        _forward(cfg, inp)
    torch.cuda.synchronize()


def case_backward():
    import synth
    cfg = dataclasses.replace(
        recipes.small_variant(C["v3_bf16"], T=2048, d=7168, inter=2048, n_routed=8),
        n_group=4, topk_group=2, top_k=4)
    inp = recipes.device_inputs(cfg)
    desc = moe.desc_from_config(cfg)
    ws = moe.backward_workspace(desc)
    dh32 = torch.empty(cfg.T, cfg.d, dtype=torch.float32, device="cuda")
    synth.dev_fill_normal(dh32, 1.0, cfg.seed, 6)
    dh = dh32.to(torch.bfloat16)
    dx = torch.empty_like(dh)
    E, I, d, N = cfg.n_experts, cfg.inter, cfg.d, cfg.n_routed
    dwr = torch.empty(N, d, dtype=torch.float32, device="cuda")
    dwgu = torch.empty(E, 2 * I, d, dtype=torch.float32, device="cuda")
    dwd = torch.empty(E, d, I, dtype=torch.float32, device="cuda")
    for _ in range(2):
        moe.moe_backward(desc, inp["x"], inp["w_r"], inp["bias"], inp["w_gu"], inp["w_down"], dh,
                         dx, dwr, dwgu, dwd, ws)
    torch.cuda.synchronize()


def _quantised_weights(cfg, inp):
    E, I, d = cfg.n_experts, cfg.inter, cfg.d
    gq = torch.empty(E, 2 * I, d, dtype=torch.uint8, device="cuda")
    gs = torch.empty(E, 2 * I // 128, d // 128, dtype=torch.float32, device="cuda")
    dq = torch.empty(E, d, I, dtype=torch.uint8, device="cuda")
    ds = torch.empty(E, d // 128, I // 128, dtype=torch.float32, device="cuda")
    moe.moe_quantize_fp8_blockwise(inp["w_gu"], 2 * I, d, E, gq, gs)
    moe.moe_quantize_fp8_blockwise(inp["w_down"], d, I, E, dq, ds)
    inp.update(w_gu=gq, w_gu_scale=gs, w_down=dq, w_down_scale=ds)


def case_ep():
    import numpy as np
    for dtype in ("bf16", "e4m3"):
        cfg = dataclasses.replace(
            recipes.small_variant(C["v3_bf16"], T=4096, d=7168, inter=2048, n_routed=32),
            n_group=8, topk_group=4, dtype=dtype)
        inp = recipes.device_inputs(cfg)
        fp8 = dtype == "e4m3"
        if fp8:
            _quantised_weights(cfg, inp)
        W = 2
        pl = ep.Placement(cfg.n_routed, W)
        full = (inp["w_gu"], inp["w_down"]) + \
            ((inp["w_gu_scale"], inp["w_down_scale"]) if fp8 else ())
        weights = [ep.local_weights(pl, r, cfg.n_shared, *full) for r in range(W)]
        half = cfg.T // W
        descs = [moe.desc_from_config(dataclasses.replace(cfg, T=half)) for _ in range(W)]
        xs = [inp["x"][r * half:(r + 1) * half].contiguous() for r in range(W)]
        for _ in range(2):
            steps = [ep.ep_dispatch(descs[r], pl, r, xs[r], inp["w_r"], inp["bias"],
                                    build_send=False) for r in range(W)]
            M = np.stack([st.plan.send_counts for st in steps])
            cap = int(M.sum(axis=(0, 2)).max())
            exs = [ep.PeerExchange(descs[r], pl, r, cap, "cuda", torch.bfloat16)
                   for r in range(W)]
            ep.PeerExchange.link(exs)
            for r in range(W):
                ep.peer_dispatch(descs[r], exs[r], steps[r], xs[r], M)
            for r in range(W):
                ep.peer_compute(descs[r], exs[r], steps[r], M, *weights[r])
            for r in range(W):
                ep.peer_combine(descs[r], exs[r], steps[r], xs[r], None, *weights[r])
        torch.cuda.synchronize()
        del inp, weights, exs
        torch.cuda.empty_cache()


def case_backward_bf16():
    import synth
    cfg = dataclasses.replace(
        recipes.small_variant(C["v3_bf16"], T=2048, d=7168, inter=2048, n_routed=8),
        n_group=4, topk_group=2, top_k=4)
    inp = recipes.device_inputs(cfg)
    desc = moe.desc_from_config(cfg)
    ws = moe.backward_workspace(desc)
    dh32 = torch.empty(cfg.T, cfg.d, dtype=torch.float32, device="cuda")
    synth.dev_fill_normal(dh32, 1.0, cfg.seed, 6)
    dh = dh32.to(torch.bfloat16)
    dx = torch.empty_like(dh)
    E, I, d, N = cfg.n_experts, cfg.inter, cfg.d, cfg.n_routed
    bf = dict(dtype=torch.bfloat16, device="cuda")
    dwr = torch.empty(N, d, **bf)
    dwgu = torch.empty(E, 2 * I, d, **bf)
    dwd = torch.empty(E, d, I, **bf)
    for _ in range(2):
        moe.moe_backward_bf16_grads(desc, inp["x"], inp["w_r"], inp["bias"], inp["w_gu"],
                                    inp["w_down"], dh, dx, dwr, dwgu, dwd, ws)
    torch.cuda.synchronize()


def _backward_case(dtype):
    import synth
    cfg = dataclasses.replace(
        recipes.small_variant(C["v3_fp8" if dtype == "e4m3" else "v3_bf16"], T=2048, d=7168,
                              inter=2048, n_routed=8),
        n_group=4, topk_group=2, top_k=4)
    inp = recipes.device_inputs(cfg)
    dh32 = torch.empty(cfg.T, cfg.d, dtype=torch.float32, device="cuda")
    synth.dev_fill_normal(dh32, 1.0, cfg.seed, 6)
    return cfg, inp, dh32.to(torch.bfloat16)


def case_backward_saved():
    cfg, inp, dh = _backward_case("bf16")
    desc = moe.desc_from_config(cfg)
    E, I, d, N = cfg.n_experts, cfg.inter, cfg.d, cfg.n_routed
    ab = torch.empty(moe.moe_saved_ab_bytes(desc) // 2, dtype=torch.bfloat16, device="cuda")
    h = torch.empty_like(dh)
    moe.moe_forward_save(desc, inp["x"], None, inp["w_r"], inp["bias"], inp["w_gu"],
                         inp["w_down"], h, None, None, ab, moe.workspace(desc))
    ws = moe.backward_workspace(desc)
    dx = torch.empty_like(dh)
    dwr = torch.empty(N, d, dtype=torch.float32, device="cuda")
    dwgu = torch.empty(E, 2 * I, d, dtype=torch.float32, device="cuda")
    dwd = torch.empty(E, d, I, dtype=torch.float32, device="cuda")
    for _ in range(2):
        moe.moe_backward_saved(desc, inp["x"], inp["w_r"], inp["bias"], inp["w_gu"],
                               inp["w_down"], dh, ab, dx, dwr, dwgu, dwd, ws)
    torch.cuda.synchronize()


def case_backward_fp8():
    cfg, inp, dh = _backward_case("e4m3")
    desc = moe.desc_from_config(cfg)
    E, I, d, N = cfg.n_experts, cfg.inter, cfg.d, cfg.n_routed

    W = moe.fp8_backward_weights(inp["w_gu"], inp["w_down"])
    ws = moe.backward_fp8_workspace(desc)
    bf = dict(dtype=torch.bfloat16, device="cuda")
    dx = torch.empty_like(dh)
    dwr = torch.empty(N, d, **bf)
    dwgu = torch.empty(E, 2 * I, d, **bf)
    dwd = torch.empty(E, d, I, **bf)
    for _ in range(2):
        moe.moe_backward_fp8(desc, inp["x"], inp["w_r"], inp["bias"], *W, dh, dx, dwr, dwgu,
                             dwd, ws)
    torch.cuda.synchronize()


CASES = {"route": case_route, "v3": case_v3, "fp8": case_fp8, "tiny": case_tiny,
         "backward": case_backward, "ep": case_ep, "backward_bf16": case_backward_bf16,
         "backward_saved": case_backward_saved, "backward_fp8": case_backward_fp8}


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--only", choices=list(CASES), nargs="*")
    args = ap.parse_args()
    torch.cuda.set_device(0)
    for name in args.only or list(CASES):
        CASES[name]()
        torch.cuda.empty_cache()
        st = moe.moe_last_device_status()
        if st != moe.OK:
            raise SystemExit(f"{name}: device status {moe.moe_status_string(st)}")
    print("profile cases ok")


if __name__ == "__main__":
    main()
