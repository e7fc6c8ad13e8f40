"""moe_permute_noalloc: the permutation for callers that cannot allocate device
memory (a host framework that owns all device memory and hands an operator no
scratch buffer, or a C caller holding only the layer's inputs and outputs).

It must give exactly what moe_permute gives with a caller-provided workspace:
offsets, perm_src and slot_of are integers and the gathered rows are byte
copies, so the comparison is bit for bit.  Two calls in a row with different
routings check that the shared fixed scratch carries nothing from one call
into the next.  This file is collected last on purpose.
"""
import ctypes

import pytest
import torch

import forward_moe_route_b200 as moe
from synth import recipes


def _route(cfg, inp):
    desc = moe.desc_from_config(cfg)
    ws = moe.workspace(desc)
    T, K, N = cfg.T, cfg.top_k, cfg.n_routed
    idx = torch.empty(T, K, dtype=torch.int32, device="cuda")
    w = torch.empty(T, K, dtype=torch.float32, device="cuda")
    counts = torch.empty(N, dtype=torch.int32, device="cuda")
    moe.moe_route(desc, inp["x"], inp["w_r"], inp["bias"], idx, w, counts, ws)
    return desc, ws, idx, counts


def _outputs(cfg):
    T, K, N, d = cfg.T, cfg.top_k, cfg.n_routed, cfg.d
    i32 = dict(dtype=torch.int32, device="cuda")
    return (torch.full((N + 1,), -1, **i32), torch.full((T * K,), -1, **i32),
            torch.full((T * K,), -1, **i32),
            torch.zeros(T * K, d, dtype=torch.bfloat16, device="cuda"))


@pytest.mark.gpu
def test_noalloc_permute_matches_workspace_permute_twice():
    base = recipes.CONFIGS["v3_bf16"]
    cfgs = [recipes.small_variant(base, T=1500, d=512, inter=256),
            recipes.small_variant(base, T=700, d=512, inter=256)]
    for call, cfg in enumerate(cfgs):
        inp = recipes.device_inputs(cfg)
        if call == 1:
            inp["bias"][8:16] += 0.5       # a different routing on the second call
        desc, ws, idx, counts = _route(cfg, inp)
        ref = _outputs(cfg)
        moe.moe_permute(desc, inp["x"], idx, counts, *ref, None, ws)
        got = _outputs(cfg)
        moe.moe_permute_noalloc(desc, inp["x"], idx, counts, *got, None)
        assert moe.moe_last_device_status() == moe.OK
        for a, b in zip(ref, got):
            assert torch.equal(a, b), f"call {call}: no-alloc result differs"


@pytest.mark.gpu
def test_noalloc_permute_e4m3_and_empty_batch():
    # E4M3 layer: the quantising gather (codes and 1x128 scales, rows R..R+T-1
    # holding x in token order) must match the workspace path byte for byte
    cfg = recipes.small_variant(recipes.CONFIGS["v3_fp8"], T=300, d=512, inter=256)
    inp = recipes.device_inputs(cfg)
    desc, ws, idx, counts = _route(cfg, inp)
    T, K, N, d = cfg.T, cfg.top_k, cfg.n_routed, cfg.d
    rows = T * K + T

    def outs():
        i32 = dict(dtype=torch.int32, device="cuda")
        return (torch.full((N + 1,), -1, **i32), torch.full((T * K,), -1, **i32),
                torch.full((T * K,), -1, **i32),
                torch.zeros(rows, d, dtype=torch.uint8, device="cuda"),
                torch.zeros(rows, d // 128, dtype=torch.float32, device="cuda"))
    ref, got = outs(), outs()
    moe.moe_permute(desc, inp["x"], idx, counts, *ref, ws)
    moe.moe_permute_noalloc(desc, inp["x"], idx, counts, *got)
    assert moe.moe_last_device_status() == moe.OK
    for a, b in zip(ref, got):
        assert torch.equal(a, b), "no-alloc E4M3 result differs"
    # T = 0: offsets are all zero, nothing else is touched
    empty = moe.make_desc(0, 512, 1, 32, 8, 256, "sigmoid", True, 2.5, 4, 2, "bf16")
    offsets = torch.full((33,), -1, dtype=torch.int32, device="cuda")
    dummy = torch.zeros(64, dtype=torch.int32, device="cuda")   # >= N int32 for counts
    moe.moe_permute_noalloc(empty, dummy, dummy, dummy, offsets, dummy, dummy, dummy, None)
    assert moe.moe_last_device_status() == moe.OK
    assert torch.count_nonzero(offsets) == 0


def test_noalloc_rejects_shapes_beyond_the_fixed_scratch():
    # ceil(T/128) * N above MOE_NOALLOC_HIST_INTS is refused before any CUDA call
    big = moe.make_desc(131073, 7168, 1, 256, 8, 2048, "sigmoid", True, 2.5, 8, 4, "bf16")
    rc = moe.lib().moe_permute_noalloc(ctypes.byref(big), 16, 16, 16, 16, 16, 16, 16, None, None)
    assert rc == moe.ERR_UNSUPPORTED
    assert b"fixed scratch" in moe.lib().moe_last_error_message()
    ok = moe.make_desc(131072, 7168, 1, 256, 8, 2048, "sigmoid", True, 2.5, 8, 4, "bf16")
    assert moe.moe_workspace_size(ok) > 0
