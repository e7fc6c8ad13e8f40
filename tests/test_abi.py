"""The C ABI library: it loads, exports every symbol include/moe.h declares,
and its host-side validation rejects bad problem statements (no GPU needed:
these calls return before touching CUDA)."""
import ctypes
import os
import re

import pytest

import forward_moe_route_b200 as moe

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def declared_functions():
    with open(os.path.join(ROOT, "include", "moe.h")) as f:
        text = f.read()
    text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
    names = re.findall(r"^\s*(?:const\s+)?[a-z_0-9]+\s*\*?\s+(moe_[a-z_0-9]+)\s*\(", text, re.M)
    return sorted(set(names))


def test_every_declared_symbol_is_exported():
    names = declared_functions()
    assert len(names) >= 11
    for n in names:
        assert hasattr(moe.lib(), n), f"{n} declared but not exported"
    assert set(names) == set(moe.EXPORTED)


def test_desc_struct_matches_header_layout():
    # 13 four-byte fields, no padding
    assert ctypes.sizeof(moe.MoeLayerDesc) == 13 * 4


def v3(**kw):
    base = dict(T=16384, d=7168, n_shared=1, n_routed=256, top_k=8, inter=2048, gate="sigmoid",
                renorm=True, route_scale=2.5, n_group=8, topk_group=4, dtype="bf16")
    base.update(kw)
    return moe.make_desc(**base)


def test_workspace_size_valid_configs():
    assert moe.moe_workspace_size(v3()) > 4e9
    assert moe.moe_workspace_size(v3(dtype="e4m3")) > 0
    tiny = moe.make_desc(64, 256, 1, 16, 4, 64, "softmax", True, 1.0, 1, 1, "f32")
    assert moe.moe_workspace_size(tiny) > 0
    assert moe.moe_workspace_size(v3(T=0)) > 0


@pytest.mark.parametrize("kw", [
    dict(top_k=300),                      # K > N
    dict(top_k=17),                       # K above the supported maximum
    dict(n_group=8, topk_group=1),        # 1 group of 32 experts < K? (32 >= 8: valid) -> see below
    dict(n_group=7),                      # N not divisible by n_group
    dict(n_group=8, topk_group=9),        # topk_group > n_group
    dict(n_routed=16, n_group=16, topk_group=3, top_k=8),  # groups of 1 expert
    dict(d=7100),                         # d not a multiple of 64 (bf16)
    dict(inter=8),
    dict(dtype="e4m3", d=7168 + 64),      # FP8 needs multiples of 128
    dict(T=-1),
    dict(route_scale=0.0),
    dict(route_scale=float("nan")),
    dict(n_routed=0),
    dict(n_routed=1024, n_group=1, topk_group=1),
    dict(n_shared=65),
])
def test_invalid_descriptors(kw):
    d = v3(**kw)
    if kw == dict(n_group=8, topk_group=1):
        assert moe.moe_workspace_size(d) > 0   # 1 group of 32 experts holds K=8: valid
        return
    assert moe.moe_workspace_size(d) == 0


def test_group_capacity_rule():
    # topk_group * (N / n_group) must be >= K
    assert moe.moe_workspace_size(v3(n_routed=32, n_group=8, topk_group=1, top_k=8)) == 0
    assert moe.moe_workspace_size(v3(n_routed=32, n_group=8, topk_group=2, top_k=8)) > 0


def test_bad_dtype_pair():
    d = v3()
    d.act_dtype, d.w_dtype = moe.DT_E4M3, moe.DT_E4M3
    assert moe.moe_workspace_size(d) == 0
    d.act_dtype, d.w_dtype = moe.DT_F32, moe.DT_BF16
    assert moe.moe_workspace_size(d) == 0


def test_entry_points_reject_before_touching_cuda():
    L = moe.lib()
    bad = v3(top_k=300)
    assert L.moe_route(ctypes.byref(bad), None, None, None, None, None, None, None, 0,
                       None) == moe.ERR_INVALID_ARG
    good = v3()
    # bias with softmax gating is not part of the method
    sm = v3(gate="softmax", n_group=1, topk_group=1)
    assert L.moe_route(ctypes.byref(sm), 16, 16, 16, 16, 16, 16, 16, 1 << 40,
                       None) == moe.ERR_INVALID_ARG
    # null / misaligned pointers
    assert L.moe_route(ctypes.byref(good), None, 16, None, 16, 16, 16, 16, 1 << 40,
                       None) == moe.ERR_INVALID_ARG
    assert L.moe_route(ctypes.byref(good), 17, 16, None, 16, 16, 16, 16, 1 << 40,
                       None) == moe.ERR_INVALID_ARG
    # workspace too small
    assert L.moe_route(ctypes.byref(good), 16, 16, None, 16, 16, 16, 16, 1024,
                       None) == moe.ERR_WORKSPACE
    assert L.moe_forward(ctypes.byref(good), 16, None, 16, None, 16, None, 16, None, 16, None,
                         None, 16, 1024, None) == moe.ERR_WORKSPACE
    # FP8 forward needs the weight scales
    f8 = v3(dtype="e4m3")
    assert L.moe_forward(ctypes.byref(f8), 16, None, 16, None, 16, None, 16, None, 16, None,
                         None, 16, 1 << 40, None) == moe.ERR_INVALID_ARG
    # permute: E4M3 needs the scale output, bf16 must not get one
    assert L.moe_permute(ctypes.byref(good), 16, 16, 16, 16, 16, 16, 16, 16, 16, 1 << 40,
                         None) == moe.ERR_INVALID_ARG
    assert L.moe_quantize_fp8_blockwise(16, 100, 128, 1, 16, 16, None) == moe.ERR_INVALID_ARG
    assert L.moe_selftest_bounded_wait(0, None) == moe.ERR_INVALID_ARG


def test_status_strings():
    for s in range(7):
        assert moe.moe_status_string(s)
    assert moe.moe_status_string(99) == "unknown status"


def test_launch_count():
    # router GEMM, top-K, histogram, scan, slots, gather, group table, GEMM1,
    # GEMM2, combine; fp32 routes in one kernel
    assert moe.moe_forward_launch_count(v3()) == 10
    assert moe.moe_forward_launch_count(v3(dtype="e4m3")) == 10
    assert moe.moe_forward_launch_count(v3(dtype="f32")) == 9
    assert moe.moe_forward_launch_count(v3(T=0)) == 2
    assert moe.moe_forward_launch_count(v3(top_k=300)) == 0
    # router GEMM, top-K, histogram, scan, slots, prep, gather, zero pads, the
    # six GEMMs G1, G2, G3, G6a, G4, G5, gate backward, combine, G6b (the
    # serialised launch list of `bench.py --backward` shows these 17 per pass)
    assert moe.moe_backward_launch_count(v3()) == 17
    assert moe.moe_backward_launch_count(v3(T=0)) == 0


def test_binding_refuses_short_or_strided_buffers():
    # the ABI takes plain pointers, so the binding checks every tensor against
    # the descriptor before calling in; CPU tensors suffice for the check
    import torch

    desc = moe.make_desc(T=64, d=256, n_shared=1, n_routed=16, top_k=4, inter=64,
                         gate="softmax", renorm=True, route_scale=1.0, dtype="bf16")
    E = 17
    x = torch.zeros(64, 256, dtype=torch.bfloat16)
    w_r = torch.zeros(16, 256, dtype=torch.bfloat16)
    w_gu = torch.zeros(E, 128, 256, dtype=torch.bfloat16)
    w_d = torch.zeros(E, 256, 64, dtype=torch.bfloat16)
    short_h = torch.zeros(63, 256, dtype=torch.bfloat16)
    with pytest.raises(moe.MoeError, match="h holds"):
        moe.moe_forward(desc, x, None, w_r, None, w_gu, None, w_d, None, short_h, None, None,
                        None)
    strided = torch.zeros(256, 64, dtype=torch.bfloat16).t()
    with pytest.raises(moe.MoeError, match="not contiguous"):
        moe.moe_forward(desc, strided, None, w_r, None, w_gu, None, w_d, None, x, None, None,
                        None)
    short_w = torch.zeros(E - 1, 128, 256, dtype=torch.bfloat16)
    x_perm = torch.zeros(64 * 4, 256, dtype=torch.bfloat16)
    with pytest.raises(moe.MoeError, match="w_gu holds"):
        moe.moe_grouped_swiglu(desc, x, x_perm, None, None, None, None, None, short_w, None, w_d,
                               None, None, None)
    fp8 = moe.make_desc(T=64, d=256, n_shared=1, n_routed=16, top_k=4, inter=128,
                        gate="softmax", renorm=True, route_scale=1.0, dtype="e4m3")
    xp = torch.zeros(64 * 4 + 64, 256, dtype=torch.uint8)
    short_scale = torch.zeros(64 * 4, 2, dtype=torch.float32)      # the T shared rows missing
    with pytest.raises(moe.MoeError, match="x_perm_scale holds"):
        moe.moe_permute(fp8, x, None, None, None, None, None, xp, short_scale, None)


def test_expert_parallel_entry_points_reject_bad_arguments():
    """The peer-memory, FP8 and IPC entry points refuse bad arguments on the
    host, before any CUDA call."""
    L = moe.lib()
    bf, f8 = v3(T=64), v3(T=64, dtype="e4m3")
    # peer dispatch: n_ranks out of range, start[] not ending at n_rows
    P = moe.MoePeerRows()
    P.n_ranks = 0
    assert L.moe_dispatch_rows_to(ctypes.byref(bf), 16, 16, 16, 64, ctypes.byref(P),
                                  None) == moe.ERR_INVALID_ARG
    P.n_ranks = moe.MAX_PEERS + 1
    assert L.moe_dispatch_rows_to(ctypes.byref(bf), 16, 16, 16, 64, ctypes.byref(P),
                                  None) == moe.ERR_INVALID_ARG
    P.n_ranks = 2
    P.start[0], P.start[1], P.start[2] = 0, 10, 20          # does not end at n_rows = 64
    P.x[0] = P.x[1] = 16
    assert L.moe_dispatch_rows_to(ctypes.byref(bf), 16, 16, 16, 64, ctypes.byref(P),
                                  None) == moe.ERR_INVALID_ARG
    P.start[2] = 64
    P.x[1] = 17                                              # misaligned destination
    assert L.moe_dispatch_rows_to(ctypes.byref(bf), 16, 16, 16, 64, ctypes.byref(P),
                                  None) == moe.ERR_INVALID_ARG
    P.x[1] = 16                                              # E4M3 rows need scale buffers
    assert L.moe_dispatch_rows_to(ctypes.byref(f8), 16, 16, 16, 64, ctypes.byref(P),
                                  None) == moe.ERR_INVALID_ARG
    # FP8 dispatch / quantisation only for E4M3 layers, with a scale output
    assert L.moe_dispatch_rows_fp8(ctypes.byref(bf), 16, 16, 16, 64, 16, 16, 16,
                                   None) == moe.ERR_INVALID_ARG
    assert L.moe_dispatch_rows_fp8(ctypes.byref(f8), 16, 16, 16, 64, 16, None, 16,
                                   None) == moe.ERR_INVALID_ARG
    assert L.moe_quantize_rows_fp8(ctypes.byref(bf), 16, 4, 16, 16, None) == moe.ERR_INVALID_ARG
    # FP8 expert FFN: exactly one of y_rows / group_out; bf16 layers go to moe_expert_ffn
    args = (1, 1, 16, 64, 64, 16, 16, 16, 16, 16, 16, 16)
    assert L.moe_expert_ffn_fp8(ctypes.byref(f8), *args, None, None, 16, 1 << 30,
                                None) == moe.ERR_INVALID_ARG
    assert L.moe_expert_ffn_fp8(ctypes.byref(f8), *args, 16, 16, 16, 1 << 30,
                                None) == moe.ERR_INVALID_ARG
    assert L.moe_expert_ffn_fp8(ctypes.byref(bf), *args, 16, None, 16, 1 << 30,
                                None) == moe.ERR_INVALID_ARG
    # per-group output addresses must be 8-byte aligned
    assert L.moe_expert_ffn_to(ctypes.byref(bf), 1, 1, 16, 64, 64, 16, 16, 16, 16, 12, 16,
                               1 << 30, None) == moe.ERR_INVALID_ARG
    # IPC: null pointers
    off = ctypes.c_uint64()
    assert L.moe_ipc_get_handle(None, ctypes.create_string_buffer(64),
                                ctypes.byref(off)) == moe.ERR_INVALID_ARG
    assert L.moe_ipc_open(None, None) == moe.ERR_INVALID_ARG
    assert L.moe_ipc_close(None) == moe.ERR_INVALID_ARG


def test_saved_activation_entry_points_reject_bad_arguments():
    """moe_forward_save / moe_backward_saved: bf16 layers only, a 16-byte
    aligned ab_saved of moe_saved_ab_bytes bytes, checked before any CUDA call."""
    L = moe.lib()
    bf = v3(T=64)
    T, K, Ks, I = bf.T, bf.top_k, bf.n_shared, bf.inter
    assert moe.moe_saved_ab_bytes(bf) == (T * K + Ks * T) * 2 * I * 2
    assert moe.moe_saved_ab_bytes(v3(dtype="e4m3")) == 0
    assert moe.moe_saved_ab_bytes(v3(dtype="f32")) == 0
    assert moe.moe_saved_ab_bytes(v3(top_k=300)) == 0
    fwd = (16, None, 16, None, 16, 16, 16, None, None)
    # no or misaligned ab_saved; FP8 and fp32 layers refused
    assert L.moe_forward_save(ctypes.byref(bf), *fwd, None, 16, 1 << 30,
                              None) == moe.ERR_INVALID_ARG
    assert L.moe_forward_save(ctypes.byref(bf), *fwd, 24, 16, 1 << 30,
                              None) == moe.ERR_INVALID_ARG
    assert L.moe_forward_save(ctypes.byref(v3(dtype="e4m3")), *fwd, 16, 16, 1 << 30,
                              None) == moe.ERR_UNSUPPORTED
    assert L.moe_forward_save(ctypes.byref(v3(dtype="f32")), *fwd, 16, 16, 1 << 30,
                              None) == moe.ERR_UNSUPPORTED
    bwd = (16, 16, None, 16, 16, 16)
    grads = (16, 16, 16, 16)
    assert L.moe_backward_saved(ctypes.byref(bf), *bwd, None, *grads, 0, 16, 1 << 40,
                                None) == moe.ERR_INVALID_ARG
    assert L.moe_backward_saved(ctypes.byref(bf), *bwd, 40, *grads, 0, 16, 1 << 40,
                                None) == moe.ERR_INVALID_ARG
    assert L.moe_backward_saved(ctypes.byref(v3(dtype="f32")), *bwd, 16, *grads, 0, 16,
                                1 << 40, None) == moe.ERR_UNSUPPORTED
    # the binding refuses a short ab_saved
    import torch
    x = torch.zeros(T, bf.d, dtype=torch.bfloat16)
    short = torch.zeros(T * K, 2 * I, dtype=torch.bfloat16)     # the shared rows missing
    with pytest.raises(moe.MoeError, match="ab_saved holds"):
        moe.moe_forward_save(bf, x, None, None, None, None, None, x, None, None, short, None)


def test_fp8_backward_entry_point_rejects_bad_arguments():
    """moe_backward_fp8: E4M3 layers only, d a multiple of 256, every pointer
    present and aligned, checked before any CUDA call."""
    L = moe.lib()
    f8 = v3(T=64, dtype="e4m3")
    assert moe.moe_backward_fp8_workspace_size(f8) > 0
    assert moe.moe_backward_fp8_workspace_size(v3(T=64)) == 0
    assert moe.moe_backward_fp8_launch_count(f8) == 22
    assert moe.moe_backward_fp8_launch_count(v3(T=0, dtype="e4m3")) == 0
    ptrs = [16] * 14          # x, w_router, bias, 6 weight pointers, dh, dx, 3 gradients
    ptrs[2] = None            # bias
    assert L.moe_backward_fp8(ctypes.byref(v3(T=64)), *ptrs, 16, 1 << 40,
                              None) == moe.ERR_UNSUPPORTED
    assert L.moe_backward_fp8(ctypes.byref(v3(T=64, d=7168 + 128, dtype="e4m3")), *ptrs, 16,
                              1 << 40, None) == moe.ERR_UNSUPPORTED
    for i in (0, 3, 5, 8, 9, 13):         # a missing tensor or scale
        bad = list(ptrs)
        bad[i] = None
        assert L.moe_backward_fp8(ctypes.byref(f8), *bad, 16, 1 << 40,
                                  None) == moe.ERR_INVALID_ARG
    bad = list(ptrs)
    bad[5] = 24                           # a misaligned transposed weight (w_gu_t)
    assert L.moe_backward_fp8(ctypes.byref(f8), *bad, 16, 1 << 40, None) == moe.ERR_INVALID_ARG
    bad = list(ptrs)
    bad[4] = 18                           # a scale (w_gu_scale) not 4-byte aligned
    assert L.moe_backward_fp8(ctypes.byref(f8), *bad, 16, 1 << 40, None) == moe.ERR_INVALID_ARG
    assert L.moe_backward_fp8(ctypes.byref(f8), *ptrs, 16, 1024, None) == moe.ERR_WORKSPACE


def test_transposed_weight_quantisation_rejects_bad_arguments():
    L = moe.lib()
    assert L.moe_quantize_fp8_blockwise_t(16, 100, 128, 1, 16, 16, None) == moe.ERR_INVALID_ARG
    assert L.moe_quantize_fp8_blockwise_t(16, 128, 128, 0, 16, 16, None) == moe.ERR_INVALID_ARG
    assert L.moe_quantize_fp8_blockwise_t(16, 128, 128, 1, 24, 16, None) == moe.ERR_INVALID_ARG
    assert L.moe_quantize_fp8_blockwise_t(None, 128, 128, 1, 16, 16, None) == moe.ERR_INVALID_ARG
