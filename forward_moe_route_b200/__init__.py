"""Python binding of the B200 DeepSeekMoE layer-forward library (libmoe_b200.so).

Argument marshalling only: every function here forwards torch tensors' device
pointers and the current CUDA stream to the C ABI of the same name
(include/moe.h) and turns a non-OK status into MoeError.  Because the ABI
takes plain pointers, the binding first checks that each tensor argument is
contiguous and holds at least the bytes the descriptor implies, and refuses a
short or strided buffer instead of letting a kernel overrun it.  All
computation runs in the library's CUDA kernels; there is no fallback.
Importing this package fails loudly if the compiled library is missing.
"""
from __future__ import annotations

import ctypes
import os
from typing import Optional

_HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_HERE, "libmoe_b200.so")

if not os.path.exists(LIB_PATH):
    raise ImportError(
        f"{LIB_PATH} is missing: build it with `python forward_moe_route_b200/build.py` "
        "(nvcc, sm_100a). The layer has no CPU or Python fallback.")

_lib = ctypes.CDLL(LIB_PATH)

# status codes (moe_status)
OK, ERR_INVALID_ARG, ERR_UNSUPPORTED, ERR_WORKSPACE, ERR_CUDA, ERR_TIMEOUT, ERR_DEVICE_CHECK = \
    range(7)
GATE_SOFTMAX, GATE_SIGMOID = 0, 1
DT_F32, DT_BF16, DT_E4M3 = 0, 1, 2


class MoeLayerDesc(ctypes.Structure):
    _fields_ = [("T", ctypes.c_int32), ("d", ctypes.c_int32), ("n_shared", ctypes.c_int32),
                ("n_routed", ctypes.c_int32), ("top_k", ctypes.c_int32),
                ("inter", ctypes.c_int32), ("gate", ctypes.c_int32), ("renorm", ctypes.c_int32),
                ("route_scale", ctypes.c_float), ("n_group", ctypes.c_int32),
                ("topk_group", ctypes.c_int32), ("act_dtype", ctypes.c_int32),
                ("w_dtype", ctypes.c_int32)]


MAX_PEERS = 16
IPC_HANDLE_BYTES = 64


class MoePeerRows(ctypes.Structure):
    """moe_peer_rows: where the send-order rows of a peer dispatch land."""
    _fields_ = [("x", ctypes.c_void_p * MAX_PEERS), ("w", ctypes.c_void_p * MAX_PEERS),
                ("scale", ctypes.c_void_p * MAX_PEERS),
                ("start", ctypes.c_int32 * (MAX_PEERS + 1)), ("base", ctypes.c_int32 * MAX_PEERS),
                ("n_ranks", ctypes.c_int32)]


class MoeError(RuntimeError):
    def __init__(self, status: int, where: str):
        self.status = status
        super().__init__(f"{where}: {moe_status_string(status)} (status {status})")


_P = ctypes.c_void_p
_D = ctypes.POINTER(MoeLayerDesc)
_SIGS = {
    "moe_workspace_size": (ctypes.c_size_t, [_D]),
    "moe_route": (ctypes.c_int, [_D, _P, _P, _P, _P, _P, _P, _P, ctypes.c_size_t, _P]),
    "moe_permute": (ctypes.c_int, [_D, _P, _P, _P, _P, _P, _P, _P, _P, _P, ctypes.c_size_t, _P]),
    "moe_permute_noalloc": (ctypes.c_int, [_D, _P, _P, _P, _P, _P, _P, _P, _P, _P]),
    "moe_grouped_swiglu": (ctypes.c_int, [_D, _P, _P, _P, _P, _P, _P, _P, _P, _P, _P, _P, _P, _P,
                                          ctypes.c_size_t, _P]),
    "moe_combine": (ctypes.c_int, [_D, _P, _P, _P, _P]),
    "moe_forward": (ctypes.c_int, [_D, _P, _P, _P, _P, _P, _P, _P, _P, _P, _P, _P, _P,
                                   ctypes.c_size_t, _P]),
    "moe_route_affinities": (ctypes.c_int, [_D, _P, _P, _P, _P, ctypes.c_size_t, _P]),
    "moe_balance_stats": (ctypes.c_int, [_D, _P, _P, ctypes.c_int32, _P, _P, _P]),
    "moe_bias_update": (ctypes.c_int, [_D, _P, _P, ctypes.c_float, _P]),
    "moe_quantize_fp8_blockwise": (ctypes.c_int, [_P, ctypes.c_int32, ctypes.c_int32,
                                                  ctypes.c_int32, _P, _P, _P]),
    "moe_quantize_fp8_blockwise_t": (ctypes.c_int, [_P, ctypes.c_int32, ctypes.c_int32,
                                                    ctypes.c_int32, _P, _P, _P]),
    "moe_status_string": (ctypes.c_char_p, [ctypes.c_int]),
    "moe_last_device_status": (ctypes.c_int, [_P]),
    "moe_forward_launch_count": (ctypes.c_int32, [_D]),
    "moe_last_error_message": (ctypes.c_char_p, []),
    "moe_trace_events": (ctypes.c_int, [ctypes.POINTER(ctypes.c_void_p), ctypes.c_int32]),
    "moe_selftest_bounded_wait": (ctypes.c_int, [ctypes.c_uint32, _P]),
    "moe_backward_workspace_size": (ctypes.c_size_t, [_D]),
    "moe_backward": (ctypes.c_int, [_D, _P, _P, _P, _P, _P, _P, _P, _P, _P, _P, _P,
                                    ctypes.c_size_t, _P]),
    "moe_backward_launch_count": (ctypes.c_int32, [_D]),
    "moe_backward_bf16_grads": (ctypes.c_int, [_D, _P, _P, _P, _P, _P, _P, _P, _P, _P, _P, _P,
                                               ctypes.c_size_t, _P]),
    "moe_expert_ffn_workspace_size": (ctypes.c_size_t, [_D, ctypes.c_int32, ctypes.c_int32]),
    "moe_expert_ffn": (ctypes.c_int, [_D, ctypes.c_int32, ctypes.c_int32, _P, ctypes.c_int32,
                                      ctypes.c_int32, _P, _P, _P, _P, _P, _P, ctypes.c_size_t,
                                      _P]),
    "moe_combine_rows": (ctypes.c_int, [_D, _P, _P, _P, _P, ctypes.c_int32, _P, _P]),
    "moe_dispatch_rows": (ctypes.c_int, [_D, _P, _P, _P, ctypes.c_int32, _P, _P, _P]),
    "moe_dispatch_rows_to": (ctypes.c_int, [_D, _P, _P, _P, ctypes.c_int32, _P, _P]),
    "moe_expert_ffn_to": (ctypes.c_int, [_D, ctypes.c_int32, ctypes.c_int32, _P, ctypes.c_int32,
                                         ctypes.c_int32, _P, _P, _P, _P, _P, _P, ctypes.c_size_t,
                                         _P]),
    "moe_ipc_get_handle": (ctypes.c_int, [_P, _P, ctypes.POINTER(ctypes.c_uint64)]),
    "moe_dispatch_rows_fp8": (ctypes.c_int, [_D, _P, _P, _P, ctypes.c_int32, _P, _P, _P, _P]),
    "moe_quantize_rows_fp8": (ctypes.c_int, [_D, _P, ctypes.c_int32, _P, _P, _P]),
    "moe_expert_ffn_fp8": (ctypes.c_int, [_D, ctypes.c_int32, ctypes.c_int32, _P, ctypes.c_int32,
                                          ctypes.c_int32, _P, _P, _P, _P, _P, _P, _P, _P, _P,
                                          _P, ctypes.c_size_t, _P]),
    "moe_ipc_open": (ctypes.c_int, [_P, ctypes.POINTER(ctypes.c_void_p)]),
    "moe_ipc_close": (ctypes.c_int, [_P]),
    "moe_backward_fp8_workspace_size": (ctypes.c_size_t, [_D]),
    "moe_backward_fp8": (ctypes.c_int, [_D] + [_P] * 15 + [ctypes.c_size_t, _P]),
    "moe_backward_fp8_launch_count": (ctypes.c_int32, [_D]),
    "moe_saved_ab_bytes": (ctypes.c_size_t, [_D]),
    "moe_forward_save": (ctypes.c_int, [_D, _P, _P, _P, _P, _P, _P, _P, _P, _P, _P, _P,
                                        ctypes.c_size_t, _P]),
    "moe_backward_saved": (ctypes.c_int, [_D, _P, _P, _P, _P, _P, _P, _P, _P, _P, _P, _P,
                                          ctypes.c_int32, _P, ctypes.c_size_t, _P]),
}
for _name, (_res, _args) in _SIGS.items():
    _f = getattr(_lib, _name)
    _f.restype = _res
    _f.argtypes = _args

EXPORTED = tuple(_SIGS)


def lib() -> ctypes.CDLL:
    return _lib


def _ptr(t) -> Optional[int]:
    if t is None:
        return None
    if isinstance(t, int):
        return t
    return t.data_ptr()


def _stream(stream) -> Optional[int]:
    if stream is None:
        import torch
        return torch.cuda.current_stream().cuda_stream
    if isinstance(stream, int):
        return stream
    return stream.cuda_stream


def _check(rc: int, where: str) -> None:
    if rc != OK:
        if rc == ERR_CUDA:
            where = f"{where} [{_lib.moe_last_error_message().decode()}]"
        raise MoeError(rc, where)


def _sizes(desc) -> dict:
    """Bytes each buffer of the ABI needs for this descriptor."""
    T, d, Ks, N = desc.T, desc.d, desc.n_shared, desc.n_routed
    K, I = desc.top_k, desc.inter
    E, R = Ks + N, desc.T * desc.top_k
    a = 4 if desc.act_dtype == DT_F32 else 2
    w = {DT_F32: 4, DT_BF16: 2, DT_E4M3: 1}[desc.w_dtype]
    fp8 = desc.w_dtype == DT_E4M3
    xp_rows = R + (T if fp8 else 0)
    return {
        "x": T * d * a, "h": T * d * a, "x_residual": T * d * a, "w_router": N * d * a,
        "bias": N * 4, "topk_idx": R * 4, "topk_w": R * 4, "counts": N * 4,
        "offsets": (N + 1) * 4, "perm_src": R * 4, "slot_of": R * 4,
        "x_perm": xp_rows * d * (1 if fp8 else a),
        "x_perm_scale": xp_rows * (d // 128) * 4 if fp8 else 0,
        "w_gu": E * 2 * I * d * w, "w_down": E * d * I * w,
        "w_gu_scale": E * (2 * I // 128) * (d // 128) * 4 if fp8 else 0,
        "w_down_scale": E * (d // 128) * (I // 128) * 4 if fp8 else 0,
        "y_slots": T * (K + Ks) * d * a, "s_out": T * N * 4,
        "dh": T * d * a, "dx": T * d * a, "dw_router": N * d * 4, "dw_gu": E * 2 * I * d * 4,
        "dw_down": E * d * I * 4, "ab_saved": (R + Ks * T) * 2 * I * 2,
        "w_gu_t": E * d * 2 * I * w, "w_down_t": E * I * d * w,
        "w_gu_t_scale": E * (d // 128) * (2 * I // 128) * 4 if fp8 else 0,
        "w_down_t_scale": E * (I // 128) * (d // 128) * 4 if fp8 else 0,
    }


def _need(where: str, desc, **tensors) -> None:
    """Refuse a tensor argument that is strided or smaller than the descriptor needs."""
    sizes = _sizes(desc)
    for name, t in tensors.items():
        if t is None or isinstance(t, int) or not hasattr(t, "element_size"):
            continue
        if not t.is_contiguous():
            raise MoeError(ERR_INVALID_ARG, f"{where}: {name} is not contiguous")
        have = t.numel() * t.element_size()
        if have < sizes[name]:
            raise MoeError(ERR_INVALID_ARG,
                           f"{where}: {name} holds {have} bytes, the layer needs {sizes[name]}")


def moe_status_string(status: int) -> str:
    return _lib.moe_status_string(status).decode()


def make_desc(T: int, d: int, n_shared: int, n_routed: int, top_k: int, inter: int, gate: str,
              renorm: bool, route_scale: float, n_group: int = 1, topk_group: int = 1,
              dtype: str = "bf16") -> MoeLayerDesc:
    act, w = {"f32": (DT_F32, DT_F32), "bf16": (DT_BF16, DT_BF16),
              "e4m3": (DT_BF16, DT_E4M3)}[dtype]
    return MoeLayerDesc(T, d, n_shared, n_routed, top_k, inter,
                        {"softmax": GATE_SOFTMAX, "sigmoid": GATE_SIGMOID}[gate], int(renorm),
                        route_scale, n_group, topk_group, act, w)


def desc_from_config(cfg) -> MoeLayerDesc:
    """Descriptor of a synth.recipes.LayerConfig-like object."""
    return make_desc(cfg.T, cfg.d, cfg.n_shared, cfg.n_routed, cfg.top_k, cfg.inter, cfg.gate,
                     cfg.renorm, cfg.route_scale, cfg.n_group, cfg.topk_group, cfg.dtype)


def moe_workspace_size(desc: MoeLayerDesc) -> int:
    return int(_lib.moe_workspace_size(ctypes.byref(desc)))


def workspace(desc: MoeLayerDesc, device="cuda"):
    """A uint8 CUDA tensor of moe_workspace_size(desc) bytes."""
    import torch
    n = moe_workspace_size(desc)
    if n == 0:
        raise MoeError(ERR_INVALID_ARG, "moe_workspace_size")
    return torch.empty(n, dtype=torch.uint8, device=device)


def moe_route(desc, x, w_router, bias, topk_idx, topk_w, counts, ws, stream=None) -> None:
    _need("moe_route", desc, x=x, w_router=w_router, bias=bias, topk_idx=topk_idx,
          topk_w=topk_w, counts=counts)
    _check(_lib.moe_route(ctypes.byref(desc), _ptr(x), _ptr(w_router), _ptr(bias), _ptr(topk_idx),
                          _ptr(topk_w), _ptr(counts), _ptr(ws), ws.numel() if ws is not None
                          else 0, _stream(stream)), "moe_route")


def moe_permute(desc, x, topk_idx, counts, offsets, perm_src, slot_of, x_perm, x_perm_scale, ws,
                stream=None) -> None:
    _need("moe_permute", desc, x=x, topk_idx=topk_idx, counts=counts, offsets=offsets,
          perm_src=perm_src, slot_of=slot_of, x_perm=x_perm, x_perm_scale=x_perm_scale)
    _check(_lib.moe_permute(ctypes.byref(desc), _ptr(x), _ptr(topk_idx), _ptr(counts),
                            _ptr(offsets), _ptr(perm_src), _ptr(slot_of), _ptr(x_perm),
                            _ptr(x_perm_scale), _ptr(ws), ws.numel() if ws is not None else 0,
                            _stream(stream)), "moe_permute")


def moe_permute_noalloc(desc, x, topk_idx, counts, offsets, perm_src, slot_of, x_perm,
                        x_perm_scale, stream=None) -> None:
    """moe_permute without a workspace (fixed 1 MiB device scratch; see include/moe.h)."""
    _need("moe_permute_noalloc", desc, x=x, topk_idx=topk_idx, counts=counts,
          offsets=offsets, perm_src=perm_src, slot_of=slot_of, x_perm=x_perm,
          x_perm_scale=x_perm_scale)
    _check(_lib.moe_permute_noalloc(ctypes.byref(desc), _ptr(x), _ptr(topk_idx), _ptr(counts),
                                    _ptr(offsets), _ptr(perm_src), _ptr(slot_of), _ptr(x_perm),
                                    _ptr(x_perm_scale), _stream(stream)), "moe_permute_noalloc")


def moe_grouped_swiglu(desc, x, x_perm, x_perm_scale, offsets, perm_src, slot_of, topk_w, w_gu,
                       w_gu_scale, w_down, w_down_scale, y_slots, ws, stream=None) -> None:
    _need("moe_grouped_swiglu", desc, x=x, x_perm=x_perm, x_perm_scale=x_perm_scale,
          offsets=offsets, perm_src=perm_src, slot_of=slot_of, topk_w=topk_w, w_gu=w_gu,
          w_gu_scale=w_gu_scale, w_down=w_down, w_down_scale=w_down_scale, y_slots=y_slots)
    _check(_lib.moe_grouped_swiglu(ctypes.byref(desc), _ptr(x), _ptr(x_perm), _ptr(x_perm_scale),
                                   _ptr(offsets), _ptr(perm_src), _ptr(slot_of), _ptr(topk_w),
                                   _ptr(w_gu), _ptr(w_gu_scale), _ptr(w_down),
                                   _ptr(w_down_scale), _ptr(y_slots), _ptr(ws),
                                   ws.numel() if ws is not None else 0, _stream(stream)),
           "moe_grouped_swiglu")


def moe_combine(desc, x_residual, y_slots, h, stream=None) -> None:
    _need("moe_combine", desc, x_residual=x_residual, y_slots=y_slots, h=h)
    _check(_lib.moe_combine(ctypes.byref(desc), _ptr(x_residual), _ptr(y_slots), _ptr(h),
                            _stream(stream)), "moe_combine")


def moe_forward(desc, x, x_residual, w_router, bias, w_gu, w_gu_scale, w_down, w_down_scale, h,
                topk_idx, counts, ws, stream=None) -> None:
    _need("moe_forward", desc, x=x, x_residual=x_residual, w_router=w_router, bias=bias,
          w_gu=w_gu, w_gu_scale=w_gu_scale, w_down=w_down, w_down_scale=w_down_scale, h=h,
          topk_idx=topk_idx, counts=counts)
    _check(_lib.moe_forward(ctypes.byref(desc), _ptr(x), _ptr(x_residual), _ptr(w_router),
                            _ptr(bias), _ptr(w_gu), _ptr(w_gu_scale), _ptr(w_down),
                            _ptr(w_down_scale), _ptr(h), _ptr(topk_idx), _ptr(counts), _ptr(ws),
                            ws.numel() if ws is not None else 0, _stream(stream)), "moe_forward")


def moe_saved_ab_bytes(desc: MoeLayerDesc) -> int:
    return int(_lib.moe_saved_ab_bytes(ctypes.byref(desc)))


def moe_forward_save(desc, x, x_residual, w_router, bias, w_gu, w_down, h, topk_idx, counts,
                     ab_saved, ws, stream=None) -> None:
    """moe_forward that also writes the expert pre-activations a | b to ab_saved."""
    _need("moe_forward_save", desc, x=x, x_residual=x_residual, w_router=w_router, bias=bias,
          w_gu=w_gu, w_down=w_down, h=h, topk_idx=topk_idx, counts=counts, ab_saved=ab_saved)
    _check(_lib.moe_forward_save(ctypes.byref(desc), _ptr(x), _ptr(x_residual), _ptr(w_router),
                                 _ptr(bias), _ptr(w_gu), _ptr(w_down), _ptr(h), _ptr(topk_idx),
                                 _ptr(counts), _ptr(ab_saved), _ptr(ws),
                                 ws.numel() if ws is not None else 0, _stream(stream)),
           "moe_forward_save")


def moe_route_affinities(desc, x, w_router, s_out, ws, stream=None) -> None:
    _need("moe_route_affinities", desc, x=x, w_router=w_router, s_out=s_out)
    _check(_lib.moe_route_affinities(ctypes.byref(desc), _ptr(x), _ptr(w_router), _ptr(s_out),
                                     _ptr(ws), ws.numel() if ws is not None else 0,
                                     _stream(stream)), "moe_route_affinities")


def moe_balance_stats(desc, s, topk_idx, seq_len: int, f_out, p_out, stream=None) -> None:
    _check(_lib.moe_balance_stats(ctypes.byref(desc), _ptr(s), _ptr(topk_idx), seq_len,
                                  _ptr(f_out), _ptr(p_out), _stream(stream)), "moe_balance_stats")


def moe_bias_update(desc, counts, bias, gamma: float, stream=None) -> None:
    _check(_lib.moe_bias_update(ctypes.byref(desc), _ptr(counts), _ptr(bias), gamma,
                                _stream(stream)), "moe_bias_update")


def moe_quantize_fp8_blockwise(w_bf16, rows: int, cols: int, batch: int, w_e4m3, scale,
                               stream=None) -> None:
    _check(_lib.moe_quantize_fp8_blockwise(_ptr(w_bf16), rows, cols, batch, _ptr(w_e4m3),
                                           _ptr(scale), _stream(stream)),
           "moe_quantize_fp8_blockwise")


def moe_quantize_fp8_blockwise_t(w_bf16, rows: int, cols: int, batch: int, w_e4m3_t, scale_t,
                                 stream=None) -> None:
    _check(_lib.moe_quantize_fp8_blockwise_t(_ptr(w_bf16), rows, cols, batch, _ptr(w_e4m3_t),
                                             _ptr(scale_t), _stream(stream)),
           "moe_quantize_fp8_blockwise_t")


def fp8_backward_weights(w_gu, w_down, stream=None):
    """The E4M3 weights moe_backward_fp8 takes, from a layer's bf16 expert
    weights w_gu [E, 2I, d] and w_down [E, d, I], in its argument order:
    (w_gu, w_gu_scale, w_gu_t, w_gu_t_scale, w_down_t, w_down_t_scale)."""
    import torch
    E, two_i, d = w_gu.shape
    I = w_down.shape[2]
    out = []
    for quant, w, rows, cols in ((moe_quantize_fp8_blockwise, w_gu, two_i, d),
                                 (moe_quantize_fp8_blockwise_t, w_gu, two_i, d),
                                 (moe_quantize_fp8_blockwise_t, w_down, d, I)):
        r, c = (rows, cols) if quant is moe_quantize_fp8_blockwise else (cols, rows)
        q = torch.empty(E, r, c, dtype=torch.uint8, device=w.device)
        sc = torch.empty(E, r // 128, c // 128, dtype=torch.float32, device=w.device)
        quant(w, rows, cols, E, q, sc, stream)
        out += [q, sc]
    return tuple(out)


def moe_last_device_status(stream=None) -> int:
    return int(_lib.moe_last_device_status(_stream(stream)))


def moe_forward_launch_count(desc) -> int:
    return int(_lib.moe_forward_launch_count(ctypes.byref(desc)))


def moe_trace_events(events) -> None:
    """Record stage-boundary events (a list of 6 torch.cuda.Event, or None to stop)."""
    global _trace_keep
    if events is None:
        _trace_keep = None
        _check(_lib.moe_trace_events(None, 0), "moe_trace_events")
        return
    handles = [e.cuda_event for e in events]
    if not all(handles):
        raise ValueError("trace events must exist: record each torch.cuda.Event once first")
    arr = (ctypes.c_void_p * len(events))(*handles)
    _trace_keep = arr
    _check(_lib.moe_trace_events(arr, len(events)), "moe_trace_events")


_trace_keep = None


def moe_selftest_bounded_wait(limit_us: int, stream=None) -> None:
    _check(_lib.moe_selftest_bounded_wait(limit_us, _stream(stream)), "moe_selftest_bounded_wait")


def moe_backward_workspace_size(desc: MoeLayerDesc) -> int:
    return int(_lib.moe_backward_workspace_size(ctypes.byref(desc)))


def backward_workspace(desc: MoeLayerDesc, device="cuda"):
    """A uint8 CUDA tensor of moe_backward_workspace_size(desc) bytes."""
    import torch
    n = moe_backward_workspace_size(desc)
    if n == 0:
        raise MoeError(ERR_UNSUPPORTED, "moe_backward_workspace_size")
    return torch.empty(n, dtype=torch.uint8, device=device)


def moe_backward(desc, x, w_router, bias, w_gu, w_down, dh, dx, dw_router, dw_gu, dw_down, ws,
                 stream=None) -> None:
    _need("moe_backward", desc, x=x, w_router=w_router, bias=bias, w_gu=w_gu, w_down=w_down,
          dh=dh, dx=dx, dw_router=dw_router, dw_gu=dw_gu, dw_down=dw_down)
    _check(_lib.moe_backward(ctypes.byref(desc), _ptr(x), _ptr(w_router), _ptr(bias), _ptr(w_gu),
                             _ptr(w_down), _ptr(dh), _ptr(dx), _ptr(dw_router), _ptr(dw_gu),
                             _ptr(dw_down), _ptr(ws), ws.numel() if ws is not None else 0,
                             _stream(stream)), "moe_backward")


def moe_backward_bf16_grads(desc, x, w_router, bias, w_gu, w_down, dh, dx, dw_router, dw_gu,
                            dw_down, ws, stream=None) -> None:
    """moe_backward with the weight gradients written as bf16 tensors."""
    _need("moe_backward_bf16_grads", desc, x=x, w_router=w_router, bias=bias, w_gu=w_gu,
          w_down=w_down, dh=dh, dx=dx)
    sz = _sizes(desc)
    for name, t in (("dw_router", dw_router), ("dw_gu", dw_gu), ("dw_down", dw_down)):
        if not t.is_contiguous() or t.element_size() != 2 or 2 * t.numel() * 2 < sz[name]:
            raise MoeError(ERR_INVALID_ARG, f"moe_backward_bf16_grads: {name} must be a "
                           "contiguous bf16 tensor of the gradient's shape")
    _check(_lib.moe_backward_bf16_grads(ctypes.byref(desc), _ptr(x), _ptr(w_router), _ptr(bias),
                                        _ptr(w_gu), _ptr(w_down), _ptr(dh), _ptr(dx),
                                        _ptr(dw_router), _ptr(dw_gu), _ptr(dw_down), _ptr(ws),
                                        ws.numel() if ws is not None else 0, _stream(stream)),
           "moe_backward_bf16_grads")


def moe_backward_saved(desc, x, w_router, bias, w_gu, w_down, dh, ab_saved, dx, dw_router,
                       dw_gu, dw_down, ws, bf16_grads: bool = False, stream=None) -> None:
    """The backward from the pre-activations moe_forward_save kept."""
    _need("moe_backward_saved", desc, x=x, w_router=w_router, bias=bias, w_gu=w_gu,
          w_down=w_down, dh=dh, dx=dx, ab_saved=ab_saved)
    sz = _sizes(desc)
    esz = 2 if bf16_grads else 4
    for name, t in (("dw_router", dw_router), ("dw_gu", dw_gu), ("dw_down", dw_down)):
        if t is None:
            continue
        if not t.is_contiguous() or t.element_size() != esz or t.numel() * 4 < sz[name]:
            raise MoeError(ERR_INVALID_ARG, f"moe_backward_saved: {name} must be a contiguous "
                           f"{'bf16' if bf16_grads else 'fp32'} tensor of the gradient's shape")
    _check(_lib.moe_backward_saved(ctypes.byref(desc), _ptr(x), _ptr(w_router), _ptr(bias),
                                   _ptr(w_gu), _ptr(w_down), _ptr(dh), _ptr(ab_saved), _ptr(dx),
                                   _ptr(dw_router), _ptr(dw_gu), _ptr(dw_down),
                                   1 if bf16_grads else 0, _ptr(ws),
                                   ws.numel() if ws is not None else 0, _stream(stream)),
           "moe_backward_saved")


def moe_backward_fp8_workspace_size(desc: MoeLayerDesc) -> int:
    return int(_lib.moe_backward_fp8_workspace_size(ctypes.byref(desc)))


def backward_fp8_workspace(desc: MoeLayerDesc, device="cuda"):
    """A uint8 CUDA tensor of moe_backward_fp8_workspace_size(desc) bytes."""
    import torch
    n = moe_backward_fp8_workspace_size(desc)
    if n == 0:
        raise MoeError(ERR_UNSUPPORTED, "moe_backward_fp8_workspace_size")
    return torch.empty(n, dtype=torch.uint8, device=device)


def moe_backward_fp8(desc, x, w_router, bias, w_gu, w_gu_scale, w_gu_t, w_gu_t_scale, w_down_t,
                     w_down_t_scale, dh, dx, dw_router, dw_gu, dw_down, ws, stream=None) -> None:
    """The backward of an E4M3 layer with FP8 GEMMs; bf16 weight gradients."""
    _need("moe_backward_fp8", desc, x=x, w_router=w_router, bias=bias, w_gu=w_gu,
          w_gu_scale=w_gu_scale, w_gu_t=w_gu_t, w_gu_t_scale=w_gu_t_scale, w_down_t=w_down_t,
          w_down_t_scale=w_down_t_scale, dh=dh, dx=dx)
    sz = _sizes(desc)
    for name, t in (("dw_router", dw_router), ("dw_gu", dw_gu), ("dw_down", dw_down)):
        if t is None:
            continue
        if not t.is_contiguous() or t.element_size() != 2 or t.numel() * 4 < sz[name]:
            raise MoeError(ERR_INVALID_ARG, f"moe_backward_fp8: {name} must be a contiguous "
                           "bf16 tensor of the gradient's shape")
    _check(_lib.moe_backward_fp8(ctypes.byref(desc), _ptr(x), _ptr(w_router), _ptr(bias),
                                 _ptr(w_gu), _ptr(w_gu_scale), _ptr(w_gu_t), _ptr(w_gu_t_scale),
                                 _ptr(w_down_t), _ptr(w_down_t_scale), _ptr(dh), _ptr(dx),
                                 _ptr(dw_router),
                                 _ptr(dw_gu), _ptr(dw_down), _ptr(ws),
                                 ws.numel() if ws is not None else 0, _stream(stream)),
           "moe_backward_fp8")


def moe_backward_fp8_launch_count(desc) -> int:
    return int(_lib.moe_backward_fp8_launch_count(ctypes.byref(desc)))


def moe_backward_launch_count(desc) -> int:
    return int(_lib.moe_backward_launch_count(ctypes.byref(desc)))


def moe_expert_ffn_workspace_size(desc: MoeLayerDesc, n_groups: int, n_rows_out: int) -> int:
    return int(_lib.moe_expert_ffn_workspace_size(ctypes.byref(desc), n_groups, n_rows_out))


def moe_expert_ffn(desc, n_experts: int, groups, x_rows, row_w, w_gu, w_down, y_rows, ws,
                   stream=None) -> None:
    """y_rows[out0 + r] = row_w[out0 + r] * FFN_expert(x_rows[row0 + r]) for each group
    (row0, rows, expert, out0) of the int32 [n_groups, 4] device tensor `groups`."""
    for name, t, rows_needed in (("x_rows", x_rows, x_rows.shape[0]),
                                 ("y_rows", y_rows, y_rows.shape[0])):
        if not t.is_contiguous() or t.shape[-1] != desc.d:
            raise MoeError(ERR_INVALID_ARG, f"moe_expert_ffn: {name} must be contiguous [rows, d]")
    if not groups.is_contiguous() or groups.dtype.itemsize != 4 or groups.shape[-1] != 4:
        raise MoeError(ERR_INVALID_ARG, "moe_expert_ffn: groups must be contiguous int32 [n, 4]")
    if row_w is not None and row_w.numel() < y_rows.shape[0]:
        raise MoeError(ERR_INVALID_ARG, "moe_expert_ffn: row_w shorter than y_rows")
    w = {DT_F32: 4, DT_BF16: 2, DT_E4M3: 1}[desc.w_dtype]
    if w_gu.numel() * w_gu.element_size() < n_experts * 2 * desc.inter * desc.d * w or \
            w_down.numel() * w_down.element_size() < n_experts * desc.d * desc.inter * w:
        raise MoeError(ERR_INVALID_ARG, "moe_expert_ffn: expert weights shorter than n_experts")
    _check(_lib.moe_expert_ffn(ctypes.byref(desc), n_experts, groups.shape[0], _ptr(groups),
                               x_rows.shape[0], y_rows.shape[0], _ptr(x_rows), _ptr(row_w),
                               _ptr(w_gu), _ptr(w_down), _ptr(y_rows), _ptr(ws),
                               ws.numel() if ws is not None else 0, _stream(stream)),
           "moe_expert_ffn")


def moe_combine_rows(desc, x_residual, y_shared, y_rows, row_of, h, stream=None) -> None:
    """h[t] = x_res[t] + sum_s y_shared[s*T + t] + sum_k y_rows[row_of[t*K + k]]."""
    _need("moe_combine_rows", desc, x_residual=x_residual, h=h)
    if row_of.numel() < desc.T * desc.top_k or not row_of.is_contiguous():
        raise MoeError(ERR_INVALID_ARG, "moe_combine_rows: row_of must hold T*K int32")
    if y_shared is not None and y_shared.numel() < desc.n_shared * desc.T * desc.d:
        raise MoeError(ERR_INVALID_ARG, "moe_combine_rows: y_shared shorter than Ks*T rows")
    _check(_lib.moe_combine_rows(ctypes.byref(desc), _ptr(x_residual), _ptr(y_shared),
                                 _ptr(y_rows), _ptr(row_of),
                                 y_rows.shape[0] if y_rows is not None else 0, _ptr(h),
                                 _stream(stream)), "moe_combine_rows")


def moe_dispatch_rows(desc, x, topk_w, row_of, x_rows, w_rows, stream=None) -> None:
    """x_rows[row_of[t*K + k]] = x[t], w_rows[row_of[t*K + k]] = topk_w[t, k]."""
    _need("moe_dispatch_rows", desc, x=x, topk_w=topk_w)
    if row_of.numel() < desc.T * desc.top_k or not row_of.is_contiguous():
        raise MoeError(ERR_INVALID_ARG, "moe_dispatch_rows: row_of must hold T*K int32")
    if not x_rows.is_contiguous() or x_rows.shape[-1] != desc.d:
        raise MoeError(ERR_INVALID_ARG, "moe_dispatch_rows: x_rows must be contiguous [rows, d]")
    if w_rows is not None and w_rows.numel() < x_rows.shape[0]:
        raise MoeError(ERR_INVALID_ARG, "moe_dispatch_rows: w_rows shorter than x_rows")
    _check(_lib.moe_dispatch_rows(ctypes.byref(desc), _ptr(x), _ptr(topk_w), _ptr(row_of),
                                  x_rows.shape[0], _ptr(x_rows), _ptr(w_rows), _stream(stream)),
           "moe_dispatch_rows")


def moe_dispatch_rows_to(desc, x, topk_w, row_of, n_rows: int, x_addr, w_addr, start, base,
                         stream=None, s_addr=None) -> None:
    """Peer dispatch: send-order row r (start[q] <= r < start[q+1]) lands at row
    base[q] + r - start[q] of the buffers at device addresses x_addr[q] (rows)
    and w_addr[q] (gate weights, or 0); for an E4M3 layer the rows are the
    quantised codes and s_addr[q] receives their 1x128 scales."""
    _need("moe_dispatch_rows_to", desc, x=x, topk_w=topk_w)
    if row_of.numel() < desc.T * desc.top_k or not row_of.is_contiguous():
        raise MoeError(ERR_INVALID_ARG, "moe_dispatch_rows_to: row_of must hold T*K int32")
    n = len(x_addr)
    if not 1 <= n <= MAX_PEERS or len(w_addr) != n or len(start) != n + 1 or len(base) != n:
        raise MoeError(ERR_INVALID_ARG, "moe_dispatch_rows_to: one address, start and base a rank")
    P = MoePeerRows()
    P.n_ranks = n
    for q in range(n):
        P.x[q] = int(x_addr[q]) or None
        P.w[q] = int(w_addr[q]) or None
        P.scale[q] = (int(s_addr[q]) or None) if s_addr is not None else None
        P.start[q] = int(start[q])
        P.base[q] = int(base[q])
    P.start[n] = int(start[n])
    _check(_lib.moe_dispatch_rows_to(ctypes.byref(desc), _ptr(x), _ptr(topk_w), _ptr(row_of),
                                     int(n_rows), ctypes.byref(P), _stream(stream)),
           "moe_dispatch_rows_to")


def moe_expert_ffn_to(desc, n_experts: int, groups, n_rows_in: int, n_rows_out: int, x_rows,
                      row_w, w_gu, w_down, group_out, ws, stream=None) -> None:
    """As moe_expert_ffn, with group i's output rows stored at the device byte
    address group_out[i] (a uint64/int64 device tensor [n_groups])."""
    if not groups.is_contiguous() or groups.dtype.itemsize != 4 or groups.shape[-1] != 4:
        raise MoeError(ERR_INVALID_ARG, "moe_expert_ffn_to: groups must be contiguous int32 [n, 4]")
    if group_out.numel() < groups.shape[0] or group_out.dtype.itemsize != 8 or \
            not group_out.is_contiguous():
        raise MoeError(ERR_INVALID_ARG, "moe_expert_ffn_to: group_out must hold one uint64 a group")
    if not x_rows.is_contiguous() or x_rows.shape[-1] != desc.d:
        raise MoeError(ERR_INVALID_ARG, "moe_expert_ffn_to: x_rows must be contiguous [rows, d]")
    _check(_lib.moe_expert_ffn_to(ctypes.byref(desc), int(n_experts), groups.shape[0],
                                  _ptr(groups), int(n_rows_in), int(n_rows_out), _ptr(x_rows),
                                  _ptr(row_w), _ptr(w_gu), _ptr(w_down), _ptr(group_out),
                                  _ptr(ws), ws.numel() if ws is not None else 0,
                                  _stream(stream)),
           "moe_expert_ffn_to")


def moe_ipc_get_handle(t):
    """(handle, offset): the CUDA IPC handle of the allocation holding tensor
    t's data and the data's byte offset in it."""
    buf = ctypes.create_string_buffer(IPC_HANDLE_BYTES)
    off = ctypes.c_uint64()
    _check(_lib.moe_ipc_get_handle(_ptr(t), buf, ctypes.byref(off)), "moe_ipc_get_handle")
    return buf.raw, int(off.value)


def moe_ipc_open(handle: bytes) -> int:
    """Device address, in this process, of another process's allocation (its
    base: add the offset moe_ipc_get_handle returned with the handle)."""
    if len(handle) != IPC_HANDLE_BYTES:
        raise MoeError(ERR_INVALID_ARG, "moe_ipc_open: handle must be 64 bytes")
    out = ctypes.c_void_p()
    _check(_lib.moe_ipc_open(ctypes.create_string_buffer(handle, IPC_HANDLE_BYTES),
                             ctypes.byref(out)), "moe_ipc_open")
    return int(out.value)


def moe_ipc_close(addr: int) -> None:
    _check(_lib.moe_ipc_close(ctypes.c_void_p(addr)), "moe_ipc_close")


def moe_dispatch_rows_fp8(desc, x, topk_w, row_of, x_rows, x_rows_scale, w_rows,
                          stream=None) -> None:
    """E4M3 dispatch: each token's row quantised per 1x128 tile once, codes to
    x_rows[row_of[t*K + k]], scales to x_rows_scale, gate weights to w_rows."""
    _need("moe_dispatch_rows_fp8", desc, x=x, topk_w=topk_w)
    if row_of.numel() < desc.T * desc.top_k or not row_of.is_contiguous():
        raise MoeError(ERR_INVALID_ARG, "moe_dispatch_rows_fp8: row_of must hold T*K int32")
    n = x_rows.shape[0]
    if not x_rows.is_contiguous() or x_rows.shape[-1] != desc.d or x_rows.element_size() != 1:
        raise MoeError(ERR_INVALID_ARG, "moe_dispatch_rows_fp8: x_rows must be uint8 [rows, d]")
    if x_rows_scale.numel() < n * (desc.d // 128) or (w_rows is not None and w_rows.numel() < n):
        raise MoeError(ERR_INVALID_ARG, "moe_dispatch_rows_fp8: scale / weight rows too short")
    _check(_lib.moe_dispatch_rows_fp8(ctypes.byref(desc), _ptr(x), _ptr(topk_w), _ptr(row_of), n,
                                      _ptr(x_rows), _ptr(x_rows_scale), _ptr(w_rows),
                                      _stream(stream)), "moe_dispatch_rows_fp8")


def moe_quantize_rows_fp8(desc, x, codes, scales, stream=None) -> None:
    """1x128 E4M3 quantisation of the bf16 rows of x [n, d]."""
    n = x.shape[0]
    if codes.numel() < n * desc.d or scales.numel() < n * (desc.d // 128):
        raise MoeError(ERR_INVALID_ARG, "moe_quantize_rows_fp8: outputs too short")
    _check(_lib.moe_quantize_rows_fp8(ctypes.byref(desc), _ptr(x), n, _ptr(codes), _ptr(scales),
                                      _stream(stream)), "moe_quantize_rows_fp8")


def moe_expert_ffn_fp8(desc, n_experts: int, groups, n_rows_in: int, n_rows_out: int, x_rows,
                       x_rows_scale, row_w, w_gu, w_gu_scale, w_down, w_down_scale, ws,
                       y_rows=None, group_out=None, stream=None) -> None:
    """The FP8 expert GEMMs over caller-given row groups; outputs to y_rows or
    to the per-group addresses of group_out."""
    if not groups.is_contiguous() or groups.dtype.itemsize != 4 or groups.shape[-1] != 4:
        raise MoeError(ERR_INVALID_ARG, "moe_expert_ffn_fp8: groups must be contiguous int32 [n, 4]")
    if (y_rows is None) == (group_out is None):
        raise MoeError(ERR_INVALID_ARG, "moe_expert_ffn_fp8: give y_rows or group_out")
    _check(_lib.moe_expert_ffn_fp8(ctypes.byref(desc), int(n_experts), groups.shape[0],
                                   _ptr(groups), int(n_rows_in), int(n_rows_out), _ptr(x_rows),
                                   _ptr(x_rows_scale), _ptr(row_w), _ptr(w_gu), _ptr(w_gu_scale),
                                   _ptr(w_down), _ptr(w_down_scale), _ptr(y_rows),
                                   _ptr(group_out), _ptr(ws),
                                   ws.numel() if ws is not None else 0, _stream(stream)),
           "moe_expert_ffn_fp8")
