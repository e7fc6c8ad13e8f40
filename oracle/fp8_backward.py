"""The DeepSeekMoE layer backward with FP8 GEMMs, emulated in float64 (oracle side).

TEST INFRASTRUCTURE: used only by the tests.  Shares no code with the CUDA
path.

DeepSeek Technical Report: MoE Architecture, §3.6 (FP8 mixed precision) puts
the activation-backward and the weight-backward GEMMs of every linear layer in
FP8 E4M3, next to the forward GEMMs; activations are grouped in 1x128 tiles
and weights in 128x128 blocks, with fp32 accumulation promoted every 128
elements; the MoE gating stays in BF16 and weight gradients are kept in BF16.
The gradients themselves follow oracle/moe_backward.py (the chain rule of the
layer's output equation, §1.1(2) / equation [1] of §5.3).

Readings taken where the pages are silent:
  * A scale is only usable per 128-element block of the contraction, so an
    activation's 1x128 tile runs along the dimension the GEMM contracts over:
    along the features for the activation-backward GEMMs (dh rows over d, the
    [da | db] rows over 2I, x rows over d for the recomputed pre-activations),
    and along the rows (tokens) for the weight-backward GEMMs, which contract
    over an expert's rows: there a tile is 128 rows of one column.
  * An expert's rows, for those 128-row tiles, are its tokens in increasing
    token order (the permutation's order), padded with zero rows to a multiple
    of 128; a shared expert's rows are all T tokens.
  * Which tensors are quantised: the inputs x and dh, and the intermediates
    [da | db] and g z.  The pre-activations a, b and the product dz' = dh W_down
    come out of FP8 GEMMs with fp32 accumulation and are not requantised.
  * dg (the gradient of a gate weight) is <dz', z> with dz' from that FP8
    GEMM, as the unquantised layer's <dh, W_down z> = <W_down^T dh, z>.
  * Intermediates: by default a, b, g z and [da | db] are held in fp32 before
    they are used or quantised.  With intermediates="bf16" they are rounded
    to bfloat16 (nearest even, from fp32) first, as a GPU that stores them in
    bf16 does; that form isolates the GEMMs' own error from this storage
    choice.
  * The gating backward (gate weights, affinities, the router GEMMs) is exact
    here; on the GPU it runs in BF16 / fp32 as the forward's gating does.

Every GEMM below multiplies dequantised operands in float64: each 128-element
block of a dot product is then exact and scaled by its two fp32 scales, which
is what promotion per 128 elements computes up to fp32 rounding.
"""
from __future__ import annotations

from typing import Callable, Dict, Optional, Tuple

import numpy as np

from oracle import fp8 as of8
from oracle import moe_backward as mb
from oracle import moe_oracle as mo

F32 = np.float32
ExpertFn = Callable[[int], Tuple[np.ndarray, np.ndarray, np.ndarray]]


def pad128(n: int) -> int:
    return (n + 127) // 128 * 128


def quantize_rows_along_tokens(rows: np.ndarray):
    """Rows [M, C] of an operand whose GEMM contracts over the rows.

    The rows are padded with zeros to a multiple of 128 and quantised in tiles
    of 128 rows x 1 column.  Returns the transposed codes as values
    q [C, Mp] and the tile scales s [C, Mp / 128], i.e. the 1x128 tiles of the
    transposed matrix."""
    rows = np.asarray(rows, np.float64)
    M, C = rows.shape
    t = np.zeros((C, pad128(max(M, 1))), np.float64)
    t[:, :M] = rows.T
    return of8.quantize_act_1x128(t.astype(F32))


def fp8_weight_grad(a_rows: np.ndarray, b_rows: np.ndarray) -> np.ndarray:
    """sum_r a_rows[r]^T b_rows[r] -> [Ca, Cb] as an FP8 weight-backward GEMM:
    both operands quantised per 128-row x 1-column tile, exact block products."""
    qa, sa = quantize_rows_along_tokens(a_rows)
    qb, sb = quantize_rows_along_tokens(b_rows)
    return of8.dequant_act(qa, sa) @ of8.dequant_act(qb, sb).T


def round_bf16(v: np.ndarray) -> np.ndarray:
    """Nearest bfloat16 values (ties to even) of v rounded to fp32 first, as float64."""
    f = np.ascontiguousarray(np.asarray(v, np.float64).astype(np.float32))
    u = f.view(np.uint32).astype(np.uint64)
    u = ((u + 0x7FFF + ((u >> 16) & 1)) >> 16) << 16
    return u.astype(np.uint32).view(np.float32).astype(np.float64)


def fp8_act(rows: np.ndarray) -> np.ndarray:
    """Rows quantised per 1x128 tile along their columns, dequantised."""
    q, s = of8.quantize_act_1x128(np.asarray(rows, np.float64).astype(F32))
    return of8.dequant_act(q, s)


def expert_backward_fp8(u: np.ndarray, dh: np.ndarray, g: np.ndarray, w_gate: np.ndarray,
                        w_up: np.ndarray, w_down: np.ndarray, intermediates: str = "fp32"):
    """One expert's backward with FP8 GEMMs.

    u [M, d] and dh [M, d] are the expert's input rows and the upstream
    gradient rows (token order), g [M] the gate weights (1 for a shared
    expert), the weights dequantised E4M3.  Returns
    (du [M, d], dg [M], dW_gate [I, d], dW_up [I, d], dW_down [d, I])."""
    u = np.asarray(u, np.float64)
    dh = np.asarray(dh, np.float64)
    g = np.asarray(g, np.float64)
    I = w_gate.shape[0]
    keep = round_bf16 if intermediates == "bf16" else (lambda v: v)
    # the pre-activations, recomputed by the FP8 forward GEMM
    uh = fp8_act(u)
    a = keep(uh @ w_gate.T)
    b = keep(uh @ w_up.T)
    # activation backward through W_down: dz' = dh W_down, dh rows in FP8
    dzp = fp8_act(dh) @ w_down
    z = mo.silu(a) * b
    dg = np.sum(dzp * z, axis=1)
    dz = g[:, None] * dzp
    da = keep(dz * b * mb.silu_grad(a))
    db = keep(dz * mo.silu(a))
    dab = np.concatenate([da, db], axis=1)
    # activation backward through W_gate, W_up: [da | db] rows in FP8
    du = fp8_act(dab) @ np.concatenate([w_gate, w_up], axis=0)
    # weight backward: contract over the expert's rows, 128-row tiles
    dw_down = fp8_weight_grad(dh, keep(g[:, None] * z))
    dw_gu = fp8_weight_grad(dab, u)
    return du, dg, dw_gu[:I], dw_gu[I:], dw_down


def moe_backward_fp8(x, w_r, bias, expert: ExpertFn, dh, *, n_shared: int, gate: str,
                     top_k: int, n_group: int = 1, topk_group: int = 1, renorm: bool = False,
                     route_scale: float = 1.0, idx_override: Optional[np.ndarray] = None,
                     intermediates: str = "fp32") -> Dict:
    """Gradients of the FP8 layer (u = x, separate residual), in the format of
    oracle.moe_backward.moe_backward: dx, dx_res, dw_r, experts {e: [dW_gate,
    dW_up, dW_down]} (experts no token reaches are absent), idx, g, dl.
    expert(e) returns the dequantised E4M3 weights (w_gate, w_up, w_down);
    intermediates "fp32" or "bf16" (see the module docstring)."""
    x = np.asarray(x, np.float64)
    dh = np.asarray(dh, np.float64)
    T, d = x.shape
    w_r = np.asarray(w_r, np.float64)
    N = w_r.shape[0]
    s = mo.affinity(mo.router_logits(x, w_r), gate)
    if idx_override is None:
        idx, _, _ = mo.select_experts(s, bias, top_k, n_group, topk_group)
    else:
        idx = np.asarray(idx_override, np.int64)
    g = mo.gate_weights(s, idx, renorm, route_scale)

    dx = np.zeros_like(x)
    dg = np.zeros((T, top_k))
    grads = {}

    def run(e, rows, g_rows):
        w_gate, w_up, w_down = (np.asarray(w, np.float64) for w in expert(e))
        du, dg_rows, dwg, dwu, dwd = expert_backward_fp8(x[rows], dh[rows], g_rows, w_gate,
                                                         w_up, w_down, intermediates)
        dx[rows] += du
        grads[e] = [dwg, dwu, dwd]
        return dg_rows

    for e in range(n_shared):
        run(e, np.arange(T), np.ones(T))
    for j in range(N):
        t_sel, k_sel = np.nonzero(idx == j)        # tokens in increasing order
        if len(t_sel) == 0:
            continue
        dg[t_sel, k_sel] = run(n_shared + j, t_sel, g[t_sel, k_sel])

    s_sel = np.take_along_axis(s, idx, axis=1)
    ds_sel = mb.gate_weight_backward(s_sel, dg, renorm, route_scale)
    ds = np.zeros_like(s)
    np.put_along_axis(ds, idx, ds_sel, axis=1)
    dl = mb.affinity_backward(s, ds, gate)
    dx += dl @ w_r
    return {"dx": dx, "dx_res": dh.copy(), "dw_r": dl.T @ x, "experts": grads, "idx": idx,
            "g": g, "dl": dl}
