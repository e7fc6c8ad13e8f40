"""fp64 CPU oracle of the DeepSeekMoE layer backward.

TEST INFRASTRUCTURE.  Only the tests may import or call this module; the
library's product path never does.  It shares no code with the CUDA path.

Given the upstream gradient dh = dL/dh of the forward

    h_t = x_res_t + sum_{i<Ks} FFN_i(u_t) + sum_k g_{t,k} FFN_{Ks+idx_{t,k}}(u_t),
    FFN(v) = W_down (SiLU(W_gate v) * (W_up v)),

(DeepSeek Technical Report: MoE Architecture, §1.1(2) equation / §5.3
equation [1]; SwiGLU experts as in DeepSeek-V3 아키텍처 둘러보기), it returns
the gradients of the layer's inputs and parameters.  The same report's §3.6
lists the backward GEMMs of a linear layer (activation backward and weight
backward) among the FP8 GEMMs and keeps the gating in BF16; this oracle is the
exact fp64 result those must approximate.

The selection (top-K, group limit) is piecewise constant in the inputs, so no
gradient flows through the chosen indices; the selection bias b enters only the
selection key and gets no gradient (the aux-loss-free rule updates it from the
expert counts instead, §3.3).  Gradients flow through the gate weights g into
the affinities s of the selected experts, then through softmax or sigmoid into
the router logits and W_r.

Per active (token t, expert e) pair with gate weight g (1 for shared experts):
    a = W_gate u,  b = W_up u,  z = SiLU(a) * b,  y = W_down z
    dy  = g dh_t                      dg = <dh_t, y>
    dW_down += dy z^T                 dz = W_down^T dy
    da = dz * b * SiLU'(a)            db = dz * SiLU(a)
    dW_gate += da u^T                 dW_up += db u^T
    du += W_gate^T da + W_up^T db
with SiLU'(a) = sigma(a) (1 + a (1 - sigma(a))).
Gate weights: g_k = c s_k / S (renorm, S = sum_k s_k) or c s_k:
    ds_j = c (dg_j - sum_k dg_k s_k / S) / S   or   ds_j = c dg_j.
Affinities: sigmoid ds -> dl = ds s (1 - s); softmax over the N routed experts
    dl = s * (ds - <ds, s>).
Router: dW_r += dl^T u, du += W_r^T dl.  The residual: dx_res = dh.
"""
from __future__ import annotations

from typing import Callable, Dict, Optional, Tuple

import numpy as np

from oracle import moe_oracle as mo

ExpertFn = Callable[[int], Tuple[np.ndarray, np.ndarray, np.ndarray]]


def silu_grad(a: np.ndarray) -> np.ndarray:
    """d/da [a sigma(a)] = sigma(a) (1 + a (1 - sigma(a)))."""
    sg = 1.0 / (1.0 + np.exp(-a))
    return sg * (1.0 + a * (1.0 - sg))


def expert_backward(u: np.ndarray, dy: np.ndarray, w_gate: np.ndarray, w_up: np.ndarray,
                    w_down: np.ndarray):
    """Backward of y = W_down (SiLU(W_gate u) * (W_up u)) for rows u [M, d],
    output gradients dy [M, d].  Returns (y, du, dW_gate, dW_up, dW_down)."""
    u = np.asarray(u, np.float64)
    dy = np.asarray(dy, np.float64)
    a = u @ w_gate.T
    b = u @ w_up.T
    z = mo.silu(a) * b
    y = z @ w_down.T
    dz = dy @ w_down
    da = dz * b * silu_grad(a)
    db = dz * mo.silu(a)
    return y, da @ w_gate + db @ w_up, da.T @ u, db.T @ u, dy.T @ z


def gate_weight_backward(s_sel: np.ndarray, dg: np.ndarray, renorm: bool,
                         route_scale: float) -> np.ndarray:
    """d L / d s_sel for g = c s_sel / sum(s_sel) (renorm) or g = c s_sel, rows = tokens."""
    if not renorm:
        return route_scale * dg
    S = s_sel.sum(axis=1, keepdims=True)
    return route_scale * (dg - (dg * s_sel).sum(axis=1, keepdims=True) / S) / S


def affinity_backward(s: np.ndarray, ds: np.ndarray, gate: str) -> np.ndarray:
    """d L / d logits from d L / d s (s over the N routed experts)."""
    if gate == "softmax":
        return s * (ds - (ds * s).sum(axis=1, keepdims=True))
    return ds * s * (1.0 - s)


def moe_backward(x, w_r, bias, expert: ExpertFn, dh, *, n_shared: int, gate: str, top_k: int,
                 n_group: int = 1, topk_group: int = 1, renorm: bool = False,
                 route_scale: float = 1.0, idx_override: Optional[np.ndarray] = None) -> Dict:
    """Gradients of the layer with u = x and a separate residual input.

    Returns dx (through the experts and the router), dx_res (= dh), dW_r
    [N, d], and per expert e < Ks + N the arrays dW_gate [I, d], dW_up [I, d],
    dW_down [d, I] (zeros for experts no token reaches), plus the routing used
    (idx, g).  idx_override replaces the selection (for near-tie tokens)."""
    x = np.asarray(x, np.float64)
    dh = np.asarray(dh, np.float64)
    T, d = x.shape
    w_r = np.asarray(w_r, np.float64)
    N = w_r.shape[0]
    logits = mo.router_logits(x, w_r)
    s = mo.affinity(logits, gate)
    if idx_override is None:
        idx, _, _ = mo.select_experts(s, bias, top_k, n_group, topk_group)
    else:
        idx = np.asarray(idx_override, np.int64)
    g = mo.gate_weights(s, idx, renorm, route_scale)

    dx = np.zeros_like(x)
    dg = np.zeros((T, top_k))
    grads = {}

    def accumulate(e, rows, dy):
        w_gate, w_up, w_down = (np.asarray(w, np.float64) for w in expert(e))
        y, du, dwg, dwu, dwd = expert_backward(x[rows], dy, w_gate, w_up, w_down)
        dx[rows] += du
        if e not in grads:
            grads[e] = [np.zeros_like(w_gate), np.zeros_like(w_up), np.zeros_like(w_down)]
        grads[e][0] += dwg
        grads[e][1] += dwu
        grads[e][2] += dwd
        return y

    all_rows = np.arange(T)
    for e in range(n_shared):
        accumulate(e, all_rows, dh)
    for j in range(N):
        t_sel, k_sel = np.nonzero(idx == j)
        if len(t_sel) == 0:
            continue
        y = accumulate(n_shared + j, t_sel, dh[t_sel] * g[t_sel, k_sel][:, None])
        dg[t_sel, k_sel] = np.sum(dh[t_sel] * y, axis=1)

    s_sel = np.take_along_axis(s, idx, axis=1)
    ds_sel = gate_weight_backward(s_sel, dg, renorm, route_scale)
    ds = np.zeros_like(s)
    np.put_along_axis(ds, idx, ds_sel, axis=1)
    dl = affinity_backward(s, ds, gate)
    dx += dl @ w_r
    dw_r = dl.T @ x
    return {"dx": dx, "dx_res": dh.copy(), "dw_r": dw_r, "experts": grads, "idx": idx, "g": g,
            "dl": dl}
