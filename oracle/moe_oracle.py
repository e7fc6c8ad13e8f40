"""fp64 CPU oracle of the DeepSeekMoE layer forward.

TEST INFRASTRUCTURE.  Only the tests, the smoke check and the bench's CPU
baseline leg may import or call this module; the library's product path never
does.  It shares no code with the CUDA path.

What it computes, step by step, with the passage each step follows:

  * router logits   l[t,i] = u_t . e_i
        DeepSeek Technical Report: MoE Architecture, §2.3 (gate
        g = Softmax_i(u_t^T e_i)) and §3.3 (affinity s = Sigmoid(u_t^T e_i)).
  * affinity        softmax over the N routed experts (DeepSeekMoE / V2 gate,
        same report §2.3 and the table of §5.1), or the element-wise sigmoid
        (V3, §3.3 and equation [3] of §5.3).
  * selection       TopK over the keys s_i + b_i, where the bias b only enters
        the key (same report §3.3, equation [4]; DeepSeek-V3 Technical Report
        논문 정리, auxiliary-loss-free balancing).  Optional group limit: the
        N experts form n_group contiguous groups; a group's score is the sum of
        its two largest keys; only the topk_group best groups stay eligible.
        Ties in either ranking go to the lower index.
  * gate weights    g = s of the selected experts (no renorm), or s / sum(s)
        over the selected experts; both times route_scale (1.0, or 2.5 for the
        V3 layer).  The bias never enters g.
  * permutation     counts, exclusive-scan offsets, and for each (t, k) the
        slot offsets[e] + #{t' < t : e in idx[t']}; stable by token.
  * experts         FFN(v) = W_down (SiLU(W_gate v) * (W_up v)),
        SiLU(z) = z / (1 + e^-z) (DeepSeek-V3 아키텍처 둘러보기: the MLP is
        SwiGLU).
  * output          h_t = x_res_t + sum_{i<Ks} FFN_i(u_t) + sum_k g_k FFN_{Ks+idx_k}(u_t)
        (DeepSeek Technical Report: MoE Architecture, §1.1(2) DeepSeekMoE
        equation, = equation [1] of §5.3).

All arithmetic is float64 on the exact stored input values; no intermediate is
rounded.  Readings taken where the pages are silent are listed in the repo's
design notes (group score = top-2 sum, normalise-then-scale, softmax over
routed experts only, ties to lower index).
"""
from __future__ import annotations

from typing import Callable, Dict, Optional, Sequence, Tuple

import numpy as np

NEAR_TIE = 1e-5


def router_logits(x: np.ndarray, w_r: np.ndarray) -> np.ndarray:
    """l[t, i] = <u_t, e_i> for every token t and routed expert i."""
    return np.asarray(x, np.float64) @ np.asarray(w_r, np.float64).T


def affinity(logits: np.ndarray, gate: str) -> np.ndarray:
    """Token-to-expert affinity s[t, i].

    softmax: s_i = exp(l_i - max_j l_j) / sum_j exp(l_j - max_j l_j) over the
    routed experts; sigmoid: s_i = 1 / (1 + exp(-l_i))."""
    l = np.asarray(logits, np.float64)
    if gate == "softmax":
        m = l.max(axis=1, keepdims=True)
        e = np.exp(l - m)
        return e / e.sum(axis=1, keepdims=True)
    if gate == "sigmoid":
        with np.errstate(over="ignore"):
            return 1.0 / (1.0 + np.exp(-l))
    raise ValueError(f"unknown gate {gate!r}")


def group_scores(key: np.ndarray, n_group: int) -> np.ndarray:
    """Score of each contiguous expert group: the sum of its two largest keys."""
    T, N = key.shape
    kg = np.sort(key.reshape(T, n_group, N // n_group), axis=2)
    return kg[:, :, -1] + kg[:, :, -2]


def select_experts(s: np.ndarray, bias: Optional[np.ndarray], top_k: int, n_group: int = 1,
                   topk_group: int = 1) -> Tuple[np.ndarray, np.ndarray, np.ndarray]:
    """Top-K expert indices per token, ordered by (key desc, index asc).

    Returns (idx [T,K] int64, kgap [T], ggap [T]) where kgap is the key gap
    between the K-th and (K+1)-th eligible expert and ggap the score gap
    between the topk_group-th and next group (inf when there is no next one).
    """
    s = np.asarray(s, np.float64)
    T, N = s.shape
    if n_group > 1 and (N % n_group or topk_group * (N // n_group) < top_k):
        raise ValueError("group limit leaves fewer than top_k eligible experts")
    if top_k > N:
        raise ValueError("top_k exceeds the number of routed experts")
    key = s if bias is None else s + np.asarray(bias, np.float64)[None, :]
    ggap = np.full(T, np.inf)
    eligible = np.ones((T, N), dtype=bool)
    if n_group > 1:
        gs = group_scores(key, n_group)
        gorder = np.argsort(-gs, axis=1, kind="stable")
        keep = np.zeros((T, n_group), dtype=bool)
        np.put_along_axis(keep, gorder[:, :topk_group], True, axis=1)
        eligible = np.repeat(keep, N // n_group, axis=1)
        if topk_group < n_group:
            gsorted = np.take_along_axis(gs, gorder, axis=1)
            ggap = gsorted[:, topk_group - 1] - gsorted[:, topk_group]
    masked = np.where(eligible, key, -np.inf)
    order = np.argsort(-masked, axis=1, kind="stable")
    idx = order[:, :top_k]
    ksorted = np.take_along_axis(masked, order, axis=1)
    if top_k < N:
        kgap = ksorted[:, top_k - 1] - ksorted[:, top_k]
        kgap = np.where(np.isneginf(ksorted[:, top_k]), np.inf, kgap)
    else:
        kgap = np.full(T, np.inf)
    return idx.astype(np.int64), kgap, ggap


def gate_weights(s: np.ndarray, idx: np.ndarray, renorm: bool, route_scale: float) -> np.ndarray:
    """g[t,k] = route_scale * s[t, idx[t,k]] (/ sum_k s[t, idx[t,k]] when renorm)."""
    g = np.take_along_axis(np.asarray(s, np.float64), idx, axis=1)
    if renorm:
        g = g / g.sum(axis=1, keepdims=True)
    return g * route_scale


def route(x, w_r, bias, *, gate: str, top_k: int, n_group: int = 1, topk_group: int = 1,
          renorm: bool = False, route_scale: float = 1.0) -> Dict[str, np.ndarray]:
    """Gating for every token: logits, affinities, selection, weights, tie gaps."""
    logits = router_logits(x, w_r)
    s = affinity(logits, gate)
    idx, kgap, ggap = select_experts(s, bias, top_k, n_group, topk_group)
    g = gate_weights(s, idx, renorm, route_scale)
    key = s + np.asarray(bias, np.float64)[None, :] if bias is not None else s
    return {"logits": logits, "s": s, "key": key, "idx": idx, "w": g, "kgap": kgap,
            "ggap": ggap}


def near_tie_tokens(kgap: np.ndarray, ggap: np.ndarray, thr: float = NEAR_TIE) -> np.ndarray:
    """Tokens whose selection is decided by a gap below thr (expert or group ranking)."""
    return np.nonzero((kgap < thr) | (ggap < thr))[0]


def permutation(idx: np.ndarray, n_routed: int):
    """Expert-contiguous order of the T*K (token, slot) pairs, stable by token.

    Returns counts [N], offsets [N+1] (exclusive scan), perm_src [T*K] (token of
    each permuted row) and slot_of [T*K] (permuted row of pair t*K+k)."""
    idx = np.asarray(idx, np.int64)
    T, K = idx.shape
    flat = idx.reshape(-1)
    counts = np.bincount(flat, minlength=n_routed).astype(np.int64)
    offsets = np.zeros(n_routed + 1, np.int64)
    offsets[1:] = np.cumsum(counts)
    order = np.argsort(flat, kind="stable")
    perm_src = order // K
    slot_of = np.empty(T * K, np.int64)
    slot_of[order] = np.arange(T * K)
    return counts, offsets, perm_src, slot_of


def silu(z: np.ndarray) -> np.ndarray:
    with np.errstate(over="ignore"):
        return z / (1.0 + np.exp(-z))


def swiglu_ffn(v: np.ndarray, w_gate: np.ndarray, w_up: np.ndarray,
               w_down: np.ndarray) -> np.ndarray:
    """FFN(v) = W_down (SiLU(W_gate v) * (W_up v)) for each row v of `v`.

    v [n, d]; w_gate, w_up [I, d]; w_down [d, I]."""
    return (silu(v @ w_gate.T) * (v @ w_up.T)) @ w_down.T


ExpertFn = Callable[[int], Tuple[np.ndarray, np.ndarray, np.ndarray]]


def layer_output(x_rows: np.ndarray, x_res_rows: np.ndarray, idx_rows: np.ndarray,
                 g_rows: np.ndarray, n_shared: int, expert: ExpertFn,
                 ffn: Callable = swiglu_ffn) -> Tuple[np.ndarray, np.ndarray]:
    """h = x_res + sum_shared FFN_i(u) + sum_k g_k FFN_{Ks+idx_k}(u) for the given rows.

    expert(e) returns (w_gate, w_up, w_down) of expert e (shared experts are
    0..Ks-1, routed expert j is Ks+j).  Returns (h, delta = h - x_res)."""
    x_rows = np.asarray(x_rows, np.float64)
    delta = np.zeros_like(x_rows)
    for e in range(n_shared):
        wg, wu, wd = expert(e)
        delta += ffn(x_rows, wg, wu, wd)
    for j in np.unique(idx_rows):
        rows, ks = np.nonzero(idx_rows == j)
        wg, wu, wd = expert(n_shared + int(j))
        delta[rows] += g_rows[rows, ks][:, None] * ffn(x_rows[rows], wg, wu, wd)
    return np.asarray(x_res_rows, np.float64) + delta, delta


def moe_forward(x, w_r, bias, expert: ExpertFn, *, n_shared: int, gate: str, top_k: int,
                n_group: int = 1, topk_group: int = 1, renorm: bool = False,
                route_scale: float = 1.0, x_res=None,
                tokens: Optional[Sequence[int]] = None,
                idx_override: Optional[Dict[int, Sequence[int]]] = None) -> Dict[str, np.ndarray]:
    """The whole layer: routing on all tokens, outputs on `tokens` (all by default).

    idx_override maps a token to the expert list to use downstream instead of
    the oracle's own selection (used for near-tie tokens, whose selection is
    not unique to within rounding); its gate weights are still computed here
    from the oracle's affinities."""
    x = np.asarray(x, np.float64)
    r = route(x, w_r, bias, gate=gate, top_k=top_k, n_group=n_group, topk_group=topk_group,
              renorm=renorm, route_scale=route_scale)
    idx = r["idx"].copy()
    if idx_override:
        for t, ex in idx_override.items():
            idx[t] = np.asarray(ex, np.int64)
        r["w"] = gate_weights(r["s"], idx, renorm, route_scale)
    r["idx_used"] = idx
    T = x.shape[0]
    rows = np.arange(T) if tokens is None else np.asarray(tokens, np.int64)
    xr = x if x_res is None else np.asarray(x_res, np.float64)
    h, delta = layer_output(x[rows], xr[rows], idx[rows], r["w"][rows], n_shared, expert)
    r.update({"tokens": rows, "h": h, "delta": delta})
    return r


def max_abs_rel(got: np.ndarray, ref: np.ndarray) -> float:
    """max |got - ref| / max |ref| over all elements."""
    ref = np.asarray(ref, np.float64)
    den = float(np.max(np.abs(ref))) if ref.size else 0.0
    if den == 0.0:
        return float(np.max(np.abs(np.asarray(got, np.float64)))) if ref.size else 0.0
    return float(np.max(np.abs(np.asarray(got, np.float64) - ref)) / den)


# ----------------------------------------------------------------------------- load balance
def bias_update(bias: np.ndarray, counts: np.ndarray, gamma: float) -> np.ndarray:
    """One step of the auxiliary-loss-free balancing rule.

    b_i <- b_i - gamma when expert i is overloaded (its load above the mean
    load T*K/N), b_i + gamma when underloaded (below it), unchanged at the mean
    (DeepSeek Technical Report: MoE Architecture, §3.3 bias update rule,
    gamma = 0.001).  The bias is stored in fp32, so the step is one fp32
    subtraction or addition."""
    b = np.asarray(bias, np.float32)
    c = np.asarray(counts, np.int64)
    total, n = int(c.sum()), len(c)
    over = c * n > total            # load above the mean, compared exactly in integers
    under = c * n < total
    g = np.float32(gamma)
    out = b.copy()
    out[over] = (b[over] - g).astype(np.float32)
    out[under] = (b[under] + g).astype(np.float32)
    return out


def balance_stats(s: np.ndarray, idx: np.ndarray, seq_len: int):
    """Routing statistics per sequence of seq_len consecutive tokens.

    f[q, i] = fraction of the sequence's tokens that selected expert i and
    P[q, i] = mean affinity s_i over the sequence's tokens (DeepSeek Technical
    Report: MoE Architecture, §1.2: f_i, P_i of L_ExpBal = alpha_1 sum_i f_i P_i;
    with seq_len = T they are the batch-level statistics, with a shorter
    seq_len the per-sequence ones of the sequence-wise balance loss of §3.3)."""
    s = np.asarray(s, np.float64)
    idx = np.asarray(idx, np.int64)
    T, N = s.shape
    if seq_len <= 0 or T % seq_len:
        raise ValueError("seq_len must divide T")
    S = T // seq_len
    f = np.zeros((S, N))
    P = np.zeros((S, N))
    for q in range(S):
        rows = slice(q * seq_len, (q + 1) * seq_len)
        f[q] = np.bincount(idx[rows].reshape(-1), minlength=N) / seq_len
        P[q] = s[rows].mean(axis=0)
    return f, P
