"""Pins of the fp64 oracle against things other than itself.

Each test checks the oracle against a closed form, a brute-force enumeration,
or a value the pages print, chosen so that a plausible mistake (a dropped
term, a swapped operand, a wrong tie rule, a bias leaking into the weights)
fails at least one of them.
"""
import dataclasses
import itertools
import math
import os

import numpy as np
import pytest

from oracle import moe_oracle as mo

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")


# ----------------------------------------------------------------------------- combinatorics
def n_choose_k_pascal(n, k):
    """Binomial coefficient by Pascal's rule (dynamic programming, no factorials)."""
    row = [1] + [0] * k
    for _ in range(n):
        for j in range(k, 0, -1):
            row[j] += row[j - 1]
    return row[k]


def read_golden_counts():
    out = []
    with open(os.path.join(GOLDEN, "combinatorics.txt")) as f:
        for line in f:
            if line.strip() and not line.startswith("#"):
                n, k, c = map(int, line.split())
                out.append((n, k, c))
    return out


def test_printed_combination_counts():
    rows = read_golden_counts()
    assert rows, "fixture empty"
    for n, k, c in rows:
        assert n_choose_k_pascal(n, k) == c


@pytest.mark.parametrize("N,K", [(5, 2), (6, 3), (8, 2), (7, 4)])
def test_every_k_subset_is_reachable(N, K):
    # Equal affinities and a bias of 1 on the members of S make S the unique
    # top-K, so the selection can reach every K-subset: C(N, K) distinct sets.
    T = 1
    seen = set()
    for S in itertools.combinations(range(N), K):
        s = np.full((T, N), 0.25)
        b = np.zeros(N)
        b[list(S)] = 1.0
        idx, _, _ = mo.select_experts(s, b, K)
        seen.add(tuple(sorted(idx[0].tolist())))
        assert tuple(sorted(idx[0].tolist())) == S
    assert len(seen) == n_choose_k_pascal(N, K)


def reachable_closed_form(G, n, K, Gk):
    """Number of K-subsets of G groups of n experts that use at most Gk groups
    (inclusion-exclusion over the groups actually used)."""
    total = 0
    for j in range(1, Gk + 1):
        exact_j = sum((-1) ** i * math.comb(j, i) * math.comb((j - i) * n, K) for i in range(j + 1))
        total += math.comb(G, j) * exact_j
    return total


@pytest.mark.parametrize("G,N,K,Gk", [(4, 8, 2, 1), (4, 8, 2, 2), (4, 8, 3, 2), (2, 8, 2, 1)])
def test_group_limited_reachable_sets(G, N, K, Gk):
    n = N // G
    reach = 0
    for S in itertools.combinations(range(N), K):
        s = np.full((1, N), 0.25)
        b = np.zeros(N)
        b[list(S)] = 1.0
        idx, _, _ = mo.select_experts(s, b, K, n_group=G, topk_group=Gk)
        groups = {e // n for e in S}
        got = tuple(sorted(idx[0].tolist()))
        if len(groups) <= Gk:
            assert got == S
            reach += 1
        else:
            assert got != S
            assert len({e // n for e in got}) <= Gk
    assert reach == reachable_closed_form(G, n, K, Gk)


# ----------------------------------------------------------------------------- selection
def brute_topk(key, K, eligible=None):
    """K-subset with the largest key sum; among equal sums the lexicographically
    lowest sorted index tuple; returned in (key desc, index asc) order."""
    N = len(key)
    cand = [i for i in range(N) if eligible is None or eligible[i]]
    best, best_sum = None, -math.inf
    for S in itertools.combinations(cand, K):
        tot = math.fsum(key[i] for i in S)
        if tot > best_sum:
            best, best_sum = S, tot
    return sorted(best, key=lambda i: (-key[i], i))


@pytest.mark.parametrize("seed", range(6))
def test_topk_matches_brute_force(seed):
    rng = np.random.default_rng(seed)
    for N, K in [(6, 2), (8, 3), (10, 4), (9, 1)]:
        T = 40
        # keys on a coarse grid so that ties occur often
        s = rng.integers(0, 6, size=(T, N)) / 8.0
        idx, kgap, _ = mo.select_experts(s, None, K)
        for t in range(T):
            assert idx[t].tolist() == brute_topk(s[t].tolist(), K)
            srt = sorted(s[t].tolist(), reverse=True)
            assert kgap[t] == pytest.approx(srt[K - 1] - srt[K])


def brute_group_select(key, K, G, Gk):
    N = len(key)
    n = N // G
    gscore = []
    for g in range(G):
        members = range(g * n, (g + 1) * n)
        gscore.append(max(key[a] + key[b] for a, b in itertools.combinations(members, 2)))
    best, best_sum = None, -math.inf
    for S in itertools.combinations(range(G), Gk):
        tot = math.fsum(gscore[g] for g in S)
        if tot > best_sum:
            best, best_sum = S, tot
    eligible = [(i // n) in best for i in range(N)]
    return brute_topk(key, K, eligible), sorted(gscore, reverse=True)


@pytest.mark.parametrize("seed", range(4))
def test_group_limited_selection_matches_brute_force(seed):
    rng = np.random.default_rng(100 + seed)
    for G, N, K, Gk in [(4, 8, 2, 2), (4, 8, 3, 2), (4, 16, 4, 2), (2, 8, 2, 1)]:
        T = 30
        s = rng.integers(0, 5, size=(T, N)) / 8.0
        b = rng.integers(-2, 3, size=N) / 16.0
        idx, _, ggap = mo.select_experts(s, b, K, n_group=G, topk_group=Gk)
        key = s + b[None, :]
        for t in range(T):
            want, gs = brute_group_select(key[t].tolist(), K, G, Gk)
            assert idx[t].tolist() == want
            if Gk < G:
                assert ggap[t] == pytest.approx(gs[Gk - 1] - gs[Gk])


def test_group_score_is_top2_sum_not_max():
    # group 0 has the single largest key, group 1 the larger top-2 sum.
    key = np.array([[0.9, 0.0, 0.6, 0.6]])
    gs = mo.group_scores(key, 2)
    assert gs.tolist() == [[0.9, 1.2]]
    idx, _, _ = mo.select_experts(key, None, 2, n_group=2, topk_group=1)
    assert idx[0].tolist() == [2, 3]


# ----------------------------------------------------------------------------- weights / bias
@pytest.mark.parametrize("gate,renorm,scale", [("softmax", True, 1.0), ("sigmoid", True, 2.5),
                                               ("softmax", False, 1.0)])
def test_gate_weight_sums(gate, renorm, scale):
    rng = np.random.default_rng(7)
    T, N, K = 50, 16, 4
    logits = rng.normal(size=(T, N))
    s = mo.affinity(logits, gate)
    idx, _, _ = mo.select_experts(s, None, K)
    g = mo.gate_weights(s, idx, renorm, scale)
    if renorm:
        np.testing.assert_allclose(g.sum(1), scale, rtol=0, atol=1e-12)
    else:
        topmass = np.sort(s, axis=1)[:, -K:].sum(1)
        np.testing.assert_allclose(g.sum(1), topmass, rtol=0, atol=1e-15)
        assert np.all(g.sum(1) <= 1.0 + 1e-15)
    if gate == "softmax":
        np.testing.assert_allclose(s.sum(1), 1.0, atol=1e-12)
        # closed form of one softmax entry
        t = 3
        ex = [math.exp(v) for v in logits[t]]
        assert s[t, 5] == pytest.approx(ex[5] / math.fsum(ex), rel=1e-13)
    else:
        assert s[0, 0] == pytest.approx(1 / (1 + math.exp(-logits[0, 0])), rel=1e-14)


def test_bias_only_changes_selection_not_weights():
    rng = np.random.default_rng(11)
    T, N, K = 200, 32, 4
    logits = rng.normal(size=(T, N))
    b = rng.uniform(-0.1, 0.1, size=N)
    s = mo.affinity(logits, "sigmoid")
    idx0, _, _ = mo.select_experts(s, None, K, n_group=4, topk_group=2)
    idx1, _, _ = mo.select_experts(s, b, K, n_group=4, topk_group=2)
    assert np.any(np.sort(idx0, 1) != np.sort(idx1, 1)), "bias should change some selections"
    g1 = mo.gate_weights(s, idx1, True, 2.5)
    for t in range(T):
        sel = idx1[t]
        # weights are the unbiased affinities of the selected set, renormalised
        want = 2.5 * s[t, sel] / s[t, sel].sum()
        np.testing.assert_allclose(g1[t], want, rtol=0, atol=1e-15)
        common = set(idx0[t].tolist()) & set(sel.tolist())
        if set(idx0[t].tolist()) == set(sel.tolist()):
            g0 = mo.gate_weights(s[t:t + 1], idx0[t:t + 1], True, 2.5)[0]
            assert sorted(g0.tolist()) == pytest.approx(sorted(g1[t].tolist()), abs=1e-15)
        assert common is not None
    # a constant bias shifts every key equally: same selection, same weights
    idx2, _, _ = mo.select_experts(s, np.full(N, 0.05), K, n_group=4, topk_group=2)
    assert np.array_equal(idx0, idx2)


# ----------------------------------------------------------------------------- experts
def test_silu_closed_forms():
    z = np.array([0.0, 1.0, -1.0, 40.0, -40.0])
    got = mo.silu(z)
    assert got[0] == 0.0
    assert got[1] == pytest.approx(1.0 / (1.0 + math.exp(-1.0)), rel=1e-15)
    assert got[2] == pytest.approx(-1.0 / (1.0 + math.e), rel=1e-15)
    assert got[3] == pytest.approx(40.0, rel=1e-15)
    assert abs(got[4]) < 1e-15


def test_swiglu_hand_worked_example():
    # d=2, I=1: v=(1,2), gate row (1,-1) -> z=-1, up row (2,1) -> 4,
    # H = SiLU(-1)*4 = -4/(1+e), out = W_down H with W_down = [[1],[3]].
    v = np.array([[1.0, 2.0]])
    wg, wu, wd = np.array([[1.0, -1.0]]), np.array([[2.0, 1.0]]), np.array([[1.0], [3.0]])
    H = -4.0 / (1.0 + math.e)
    out = mo.swiglu_ffn(v, wg, wu, wd)
    assert out[0].tolist() == pytest.approx([H, 3 * H], rel=1e-15)


def test_swiglu_operand_roles():
    # Gate = a*Identity, up = Identity, down = a non-symmetric permutation P:
    # FFN(v) = P (SiLU(a v) * v).  Swapping gate/up gives P(SiLU(v) * a v);
    # a transposed W_down gives P^T(...): both differ for a != 1.
    d, a = 5, 3.0
    rng = np.random.default_rng(3)
    v = rng.normal(size=(4, d))
    P = np.eye(d)[[1, 2, 3, 4, 0]]
    out = mo.swiglu_ffn(v, a * np.eye(d), np.eye(d), P)
    inner = np.array([[(a * x) / (1 + math.exp(-a * x)) * x for x in row] for row in v])
    want = inner @ P.T
    np.testing.assert_allclose(out, want, rtol=1e-13, atol=1e-15)
    assert not np.allclose(out, inner @ P, atol=1e-6)


def _random_layer(rng, T, d, Ks, N, I, scale=0.3):
    experts = [(rng.normal(size=(I, d)) * scale, rng.normal(size=(I, d)) * scale,
                rng.normal(size=(d, I)) * scale) for _ in range(Ks + N)]
    x = rng.normal(size=(T, d))
    w_r = rng.normal(size=(N, d)) * scale
    return x, w_r, experts


def test_shared_experts_always_active_and_routed_zero():
    rng = np.random.default_rng(5)
    T, d, Ks, N, K, I = 12, 6, 2, 8, 3, 4
    x, w_r, experts = _random_layer(rng, T, d, Ks, N, I)
    zero_routed = [e if i < Ks else (np.zeros_like(e[0]), np.zeros_like(e[1]), np.zeros_like(e[2]))
                   for i, e in enumerate(experts)]
    r = mo.moe_forward(x, w_r, None, lambda e: zero_routed[e], n_shared=Ks, gate="softmax",
                       top_k=K)
    shared = sum(mo.swiglu_ffn(x, *experts[i]) for i in range(Ks))
    np.testing.assert_allclose(r["h"], x + shared, rtol=1e-13, atol=1e-13)
    # Zero shared experts: routed-only output.
    zero_shared = [e if i >= Ks else (np.zeros_like(e[0]), np.zeros_like(e[1]), np.zeros_like(e[2]))
                   for i, e in enumerate(experts)]
    r2 = mo.moe_forward(x, w_r, None, lambda e: zero_shared[e], n_shared=Ks, gate="softmax",
                        top_k=K)
    r3 = mo.moe_forward(x, w_r, None, lambda e: experts[e], n_shared=Ks, gate="softmax", top_k=K)
    np.testing.assert_allclose(r3["h"] - r2["h"], shared, rtol=1e-12, atol=1e-12)


def test_expert_relabelling_invariance():
    # Permuting the routed experts together with their router rows changes nothing.
    rng = np.random.default_rng(9)
    T, d, Ks, N, K, I = 10, 6, 1, 8, 2, 4
    x, w_r, experts = _random_layer(rng, T, d, Ks, N, I)
    perm = rng.permutation(N)
    experts_p = experts[:Ks] + [experts[Ks + j] for j in perm]
    r = mo.moe_forward(x, w_r, None, lambda e: experts[e], n_shared=Ks, gate="sigmoid", top_k=K,
                       renorm=True, route_scale=2.5)
    rp = mo.moe_forward(x, w_r[perm], None, lambda e: experts_p[e], n_shared=Ks, gate="sigmoid",
                        top_k=K, renorm=True, route_scale=2.5)
    np.testing.assert_allclose(r["h"], rp["h"], rtol=1e-12, atol=1e-12)


def test_dense_softmax_mixture_when_all_experts_selected():
    # N = K with softmax and renorm: every routed expert is active with weight softmax_i.
    rng = np.random.default_rng(13)
    T, d, Ks, N, I = 7, 5, 1, 4, 3
    x, w_r, experts = _random_layer(rng, T, d, Ks, N, I)
    r = mo.moe_forward(x, w_r, None, lambda e: experts[e], n_shared=Ks, gate="softmax", top_k=N,
                       renorm=True)
    l = x @ w_r.T
    p = np.exp(l) / np.exp(l).sum(1, keepdims=True)
    want = x + mo.swiglu_ffn(x, *experts[0])
    for i in range(N):
        want += p[:, i:i + 1] * mo.swiglu_ffn(x, *experts[Ks + i])
    np.testing.assert_allclose(r["h"], want, rtol=1e-12, atol=1e-12)


def test_plain_swiglu_mlp_when_no_routed_experts():
    # Ks = 1, N = 0: the layer is x + one SwiGLU MLP, written as a textbook chain.
    rng = np.random.default_rng(17)
    T, d, I = 6, 8, 5
    x = rng.normal(size=(T, d))
    Wg, Wu, Wd = rng.normal(size=(I, d)), rng.normal(size=(I, d)), rng.normal(size=(d, I))
    h, delta = mo.layer_output(x, x, np.zeros((T, 0), np.int64), np.zeros((T, 0)), 1,
                               lambda e: (Wg, Wu, Wd))
    a = np.einsum("td,id->ti", x, Wg)
    want = x + np.einsum("ti,di->td", a * (1 / (1 + np.exp(-a))) * np.einsum("td,id->ti", x, Wu),
                         Wd)
    np.testing.assert_allclose(h, want, rtol=1e-12, atol=1e-12)


# ----------------------------------------------------------------------------- permutation
def permutation_by_definition(idx, N):
    T, K = len(idx), len(idx[0])
    counts = [0] * N
    for t in range(T):
        for k in range(K):
            counts[idx[t][k]] += 1
    offsets = [0]
    for c in counts:
        offsets.append(offsets[-1] + c)
    slot_of = [0] * (T * K)
    perm_src = [0] * (T * K)
    for t in range(T):
        for k in range(K):
            e = idx[t][k]
            earlier = sum(1 for tp in range(t) if e in idx[tp])
            slot = offsets[e] + earlier
            slot_of[t * K + k] = slot
            perm_src[slot] = t
    return counts, offsets, perm_src, slot_of


@pytest.mark.parametrize("seed", range(3))
def test_permutation_matches_definition(seed):
    rng = np.random.default_rng(seed)
    T, N, K = 37, 9, 3
    idx = np.stack([rng.choice(N, K, replace=False) for _ in range(T)])
    counts, offsets, perm_src, slot_of = mo.permutation(idx, N)
    c2, o2, p2, s2 = permutation_by_definition(idx.tolist(), N)
    assert counts.tolist() == c2 and offsets.tolist() == o2
    assert perm_src.tolist() == p2 and slot_of.tolist() == s2
    assert offsets[-1] == T * K
    for e in range(N):
        seg = perm_src[offsets[e]:offsets[e + 1]]
        assert np.all(np.diff(seg) > 0)
    for t in range(T):
        for k in range(K):
            assert perm_src[slot_of[t * K + k]] == t


# ----------------------------------------------------------------------------- end to end
def literal_layer(x, x_res, w_r, bias, experts, Ks, K, gate, G, Gk, renorm, scale):
    """The layer by literal evaluation: loops, math.exp, and enumeration for selection."""
    T, d = len(x), len(x[0])
    N = len(w_r)
    out = []
    for t in range(T):
        l = [math.fsum(x[t][j] * w_r[i][j] for j in range(d)) for i in range(N)]
        if gate == "softmax":
            m = max(l)
            ex = [math.exp(v - m) for v in l]
            z = math.fsum(ex)
            s = [v / z for v in ex]
        else:
            s = [1.0 / (1.0 + math.exp(-v)) for v in l]
        key = [s[i] + (bias[i] if bias is not None else 0.0) for i in range(N)]
        if G > 1:
            sel, _ = brute_group_select(key, K, G, Gk)
        else:
            sel = brute_topk(key, K)
        g = [s[i] for i in sel]
        if renorm:
            tot = math.fsum(g)
            g = [v / tot for v in g]
        g = [v * scale for v in g]

        def ffn(e):
            wg, wu, wd = experts[e]
            I = len(wg)
            hmid = []
            for r in range(I):
                a = math.fsum(wg[r][j] * x[t][j] for j in range(d))
                b = math.fsum(wu[r][j] * x[t][j] for j in range(d))
                hmid.append(a / (1.0 + math.exp(-a)) * b)
            return [math.fsum(wd[c][r] * hmid[r] for r in range(I)) for c in range(d)]

        h = list(x_res[t])
        for e in range(Ks):
            f = ffn(e)
            h = [h[c] + f[c] for c in range(d)]
        for k, i in enumerate(sel):
            f = ffn(Ks + i)
            h = [h[c] + g[k] * f[c] for c in range(d)]
        out.append((sel, g, h))
    return out


@pytest.mark.parametrize("gate,G,Gk,renorm,scale,use_bias", [
    ("softmax", 1, 1, True, 1.0, False),
    ("softmax", 1, 1, False, 1.0, False),
    ("sigmoid", 2, 1, True, 2.5, True),
    ("sigmoid", 1, 1, True, 2.5, True),
])
def test_four_token_eight_expert_layer_by_enumeration(gate, G, Gk, renorm, scale, use_bias):
    rng = np.random.default_rng(21)
    T, d, Ks, N, K, I = 4, 6, 1, 8, 2, 3
    x, w_r, experts = _random_layer(rng, T, d, Ks, N, I, scale=0.5)
    x_res = x + rng.normal(size=x.shape)
    bias = rng.uniform(-0.1, 0.1, size=N) if use_bias else None
    r = mo.moe_forward(x, w_r, bias, lambda e: experts[e], n_shared=Ks, gate=gate, top_k=K,
                       n_group=G, topk_group=Gk, renorm=renorm, route_scale=scale, x_res=x_res)
    lit = literal_layer(x.tolist(), x_res.tolist(), w_r.tolist(),
                        None if bias is None else bias.tolist(),
                        [(a.tolist(), b.tolist(), c.tolist()) for a, b, c in experts],
                        Ks, K, gate, G, Gk, renorm, scale)
    for t in range(T):
        sel, g, h = lit[t]
        assert r["idx"][t].tolist() == sel
        np.testing.assert_allclose(r["w"][t], g, rtol=1e-13, atol=1e-15)
        np.testing.assert_allclose(r["h"][t], h, rtol=1e-12, atol=1e-12)
        np.testing.assert_allclose(r["delta"][t], np.array(h) - x_res[t], rtol=1e-11, atol=1e-12)


def test_near_tie_detection():
    kgap = np.array([1.0, 5e-6, 1.0, 2e-5])
    ggap = np.array([np.inf, np.inf, 1e-6, np.inf])
    assert mo.near_tie_tokens(kgap, ggap).tolist() == [1, 2]


def test_max_abs_rel():
    ref = np.array([[1.0, -4.0], [2.0, 0.5]])
    got = ref + np.array([[0.0, 0.1], [-0.2, 0.0]])
    assert mo.max_abs_rel(got, ref) == pytest.approx(0.05)


def test_three_matrix_experts_reproduce_the_v2_parameter_total():
    # Reading C-9, pinned to printed totals: the oracle's SwiGLU expert holds
    # W_gate, W_up [I, d] and W_down [d, I].  DeepSeek-V2 ("DeepSeek Technical
    # Report: MoE Architecture", §2.1 and §2.3): 60 layers, hidden 5,120, MoE in
    # every layer but the first, 2 shared + 160 routed experts of width 1,536,
    # 236B parameters in all.  Three matrices put 95.5 % of the total in the
    # experts (attention and embeddings take the rest); two would leave 36 %.
    from synth import recipes

    small = dataclasses.replace(recipes.CONFIGS["tiny_f32"], d=96, inter=32)
    per_expert = sum(w.size for w in recipes.host_expert(small, 0))
    assert per_expert == 3 * small.d * small.inter
    d, I, layers, experts = 5120, 1536, 60 - 1, 2 + 160
    total = 236e9
    moe3 = layers * experts * (per_expert // (small.d * small.inter)) * d * I
    moe2 = layers * experts * 2 * d * I
    assert 0.9 * total <= moe3 <= total
    assert moe2 < 0.7 * total
