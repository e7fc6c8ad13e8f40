"""Pins of the fp64 backward oracle (oracle/moe_backward.py) against facts that
do not come from the oracle itself:

  * SiLU's derivative against central differences of SiLU and its closed
    values at 0 and in the tails;
  * every gradient of a tiny layer (inputs, router, each expert's three
    matrices) against central differences of the forward oracle for the loss
    L = <dh, h>, in softmax and sigmoid gating, with and without
    renormalisation, with a group limit and a selection bias; every token's
    selection margin is checked to exceed the perturbation, so the
    differences never cross a selection boundary;
  * the selection bias gets no gradient (it enters only the key), the
    residual's gradient is dh, softmax logit gradients sum to zero per token,
    and with renormalised top-1 gating the router gets no gradient at all.
"""
import numpy as np
import pytest

from oracle import moe_backward as mb
from oracle import moe_oracle as mo

EPS = 1e-6


def test_silu_grad_closed_forms():
    a = np.linspace(-12.0, 12.0, 97)
    fd = (mo.silu(a + EPS) - mo.silu(a - EPS)) / (2 * EPS)
    assert np.max(np.abs(mb.silu_grad(a) - fd)) < 1e-8
    assert mb.silu_grad(np.array([0.0]))[0] == 0.5
    assert abs(mb.silu_grad(np.array([40.0]))[0] - 1.0) < 1e-12
    assert abs(mb.silu_grad(np.array([-40.0]))[0]) < 1e-12


class Layer:
    def __init__(self, seed, T=5, d=6, Ks=1, N=8, K=3, I=4, gate="softmax", renorm=False,
                 scale=1.0, G=1, Gk=1, bias=False):
        rng = np.random.default_rng(seed)
        self.T, self.d, self.Ks, self.N, self.K, self.I = T, d, Ks, N, K, I
        self.gate, self.renorm, self.scale, self.G, self.Gk = gate, renorm, scale, G, Gk
        self.x = rng.normal(size=(T, d))
        self.x_res = rng.normal(size=(T, d))
        self.w_r = rng.normal(size=(N, d)) * 0.7
        self.bias = rng.uniform(-0.1, 0.1, size=N) if bias else None
        self.w = [[rng.normal(size=(I, d)) * 0.5, rng.normal(size=(I, d)) * 0.5,
                   rng.normal(size=(d, I)) * 0.5] for _ in range(Ks + N)]
        self.dh = rng.normal(size=(T, d))

    def expert(self, e):
        return tuple(self.w[e])

    def kw(self):
        return dict(n_shared=self.Ks, gate=self.gate, top_k=self.K, n_group=self.G,
                    topk_group=self.Gk, renorm=self.renorm, route_scale=self.scale)

    def loss(self):
        r = mo.moe_forward(self.x, self.w_r, self.bias, self.expert, x_res=self.x_res,
                           **self.kw())
        return float(np.sum(self.dh * r["h"])), r

    def margins(self):
        r = mo.route(self.x, self.w_r, self.bias, gate=self.gate, top_k=self.K,
                     n_group=self.G, topk_group=self.Gk)
        return min(r["kgap"].min(), r["ggap"].min())


def fd_grad(layer, arr):
    """Central differences of L = <dh, h> with respect to every element of arr
    (modified in place and restored), checking the selection stays put."""
    base_idx = layer.loss()[1]["idx"]
    out = np.zeros_like(arr)
    it = np.nditer(arr, flags=["multi_index"])
    for _ in it:
        i = it.multi_index
        v = arr[i]
        arr[i] = v + EPS
        lp, rp = layer.loss()
        arr[i] = v - EPS
        lm, rm = layer.loss()
        arr[i] = v
        assert np.array_equal(rp["idx"], base_idx) and np.array_equal(rm["idx"], base_idx)
        out[i] = (lp - lm) / (2 * EPS)
    return out


CASES = {
    "softmax": dict(seed=1, gate="softmax"),
    "softmax_renorm": dict(seed=2, gate="softmax", renorm=True),
    "sigmoid_groups_bias": dict(seed=3, gate="sigmoid", renorm=True, scale=2.5, G=4, Gk=2,
                                bias=True),
    "sigmoid_two_shared": dict(seed=4, gate="sigmoid", Ks=2, K=2, bias=True),
}


def close(a, b, tol=2e-7):
    return np.max(np.abs(a - b)) <= tol * max(1.0, np.max(np.abs(b)))


@pytest.mark.parametrize("name", list(CASES))
def test_gradients_match_central_differences(name):
    L = Layer(**CASES[name])
    assert L.margins() > 1e-3, "pick a seed whose selection has margins"
    g = mb.moe_backward(L.x, L.w_r, L.bias, L.expert, L.dh, **L.kw())
    assert np.array_equal(g["dx_res"], L.dh)
    assert close(g["dx"], fd_grad(L, L.x))
    assert close(g["dw_r"], fd_grad(L, L.w_r))
    for e in range(L.Ks + L.N):
        want = [fd_grad(L, L.w[e][m]) for m in range(3)]
        got = g["experts"].get(e, [np.zeros_like(w) for w in L.w[e]])
        for m in range(3):
            assert close(got[m], want[m]), (name, e, m)
    if L.bias is not None:
        assert np.max(np.abs(fd_grad(L, L.bias))) < 1e-8   # the bias enters only the key
    if L.gate == "softmax":
        assert np.max(np.abs(g["dl"].sum(axis=1))) < 1e-12


def test_renormalised_top1_gives_the_router_no_gradient():
    # g = c s / s = c: the gate weight does not depend on the logits
    L = Layer(seed=5, gate="sigmoid", renorm=True, scale=2.5, K=1, bias=True)
    g = mb.moe_backward(L.x, L.w_r, L.bias, L.expert, L.dh, **L.kw())
    assert np.max(np.abs(g["dw_r"])) < 1e-12
    assert np.max(np.abs(g["dl"])) < 1e-12
