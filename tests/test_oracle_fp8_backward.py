"""Pins of the FP8 backward oracle (oracle/fp8_backward.py).

- The weight-backward quantisation (128 rows x 1 column tiles along the rows
  the GEMM contracts over) against values written out from the E4M3 format
  and the scale rule, on a matrix built so that the other plausible tilings
  (1x128 along the columns, 64-row tiles, 128x128 blocks) give other values.
- Exact power-of-two scaling laws that hold only for the right tile axes:
  scaling one token's upstream gradient by 4 scales that token's dx by exactly
  4 and leaves every other token's dx unchanged (the activation-backward
  tiles run along the features); scaling one feature column of dh by 4 scales
  that row of every dW_down by exactly 4 and leaves the other rows unchanged
  (the weight-backward tiles run along the tokens).
- Distance to the exact fp64 backward (oracle/moe_backward.py, itself pinned to
  central differences of the forward) within 2^-3, twice E4M3's relative step,
  on every gradient: catches a dropped term, a wrong sign or operand.
"""
import numpy as np
import pytest

from oracle import fp8 as of8
from oracle import fp8_backward as fb
from oracle import moe_backward as mb
from oracle import moe_oracle as mo

F32 = np.float32


def scale_only(v):
    """The dequantised value of v alone in its tile: code 448 (v * 448/|v| in
    fp32 rounds to 448) times the fp32 scale |v|/448."""
    amax = F32(abs(v))
    s = F32(amax / F32(448.0))
    code = of8.e4m3_round(np.float64(F32(F32(v) * F32(F32(448.0) / amax))))
    return float(code) * float(s)


def test_weight_grad_tiles_closed_form():
    # a: 256 token rows, 2 feature columns; b: every entry 448 (scale 1, code 448)
    a = np.zeros((256, 2))
    a[100, 0] = 448.0          # tile (rows 0-127, column 0): amax 448, scale 1
    a[1, 0] = 0.3              # ... so 0.3 rounds to the E4M3 value 0.3125
    a[200, 0] = 0.3            # alone in tile (rows 128-255, column 0)
    a[1, 1] = 0.3              # alone in tile (rows 0-127, column 1)
    b = np.full((256, 1), 448.0)
    got = fb.fp8_weight_grad(a, b)
    assert got.shape == (2, 1)
    assert of8.e4m3_round(np.float64(F32(0.3))) == 0.3125
    alone = scale_only(0.3)
    assert abs(alone - 0.3) < 1e-6 and alone != 0.3125
    assert got[0, 0] == 448.0 * (448.0 + 0.3125 + alone)
    assert got[1, 0] == 448.0 * alone
    # what the other tilings would give
    along_cols = 448.0 * (448.0 + alone + alone)     # 1x128 along the features
    rows64 = 448.0 * (448.0 + alone + alone)         # 0.3 at row 1, 448 at row 100
    blocks = 448.0 * 0.3125                          # 128x128: column 1 shares amax 448
    assert got[0, 0] not in (along_cols, rows64) and got[1, 0] != blocks


def test_weight_grad_pads_rows_with_zeros():
    rng = np.random.default_rng(3)
    a = rng.normal(size=(130, 3))
    b = rng.normal(size=(130, 2))
    qa, sa = fb.quantize_rows_along_tokens(a)
    assert qa.shape == (3, 256) and sa.shape == (3, 2)
    assert np.all(qa[:, 130:] == 0)
    # two extra zero rows change nothing
    a2 = np.concatenate([a, np.zeros((2, 3))])
    b2 = np.concatenate([b, np.zeros((2, 2))])
    assert np.array_equal(fb.fp8_weight_grad(a, b), fb.fp8_weight_grad(a2, b2))


class SmallLayer:
    """A small layer with E4M3 weights (the oracle's own 128x128 quantisation)."""

    def __init__(self, gate="sigmoid", T=40, d=256, I=128, N=8, K=2, Ks=1, seed=0):
        rng = np.random.default_rng(seed)
        self.T, self.d, self.I, self.N, self.K, self.Ks = T, d, I, N, K, Ks
        self.gate = gate
        self.x = rng.normal(size=(T, d)).astype(F32).astype(np.float64)
        self.w_r = rng.normal(scale=d ** -0.5, size=(N, d))
        self.bias = rng.uniform(-0.1, 0.1, N) if gate == "sigmoid" else None
        self.dh = rng.normal(size=(T, d)).astype(F32).astype(np.float64)
        self.w = {}
        for e in range(Ks + N):
            gu = rng.normal(scale=0.05, size=(2 * I, d)).astype(F32)
            wd = rng.normal(scale=0.05, size=(d, I)).astype(F32)
            qg, sg = of8.quantize_weight_128x128(gu)
            qd, sd = of8.quantize_weight_128x128(wd)
            guh = of8.dequant_weight(qg, sg)
            self.w[e] = (guh[:I], guh[I:], of8.dequant_weight(qd, sd))

    def kw(self):
        return dict(n_shared=self.Ks, gate=self.gate, top_k=self.K,
                    renorm=self.gate == "sigmoid", route_scale=2.5 if self.gate == "sigmoid"
                    else 1.0)

    def fp8(self, dh=None):
        return fb.moe_backward_fp8(self.x, self.w_r, self.bias, self.w.__getitem__,
                                   self.dh if dh is None else dh, **self.kw())

    def exact(self):
        return mb.moe_backward(self.x, self.w_r, self.bias, self.w.__getitem__, self.dh,
                               **self.kw())


@pytest.mark.parametrize("gate", ["sigmoid", "softmax"])
def test_token_scaling_is_exact_in_dx(gate):
    L = SmallLayer(gate)
    base = L.fp8()
    t = 7
    dh = L.dh.copy()
    dh[t] *= 4.0
    got = L.fp8(dh)
    assert np.array_equal(got["dx"][t], 4.0 * base["dx"][t])
    others = np.arange(L.T) != t
    assert np.array_equal(got["dx"][others], base["dx"][others])


def test_feature_scaling_is_exact_in_dw_down():
    L = SmallLayer("sigmoid", T=200)           # routed experts with more than 128 rows too
    base = L.fp8()
    c = 37
    dh = L.dh.copy()
    dh[:, c] *= 4.0
    got = L.fp8(dh)
    assert set(got["experts"]) == set(base["experts"])
    for e in base["experts"]:
        wd0, wd1 = base["experts"][e][2], got["experts"][e][2]
        assert np.array_equal(wd1[c], 4.0 * wd0[c])
        rest = np.arange(L.d) != c
        assert np.array_equal(wd1[rest], wd0[rest])


@pytest.mark.parametrize("gate", ["sigmoid", "softmax"])
def test_fp8_backward_is_near_the_exact_backward(gate):
    L = SmallLayer(gate, T=150, seed=1)
    got, ref = L.fp8(), L.exact()
    assert np.array_equal(got["idx"], ref["idx"])
    bound = 2.0 ** -3
    errs = {"dx": mo.max_abs_rel(got["dx"], ref["dx"]),
            "dw_r": mo.max_abs_rel(got["dw_r"], ref["dw_r"])}
    for e, (wg, wu, wd) in ref["experts"].items():
        g = got["experts"][e]
        errs[f"dw_gu{e}"] = mo.max_abs_rel(np.concatenate(g[:2]), np.concatenate([wg, wu]))
        errs[f"dw_down{e}"] = mo.max_abs_rel(g[2], wd)
    worst = max(errs, key=errs.get)
    print({k: f"{v:.2e}" for k, v in errs.items()})
    assert errs[worst] <= bound, f"{worst}: {errs[worst]:.3e}"
    # and FP8 is not the exact backward: the quantisation shows
    assert errs["dx"] > 1e-4


def test_round_bf16_matches_the_library_cast():
    import torch
    rng = np.random.default_rng(5)
    v = np.concatenate([rng.normal(size=4000) * 10.0 ** rng.integers(-6, 6, 4000),
                        [0.0, -0.0, 1.0, 1.00390625, 1.01171875, -3.0e38, 65504.0]])
    want = torch.from_numpy(v.astype(np.float32)).to(torch.bfloat16).double().numpy()
    assert np.array_equal(fb.round_bf16(v), want)


def test_bf16_intermediates_stay_near_fp32_ones():
    L = SmallLayer("sigmoid", T=150, seed=2)
    a = L.fp8()
    b = fb.moe_backward_fp8(L.x, L.w_r, L.bias, L.w.__getitem__, L.dh,
                            intermediates="bf16", **L.kw())
    assert not np.array_equal(a["dx"], b["dx"])
    assert mo.max_abs_rel(b["dx"], a["dx"]) < 3e-2
    for e in a["experts"]:
        assert mo.max_abs_rel(b["experts"][e][2], a["experts"][e][2]) < 5e-2
