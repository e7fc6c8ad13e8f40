"""Pins of the oracle's FP8 E4M3 fine-grained quantisation.

E4M3 facts come from the format's definition (OCP 8-bit floating point, E4M3:
bias 7, no infinities, S.1111.111 is NaN, largest finite 448); rounding is
checked by brute force against the decoded code table and against torch's
float8_e4m3fn cast (a library routine) on in-range values.
"""
import numpy as np
import pytest
import torch

from oracle import fp8


def test_e4m3_code_table_closed_forms():
    assert fp8.e4m3_decode(0x7E) == 448.0           # S.1111.110: 1.75 * 2^8
    assert np.isnan(fp8.e4m3_decode(0x7F))
    assert fp8.e4m3_decode(0x38) == 1.0             # exponent field 7 = bias
    assert fp8.e4m3_decode(0x08) == 2.0 ** -6       # smallest normal
    assert fp8.e4m3_decode(0x01) == 2.0 ** -9       # smallest subnormal
    assert fp8.e4m3_decode(0x07) == 7 * 2.0 ** -9   # largest subnormal
    assert fp8.e4m3_decode(0xB8) == -1.0
    finite = [fp8.e4m3_decode(c) for c in range(0x80) if not np.isnan(fp8.e4m3_decode(c))]
    assert len(finite) == 127 and len(set(finite)) == 127


def _nearest_even_by_table(v):
    table = sorted({fp8.e4m3_decode(c) for c in range(0x7F)})      # +0 .. 448
    a = min(abs(v), 448.0)
    best = min(table, key=lambda q: abs(q - a))
    ties = [q for q in table if abs(q - a) == abs(best - a)]
    if len(ties) > 1:
        # ties to the code with an even mantissa field
        codes = {fp8.e4m3_decode(c): c for c in range(0x7F)}
        best = [q for q in ties if codes[q] % 2 == 0][0]
    return np.copysign(best, v)


def test_e4m3_round_brute_force():
    rng = np.random.default_rng(0)
    vals = np.concatenate([
        rng.uniform(-500, 500, 400), rng.uniform(-1, 1, 400) * 2.0 ** -5,
        rng.normal(size=400) * 3,
        # exact midpoints between neighbours (ties)
        np.array([1.0625, 1.1875, 2.0 ** -9 * 0.5, 2.0 ** -9 * 1.5, 464.0, 0.0]),
    ])
    got = fp8.e4m3_round(vals)
    want = np.array([_nearest_even_by_table(v) for v in vals])
    np.testing.assert_array_equal(got, want)


def test_e4m3_round_matches_library_cast_in_range():
    rng = np.random.default_rng(1)
    v = np.concatenate([rng.uniform(-448, 448, 20000), rng.normal(size=20000) * 0.01]).astype(
        np.float32)
    lib = torch.from_numpy(v).to(torch.float8_e4m3fn).to(torch.float64).numpy()
    np.testing.assert_array_equal(fp8.e4m3_round(v.astype(np.float64)), lib)


def test_e4m3_encode_roundtrip():
    vals = np.array([fp8.e4m3_decode(c) for c in range(256) if c not in (0x7F, 0xFF)])
    codes = fp8.e4m3_encode(vals)
    back = np.array([fp8.e4m3_decode(int(c)) for c in codes])
    np.testing.assert_array_equal(back, vals)


def test_activation_tiles_1x128():
    rng = np.random.default_rng(2)
    x = rng.normal(size=(6, 384)).astype(np.float32)
    x[2, 128:256] = 0.0                                # an all-zero tile
    x[4, :128] *= 1000.0                               # one tile with a large range
    q, s = fp8.quantize_act_1x128(x)
    assert s.shape == (6, 3) and s.dtype == np.float32
    for r in range(6):
        for b in range(3):
            tile = x[r, b * 128:(b + 1) * 128]
            amax = np.float32(np.max(np.abs(tile)))
            if amax == 0:
                assert s[r, b] == 0 and np.all(q[r, b * 128:(b + 1) * 128] == 0)
                continue
            assert s[r, b] == np.float32(amax / np.float32(448.0))
            qt = q[r, b * 128:(b + 1) * 128]
            assert np.max(np.abs(qt)) == 448.0       # the tile's amax lands on the top code
            # every code is an E4M3 value, and dequantisation is within half a step
            np.testing.assert_array_equal(fp8.e4m3_round(qt), qt)
            err = np.abs(qt * np.float64(s[r, b]) - tile)
            bound = np.abs(tile) * 2.0 ** -4 + np.float64(s[r, b]) * 2.0 ** -10 + 1e-30
            assert np.all(err <= bound * 1.0001)


def test_weight_blocks_128x128():
    rng = np.random.default_rng(3)
    w = (rng.normal(size=(256, 384)) * 0.02).astype(np.float32)
    w[130, 300] = 5.0                                  # lives in block (1, 2)
    q, s = fp8.quantize_weight_128x128(w)
    assert s.shape == (2, 3)
    for i in range(2):
        for j in range(3):
            blk = w[i * 128:(i + 1) * 128, j * 128:(j + 1) * 128]
            assert s[i, j] == np.float32(np.float32(np.abs(blk).max()) / np.float32(448.0))
    assert s[1, 2] == np.float32(np.float32(5.0) / np.float32(448.0))
    assert s[1, 1] < s[1, 2] / 10
    wh = fp8.dequant_weight(q, s)
    assert np.max(np.abs(wh - w)) <= np.max(np.abs(w)) * 2.0 ** -4


def test_fp8_ffn_exact_on_representable_inputs():
    # With activations and weights on E4M3 codes times a power of two, and the
    # top code 448 present in every tile and block, the scales are exact
    # powers of two and quantisation is the identity on the inputs, so the
    # FP8 FFN equals the fp64 FFN up to the requantised H.
    from oracle import moe_oracle as mo
    rng = np.random.default_rng(4)
    codes = np.array([fp8.e4m3_decode(c) for c in range(0x7F)])
    d, I = 128, 128

    def on_codes(shape, p2):
        m = rng.choice(codes, size=shape) * rng.choice([-1, 1], size=shape)
        m[..., 0] = 448.0
        return m * 2.0 ** p2

    v, wg, wu, wd = on_codes((3, d), -8), on_codes((I, d), -12), on_codes((I, d), -12), \
        on_codes((d, I), -12)
    vq, vs = fp8.quantize_act_1x128(v.astype(np.float32))
    np.testing.assert_array_equal(fp8.dequant_act(vq, vs), v)
    wq, ws = fp8.quantize_weight_128x128(wg.astype(np.float32))
    np.testing.assert_array_equal(fp8.dequant_weight(wq, ws), wg)
    exact = mo.swiglu_ffn(v, wg, wu, wd)
    got = fp8.fp8_swiglu_ffn(v, wg, wu, wd)
    assert mo.max_abs_rel(got, exact) < 2.0 ** -4


# ----------------------------------------------------------------------------- H requantisation
# The FP8 FFN requantises its intermediate H = SiLU(v W_gate^T) * (v W_up^T)
# per 1x128 tile along I before the down projection ("DeepSeek Technical
# Report: MoE Architecture", §3.6: activations are grouped per 1x128 tile and
# every linear forward GEMM takes E4M3 inputs).  This construction makes H
# known in closed form: v[:, 0] = 1 and every W_gate row is 64 e_0, so each
# gate pre-activation is 64 and SiLU(64) = 64 / (1 + e^-64) = 64 exactly in
# float64 (e^-64 < 2^-53); W_up row i is e_{1+i}, so H[t, i] = 64 * v[t, 1+i];
# W_down is the identity, so the FFN returns the dequantised H itself.  The
# expected codes below are worked out by hand from the E4M3 format (3 fraction
# bits, subnormal spacing 2^-9, ties to even) and the tile rule
# scale = amax / 448.
I_H = 256


def _h_design():
    H = np.zeros((2, I_H))
    want = np.zeros((2, I_H))
    # row 0, tile 0 (columns 0..127): amax 448 at column 100 -> scale 1, codes = values
    H[0, 100], want[0, 100] = 448.0, 448.0
    H[0, 1], want[0, 1] = 1.0, 1.0                   # representable
    H[0, 2], want[0, 2] = 1.0625, 1.0                # midpoint of 1 and 1.125: even mantissa -> 1
    H[0, 3], want[0, 3] = 2.0 ** -10, 0.0            # midpoint of 0 and 2^-9 -> 0
    H[0, 4], want[0, 4] = 3 * 2.0 ** -10, 2.0 ** -8  # midpoint of 1 and 2 x 2^-9 -> 2 x 2^-9
    H[0, 5], want[0, 5] = 300.0, 288.0               # spacing 32 in [256, 512): nearest is 288
    H[0, 7], want[0, 7] = 5 * 2.0 ** -11, 2.0 ** -9  # 1.25 x 2^-9 -> 1 x 2^-9
    # row 0, tile 1 (columns 128..255): amax 28 -> scale 2^-4 (28 * 16 = 448)
    H[0, 200], want[0, 200] = 28.0, 28.0
    H[0, 129], want[0, 129] = 0.53125, 0.5           # 8.5 after scaling: tie between 8 and 9 -> 8
    H[0, 130], want[0, 130] = 2.0 ** -14, 0.0        # 2^-10 after scaling: tie at zero -> 0
    # row 1, tile 0: amax 1344 -> scale 3 (fp32 448/1344 is inexact but 1344 and 3 land exactly)
    H[1, 100], want[1, 100] = 1344.0, 1344.0
    H[1, 1], want[1, 1] = 3.0, 3.0
    # row 1, tile 1 stays all zero: amax 0 -> scale 0, codes 0
    return H, want


def _h_layer(H):
    d = 1 + I_H
    v = np.zeros((2, d))
    v[:, 0] = 1.0
    v[:, 1:] = H / 64.0                              # exact: the chosen H are dyadic
    wg = np.zeros((I_H, d))
    wg[:, 0] = 64.0
    wu = np.zeros((I_H, d))
    wu[np.arange(I_H), 1 + np.arange(I_H)] = 1.0
    return v, wg, wu, np.eye(I_H)


def test_fp8_ffn_requantises_h_per_1x128_tile():
    H, want = _h_design()
    v, wg, wu, wd = _h_layer(H)
    from oracle import moe_oracle as mo
    # the construction really gives H: the unquantised FFN returns it exactly
    np.testing.assert_array_equal(mo.swiglu_ffn(v, wg, wu, wd), H)
    got = fp8.fp8_swiglu_ffn(v, wg, wu, wd)
    np.testing.assert_array_equal(got, want)


def _mutant_requant(kind):
    """Wrong readings of the H requantisation, planted in the oracle on the CPU."""
    def quant(h):
        h = np.asarray(h, np.float32)
        rows, cols = h.shape
        if kind == "none":
            return h.astype(np.float64), None
        if kind == "1x64":
            q, s = fp8._quantize_groups(h.reshape(rows, cols // 64, 64))
            return (q * s.astype(np.float64)[..., None]).reshape(rows, cols), None
        if kind == "128x128":   # one block over both rows and 128 columns
            blk = h.reshape(rows, cols // 128, 128).transpose(1, 0, 2).reshape(cols // 128, -1)
            q, s = fp8._quantize_groups(blk)
            deq = (q * s.astype(np.float64)[..., None]).reshape(cols // 128, rows, 128)
            return deq.transpose(1, 0, 2).reshape(rows, cols), None
        if kind == "column":    # tiles along the token axis instead of along I
            q, s = fp8._quantize_groups(h.T.copy())
            return (q * s.astype(np.float64)[..., None]).T, None
        raise ValueError(kind)
    return quant


def test_h_requantisation_pin_catches_wrong_readings(monkeypatch):
    H, want = _h_design()
    v, wg, wu, wd = _h_layer(H)
    for kind in ("none", "1x64", "128x128", "column"):
        mutant = _mutant_requant(kind)
        monkeypatch.setattr(fp8, "quantize_act_1x128", mutant)
        monkeypatch.setattr(fp8, "dequant_act", lambda deq, _s: deq)
        got = fp8.fp8_swiglu_ffn(v, wg, wu, wd)
        monkeypatch.undo()
        assert not np.array_equal(got, want), f"the pin does not tell apart the {kind!r} reading"
