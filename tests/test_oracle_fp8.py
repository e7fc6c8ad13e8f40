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
