"""FP8 E4M3 fine-grained quantisation and the emulating FP8 layer (oracle side).

TEST INFRASTRUCTURE: used only by the tests, the smoke check and the bench's
CPU baseline leg.  Shares no code with the CUDA path.

The recipe follows DeepSeek Technical Report: MoE Architecture, §3.6 (FP8
mixed precision: E4M3 for every linear forward GEMM, activations grouped per
1x128 tile, weights per 128x128 block, fp32 accumulation with promotion every
128 elements; MoE gating stays BF16) and DeepSeek 모델 완벽 분석 §4.2 (tile-
and block-wise scaling, E4M3 everywhere, FP32 accumulation).

E4M3 is the OCP 8-bit floating point format "E4M3" (bias 7, no infinities,
largest finite 448 = 1.75 * 2^8, smallest normal 2^-6, subnormal spacing
2^-9).  Conversion is round-to-nearest-even with saturation to +-448.

Scale rule (the pages give none; reading taken): per tile or block,
amax = max |v| in fp32, scale = fp32(amax / 448), inverse = fp32(448 / amax),
code = E4M3(fp32(v * inverse)); the dequantised value is code * scale.  A tile
whose amax is 0 gets scale 0 and all-zero codes.
"""
from __future__ import annotations

import numpy as np

E4M3_MAX = 448.0
F32 = np.float32


def e4m3_round(v: np.ndarray) -> np.ndarray:
    """Nearest E4M3 value (ties to even, saturating at +-448), as float64."""
    v = np.asarray(v, np.float64)
    a = np.abs(v)
    _, ex = np.frexp(a)                      # a = m * 2^ex, m in [0.5, 1)
    e = np.maximum(ex - 1, -6)               # binade exponent; subnormals share 2^-6's spacing
    q = np.ldexp(1.0, e - 3)                 # 3 fraction bits -> spacing 2^(e-3)
    r = np.rint(a / q) * q                   # a / q is exact (power of two); rint = ties-to-even
    r = np.minimum(r, E4M3_MAX)
    return np.copysign(r, v)


def e4m3_decode(code: int) -> float:
    """Value of an 8-bit E4M3 code (NaN for S.1111.111), from the format's definition."""
    s = -1.0 if code & 0x80 else 1.0
    e = (code >> 3) & 0xF
    m = code & 0x7
    if e == 0xF and m == 0x7:
        return float("nan")
    if e == 0:
        return s * m * 2.0 ** -9
    return s * (1.0 + m / 8.0) * 2.0 ** (e - 7)


def e4m3_encode(v: np.ndarray) -> np.ndarray:
    """E4M3 codes (uint8) of values that are already E4M3-representable."""
    v = np.asarray(v, np.float64)
    table = np.array([e4m3_decode(c) for c in range(256)])
    out = np.zeros(v.shape, np.uint8)
    flat, o = v.reshape(-1), out.reshape(-1)
    finite = np.where(np.isnan(table), np.inf, table)
    pos = np.argsort(finite[:127], kind="stable")      # codes 0..126: +0 .. +448
    for i, x in enumerate(flat):
        c = int(np.searchsorted(finite[:127][pos], abs(x)))
        code = int(pos[c])
        if finite[code] != abs(x):
            raise ValueError(f"{x} is not an E4M3 value")
        o[i] = code | (0x80 if (x < 0 or (x == 0 and np.signbit(x))) else 0)
    return out


def _quantize_groups(g32: np.ndarray):
    """g32 [..., n] fp32 groups -> (codes as float64 values, fp32 scale [...])."""
    g32 = np.asarray(g32, F32)
    amax = np.max(np.abs(g32), axis=-1)
    zero = amax == 0
    safe = np.where(zero, F32(1.0), amax).astype(F32)
    scale = (safe / F32(E4M3_MAX)).astype(F32)
    inv = (F32(E4M3_MAX) / safe).astype(F32)
    prod = (g32 * inv[..., None]).astype(F32)
    q = e4m3_round(prod.astype(np.float64))
    q = np.where(zero[..., None], 0.0, q)
    scale = np.where(zero, F32(0.0), scale).astype(F32)
    return q, scale


def quantize_act_1x128(x: np.ndarray):
    """Activations [rows, cols] (cols % 128 == 0) -> (q [rows, cols], scale [rows, cols/128])."""
    x = np.asarray(x)
    rows, cols = x.shape
    q, s = _quantize_groups(x.astype(F32).reshape(rows, cols // 128, 128))
    return q.reshape(rows, cols), s


def quantize_weight_128x128(w: np.ndarray):
    """Weights [r, c] (both % 128 == 0) -> (q [r, c], scale [r/128, c/128])."""
    w = np.asarray(w)
    r, c = w.shape
    blk = w.astype(F32).reshape(r // 128, 128, c // 128, 128).transpose(0, 2, 1, 3)
    q, s = _quantize_groups(blk.reshape(r // 128, c // 128, 128 * 128))
    q = q.reshape(r // 128, c // 128, 128, 128).transpose(0, 2, 1, 3).reshape(r, c)
    return q, s


def dequant_act(q: np.ndarray, s: np.ndarray) -> np.ndarray:
    rows, cols = q.shape
    return (q.reshape(rows, cols // 128, 128) * s.astype(np.float64)[..., None]).reshape(rows, cols)


def dequant_weight(q: np.ndarray, s: np.ndarray) -> np.ndarray:
    r, c = q.shape
    big = np.repeat(np.repeat(s.astype(np.float64), 128, axis=0), 128, axis=1)
    return q * big


def fp8_swiglu_ffn(v_hat: np.ndarray, wg_hat: np.ndarray, wu_hat: np.ndarray,
                   wd_hat: np.ndarray) -> np.ndarray:
    """SwiGLU expert with FP8 operands on both GEMMs.

    v_hat and the weights are dequantised E4M3 values; each 128-element block
    of a dot product is exact in float64 and is scaled by its two fp32 scales,
    which equals the float64 dot product of the dequantised operands.  The
    intermediate H is held in fp32 and requantised per 1x128 tile before the
    down projection."""
    hmid = (v_hat @ wg_hat.T)
    with np.errstate(over="ignore"):
        hmid = hmid / (1.0 + np.exp(-hmid)) * (v_hat @ wu_hat.T)
    hq, hs = quantize_act_1x128(hmid.astype(F32))
    return dequant_act(hq, hs) @ wd_hat.T
