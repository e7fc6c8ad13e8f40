"""Seeded synthetic inputs for the DeepSeekMoE layer forward.

This module is the one piece shared by the oracle side (tests, the CPU
baseline) and the CUDA side (tests, bench): it produces the layer's inputs and
nothing else.  None of the MoE method's arithmetic lives here.

Every tensor is a pure function of (seed, tensor id, flat element index)
through a counter-based generator (splitmix64 + Irwin-Hall(4) normals), with a
host implementation and a device implementation that agree bit for bit, so the
oracle can regenerate any block of the weights (one expert) on the host
without copying it back from the GPU.
"""
from __future__ import annotations

import ctypes
import math
import os
import subprocess
from typing import Optional

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_LIB_PATH = os.path.join(_HERE, "libmoesynth.so")
_lib: Optional[ctypes.CDLL] = None

# Tensor ids of the layer inputs.
TID_X, TID_WR, TID_WGU, TID_WD, TID_BIAS = 0, 1, 2, 3, 4

# Standard deviation of the centred Irwin-Hall(4) sum of 16-bit uniforms.
_IH4_STD = math.sqrt((65536.0 ** 2 - 1.0) / 3.0)


def build(force: bool = False) -> str:
    """Compile libmoesynth.so in-tree with nvcc (sm_100a device code)."""
    src = os.path.join(_HERE, "synth.cu")
    hdr = os.path.join(_HERE, "synth_core.h")
    if (not force and os.path.exists(_LIB_PATH)
            and os.path.getmtime(_LIB_PATH) >= max(os.path.getmtime(src), os.path.getmtime(hdr))):
        return _LIB_PATH
    nvcc = os.environ.get("NVCC", "/usr/local/cuda/bin/nvcc")
    cmd = [nvcc, "-O3", "-std=c++17", "-gencode", "arch=compute_100a,code=sm_100a",
           "-lineinfo", "-Xcompiler", "-fPIC,-ffp-contract=off", "-shared",
           "-o", _LIB_PATH, src]
    subprocess.run(cmd, check=True)
    return _LIB_PATH


def lib() -> ctypes.CDLL:
    global _lib
    if _lib is None:
        if not os.path.exists(_LIB_PATH):
            build()
        L = ctypes.CDLL(_LIB_PATH)
        u64, i32, f32, vp = ctypes.c_uint64, ctypes.c_int, ctypes.c_float, ctypes.c_void_p
        L.syn_key_of.restype = u64
        L.syn_key_of.argtypes = [u64, u64]
        for name, extra in (("normal_f32", [f32]), ("normal_bf16", [f32]),
                            ("uniform_f32", [f32, f32])):
            h = getattr(L, "syn_host_" + name)
            h.restype = i32
            h.argtypes = [vp, u64, u64, u64, u64] + extra + [i32]
            d = getattr(L, "syn_dev_" + name)
            d.restype = i32
            d.argtypes = [vp, u64, u64, u64, u64] + extra + [vp]
        _lib = L
    return _lib


def normal_scale(sigma: float) -> float:
    """fp32 multiplier that turns the Irwin-Hall integer into N(0, sigma^2)-like values."""
    return float(np.float32(sigma / _IH4_STD))


def host_threads() -> int:
    return max(1, min(os.cpu_count() or 1, 32))


# ----------------------------------------------------------------------------- host fills
def host_normal(n: int, sigma: float, seed: int, tid: int, offset: int = 0,
                bf16: bool = False) -> np.ndarray:
    """n elements of stream (seed, tid) starting at flat index `offset`.

    Returns float32 values, or (bf16=True) uint16 bf16 bit patterns."""
    out = np.empty(n, dtype=np.uint16 if bf16 else np.float32)
    fn = lib().syn_host_normal_bf16 if bf16 else lib().syn_host_normal_f32
    rc = fn(out.ctypes.data, n, seed, tid, offset, normal_scale(sigma), host_threads())
    if rc:
        raise RuntimeError("synth host fill failed")
    return out


def host_uniform(n: int, lo: float, hi: float, seed: int, tid: int, offset: int = 0) -> np.ndarray:
    out = np.empty(n, dtype=np.float32)
    rc = lib().syn_host_uniform_f32(out.ctypes.data, n, seed, tid, offset, lo, hi, host_threads())
    if rc:
        raise RuntimeError("synth host fill failed")
    return out


def bf16_bits_to_f64(bits: np.ndarray) -> np.ndarray:
    """Exact widening of bf16 bit patterns to float64."""
    return (bits.astype(np.uint32) << 16).view(np.float32).astype(np.float64)


# ----------------------------------------------------------------------------- device fills
def dev_fill_normal(t, sigma: float, seed: int, tid: int, offset: int = 0, stream=None) -> None:
    """Fill a contiguous CUDA tensor (float32 or bfloat16) in place."""
    import torch
    assert t.is_cuda and t.is_contiguous()
    s = stream if stream is not None else torch.cuda.current_stream().cuda_stream
    if t.dtype == torch.float32:
        rc = lib().syn_dev_normal_f32(t.data_ptr(), t.numel(), seed, tid, offset,
                                      normal_scale(sigma), s)
    elif t.dtype == torch.bfloat16:
        rc = lib().syn_dev_normal_bf16(t.data_ptr(), t.numel(), seed, tid, offset,
                                       normal_scale(sigma), s)
    else:
        raise TypeError(t.dtype)
    if rc:
        raise RuntimeError(f"synth device fill failed: cudaError {rc}")


def dev_fill_uniform(t, lo: float, hi: float, seed: int, tid: int, offset: int = 0,
                     stream=None) -> None:
    import torch
    assert t.is_cuda and t.is_contiguous() and t.dtype == torch.float32
    s = stream if stream is not None else torch.cuda.current_stream().cuda_stream
    rc = lib().syn_dev_uniform_f32(t.data_ptr(), t.numel(), seed, tid, offset, lo, hi, s)
    if rc:
        raise RuntimeError(f"synth device fill failed: cudaError {rc}")
