"""Layer shapes and input recipes of the synthetic DeepSeekMoE workloads.

A recipe fixes the layer's shape (T tokens, hidden d, Ks shared + N routed
SwiGLU experts of width I, top-K, gating mode, group limit) and the value
distribution of each input.  Inputs are produced either on a CUDA device (the
bench and the GPU side of the tests) or on the host (the oracle side of the
tests); both routes give the same bits.

Tensor layouts (row-major, contiguous):
  x      [T, d]             hidden states u_t (layer input)
  w_r    [N, d]             router centroids e_i
  bias   [N] fp32           selection bias b_i (sigmoid gating only)
  w_gu   [Ks+N, 2I, d]      per expert: gate rows 0..I-1, up rows I..2I-1
  w_down [Ks+N, d, I]       per expert down projection
Experts 0..Ks-1 are the shared experts; routed expert j is expert Ks+j.
"""
from __future__ import annotations

import dataclasses
from dataclasses import dataclass
from typing import Optional, Sequence

import numpy as np

from . import (TID_BIAS, TID_WD, TID_WGU, TID_WR, TID_X, bf16_bits_to_f64, host_normal,
               host_uniform)


@dataclass(frozen=True)
class LayerConfig:
    name: str
    T: int
    d: int
    n_shared: int
    n_routed: int
    top_k: int
    inter: int
    gate: str              # "softmax" | "sigmoid"
    renorm: bool
    route_scale: float
    n_group: int
    topk_group: int
    dtype: str             # "f32" | "bf16" | "e4m3" (e4m3: bf16 activations in, FP8 GEMMs)
    x_sigma: float = 1.0
    wr_sigma: float = 0.02
    wgu_sigma: float = 0.02
    wd_sigma: float = 0.02
    bias_half_range: Optional[float] = None   # bias ~ U(-a, a)
    zipf: bool = False                        # skewed load: constant feature x[:,0] = 1, w_r[:,0] += c_i
    seed: int = 0

    @property
    def n_experts(self) -> int:
        return self.n_shared + self.n_routed

    @property
    def rows_routed(self) -> int:
        return self.T * self.top_k

    def with_T(self, T: int) -> "LayerConfig":
        return dataclasses.replace(self, T=T, name=f"{self.name.split('@')[0]}@T{T}")

    def expert_gemm_flops(self) -> float:
        """Algorithmic FLOPs of the expert GEMMs: 3 matrices x 2 flop/MAC, active experts only."""
        return 6.0 * self.d * self.inter * self.T * (self.top_k + self.n_shared)

    def router_flops(self) -> float:
        return 2.0 * self.T * self.d * self.n_routed


CONFIGS = {
    # Tiny layer, fp32: softmax gating with renormalised top-k weights;
    # weights N(0, 1/sqrt(fan_in)).
    "tiny_f32": LayerConfig("tiny_f32", T=64, d=256, n_shared=1, n_routed=16, top_k=4, inter=64,
                            gate="softmax", renorm=True, route_scale=1.0, n_group=1, topk_group=1,
                            dtype="f32", x_sigma=1.0, wr_sigma=1 / 16, wgu_sigma=1 / 16,
                            wd_sigma=1 / 8),
    # DeepSeekMoE-16B-shaped: 2 shared + 64 routed of width 1408, top-6, softmax, no renorm.
    "dsmoe16b_bf16": LayerConfig("dsmoe16b_bf16", T=4096, d=2048, n_shared=2, n_routed=64,
                                 top_k=6, inter=1408, gate="softmax", renorm=False,
                                 route_scale=1.0, n_group=1, topk_group=1, dtype="bf16"),
    # DeepSeek-V2-shaped: 2 shared + 160 routed of width 1536, top-6, softmax, Zipf(1.1) load.
    "v2_bf16_zipf": LayerConfig("v2_bf16_zipf", T=8192, d=5120, n_shared=2, n_routed=160,
                                top_k=6, inter=1536, gate="softmax", renorm=False,
                                route_scale=1.0, n_group=1, topk_group=1, dtype="bf16",
                                zipf=True),
    # DeepSeek-V3-shaped: 1 shared + 256 routed of width 2048, top-8, sigmoid + bias,
    # 8 groups / top-4 groups, renormalised and scaled by 2.5.
    "v3_bf16": LayerConfig("v3_bf16", T=16384, d=7168, n_shared=1, n_routed=256, top_k=8,
                           inter=2048, gate="sigmoid", renorm=True, route_scale=2.5, n_group=8,
                           topk_group=4, dtype="bf16", bias_half_range=0.1),
    # The same V3 layer with FP8 E4M3 expert GEMMs (1x128 activation tiles, 128x128
    # weight blocks); T is swept over 256, 2048, 16384, 65536.
    "v3_fp8": LayerConfig("v3_fp8", T=16384, d=7168, n_shared=1, n_routed=256, top_k=8,
                          inter=2048, gate="sigmoid", renorm=True, route_scale=2.5, n_group=8,
                          topk_group=4, dtype="e4m3", bias_half_range=0.1),
}
FP8_SWEEP_T = (256, 2048, 16384, 65536)


def small_variant(cfg: LayerConfig, T: int, d: int, inter: int, n_routed: Optional[int] = None,
                  name: Optional[str] = None) -> LayerConfig:
    """A reduced copy of a recipe (same gating, dtype and distributions)."""
    n = cfg.n_routed if n_routed is None else n_routed
    return dataclasses.replace(cfg, name=name or f"{cfg.name}-small", T=T, d=d, inter=inter,
                               n_routed=n)


# ----------------------------------------------------------------------------- host side
def _round_like(cfg: LayerConfig, v32: np.ndarray) -> np.ndarray:
    """fp32 values -> the layer's storage precision, returned as float64."""
    if cfg.dtype == "f32":
        return v32.astype(np.float64)
    import torch
    return torch.from_numpy(v32).to(torch.bfloat16).to(torch.float64).numpy()


def host_x(cfg: LayerConfig, rows: Optional[Sequence[int]] = None) -> np.ndarray:
    """Hidden states as float64 (exactly the stored values); optionally only some rows."""
    if rows is None:
        v = host_normal(cfg.T * cfg.d, cfg.x_sigma, cfg.seed, TID_X).reshape(cfg.T, cfg.d)
    else:
        v = np.stack([host_normal(cfg.d, cfg.x_sigma, cfg.seed, TID_X, int(t) * cfg.d)
                      for t in rows]) if len(rows) else np.zeros((0, cfg.d), np.float32)
    if cfg.zipf:
        v = v.copy()
        v[:, 0] = np.float32(1.0)
    return _round_like(cfg, v)


def host_router(cfg: LayerConfig, zipf_offsets: Optional[np.ndarray] = None) -> np.ndarray:
    v = host_normal(cfg.n_routed * cfg.d, cfg.wr_sigma, cfg.seed, TID_WR).reshape(cfg.n_routed,
                                                                                  cfg.d)
    if cfg.zipf:
        if zipf_offsets is None:
            raise ValueError("skewed-load recipe needs its per-expert logit offsets")
        v = v.copy()
        v[:, 0] = v[:, 0] + np.asarray(zipf_offsets, dtype=np.float32)
    return _round_like(cfg, v)


def host_bias(cfg: LayerConfig) -> Optional[np.ndarray]:
    if cfg.bias_half_range is None:
        return None
    a = cfg.bias_half_range
    return host_uniform(cfg.n_routed, -a, a, cfg.seed, TID_BIAS).astype(np.float64)


def host_expert(cfg: LayerConfig, e: int):
    """(w_gate [I,d], w_up [I,d], w_down [d,I]) of expert e as float64 (bf16/fp32 values)."""
    I, d = cfg.inter, cfg.d
    bf = cfg.dtype != "f32"
    gu = host_normal(2 * I * d, cfg.wgu_sigma, cfg.seed, TID_WGU, e * 2 * I * d, bf16=bf)
    dn = host_normal(d * I, cfg.wd_sigma, cfg.seed, TID_WD, e * d * I, bf16=bf)
    if bf:
        gu, dn = bf16_bits_to_f64(gu), bf16_bits_to_f64(dn)
    else:
        gu, dn = gu.astype(np.float64), dn.astype(np.float64)
    gu = gu.reshape(2 * I, d)
    return gu[:I], gu[I:], dn.reshape(d, I)


def host_expert_bits(cfg: LayerConfig, e: int):
    """Stored (bf16 bit patterns or fp32) gate/up [2I,d] and down [d,I] of expert e."""
    I, d = cfg.inter, cfg.d
    bf = cfg.dtype != "f32"
    gu = host_normal(2 * I * d, cfg.wgu_sigma, cfg.seed, TID_WGU, e * 2 * I * d, bf16=bf)
    dn = host_normal(d * I, cfg.wd_sigma, cfg.seed, TID_WD, e * d * I, bf16=bf)
    return gu.reshape(2 * I, d), dn.reshape(d, I)


# ----------------------------------------------------------------------------- device side
def device_inputs(cfg: LayerConfig, device="cuda", zipf_offsets: Optional[np.ndarray] = None):
    """All layer inputs on a CUDA device, in the layer's storage dtype.

    Returns a dict with x, w_r, bias (or None), w_gu, w_down."""
    import torch

    from . import dev_fill_normal, dev_fill_uniform
    dt = torch.float32 if cfg.dtype == "f32" else torch.bfloat16
    E, I, d, N, T = cfg.n_experts, cfg.inter, cfg.d, cfg.n_routed, cfg.T
    x32 = torch.empty(T, d, dtype=torch.float32, device=device)
    dev_fill_normal(x32, cfg.x_sigma, cfg.seed, TID_X)
    wr32 = torch.empty(N, d, dtype=torch.float32, device=device)
    dev_fill_normal(wr32, cfg.wr_sigma, cfg.seed, TID_WR)
    if cfg.zipf:
        if zipf_offsets is None:
            raise ValueError("skewed-load recipe needs its per-expert logit offsets")
        x32[:, 0] = 1.0
        wr32[:, 0] += torch.as_tensor(np.asarray(zipf_offsets, np.float32), device=device)
    x = x32.to(dt)
    del x32
    w_r = wr32.to(dt)
    del wr32
    bias = None
    if cfg.bias_half_range is not None:
        bias = torch.empty(N, dtype=torch.float32, device=device)
        dev_fill_uniform(bias, -cfg.bias_half_range, cfg.bias_half_range, cfg.seed, TID_BIAS)
    w_gu = torch.empty(E, 2 * I, d, dtype=dt, device=device)
    dev_fill_normal(w_gu, cfg.wgu_sigma, cfg.seed, TID_WGU)
    w_down = torch.empty(E, d, I, dtype=dt, device=device)
    dev_fill_normal(w_down, cfg.wd_sigma, cfg.seed, TID_WD)
    return {"x": x, "w_r": w_r, "bias": bias, "w_gu": w_gu, "w_down": w_down}
