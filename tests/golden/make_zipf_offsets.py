"""Writes tests/golden/zipf_offsets_v2_bf16_zipf.txt: the per-expert router
offsets that give the V2-shaped layer its skewed (Zipf s = 1.1) expert load.

Target loads: expert i (rank i+1) gets T*K * (i+1)^-1.1 / sum_r r^-1.1 tokens,
water-filled under the cap T (an expert sees each token at most once, so the
excess of a capped expert is shared out in proportion among the others until
no target exceeds T).  The offsets c_i are added to router column 0, whose
input feature is the constant 1, so every token's logit i moves by exactly
c_i (up to the bf16 rounding of the router weight).  Fixed-point steps
c_i += eta * log(target_i / load_i) (eta 0.7, then 0.25), with the loads counted from the oracle's
own routing of the full batch, keep the best iterate.

Calls only the oracle (and the input generator).  Run from the repo root:
    python tests/golden/make_zipf_offsets.py
"""
import os
import sys

import numpy as np

HERE = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, os.path.dirname(os.path.dirname(HERE)))

from oracle import moe_oracle as mo  # noqa: E402
from synth import recipes  # noqa: E402

S_ZIPF = 1.1


def capped_zipf_targets(T, K, N, s=S_ZIPF):
    w = np.arange(1, N + 1, dtype=np.float64) ** -s
    total = float(T * K)
    target = np.zeros(N)
    capped = np.zeros(N, dtype=bool)
    while True:
        free = ~capped
        rest = total - T * capped.sum()
        target[free] = rest * w[free] / w[free].sum()
        target[capped] = T
        over = free & (target > T)
        if not over.any():
            return target
        capped |= over


def loads(cfg, x, offsets):
    w_r = recipes.host_router(cfg, offsets)
    r = mo.route(x, w_r, None, gate=cfg.gate, top_k=cfg.top_k, renorm=cfg.renorm,
                 route_scale=cfg.route_scale)
    return np.bincount(r["idx"].reshape(-1), minlength=cfg.n_routed).astype(np.float64)


def main(iters=80):
    cfg = recipes.CONFIGS["v2_bf16_zipf"]
    T, K, N = cfg.T, cfg.top_k, cfg.n_routed
    target = capped_zipf_targets(T, K, N)
    x = recipes.host_x(cfg)
    c = np.log(target / target.mean()) * 1.5
    best, best_err = c.copy(), np.inf
    for it in range(iters):
        ld = loads(cfg, x, c)
        rel = np.abs(ld - target) / target
        err = float(rel.max())
        print(f"iter {it:2d}: max rel load error {err:.3f}  max/mean {ld.max() / ld.mean():.2f}  "
              f"min/mean {ld.min() / ld.mean():.3f}", flush=True)
        if err < best_err:
            best, best_err = c.copy(), err
        if err < 0.05:
            break
        eta = 0.7 if it < 8 else 0.25
        c = c + eta * np.log(target / np.maximum(ld, 0.5))
    ld = loads(cfg, x, best)
    out = os.path.join(HERE, "zipf_offsets_v2_bf16_zipf.txt")
    hdr = (f"router column-0 offsets c_i of the skewed V2-shaped layer (T={T}, N={N}, K={K}, "
           f"Zipf s={S_ZIPF} water-filled under cap T); written by make_zipf_offsets.py\n"
           f"achieved loads: max/mean {ld.max() / ld.mean():.3f}, min/mean "
           f"{ld.min() / ld.mean():.3f}, max relative error vs target {best_err:.4f}")
    np.savetxt(out, best.astype(np.float32), fmt="%.8e", header=hdr)
    np.savetxt(os.path.join(HERE, "zipf_loads_v2_bf16_zipf.txt"),
               np.stack([target, ld], axis=1), fmt="%.3f",
               header="target load, achieved load (tokens per routed expert, oracle routing)")
    print("wrote", out)


if __name__ == "__main__":
    main()
