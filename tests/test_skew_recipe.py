"""The skewed-load (Zipf s = 1.1) recipe of the V2-shaped layer: the stored
router offsets, routed by the oracle, reproduce the stored loads, and those
loads are within 5% of the capped Zipf targets."""
import os
import sys

import numpy as np

from oracle import moe_oracle as mo
from synth import recipes

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")
sys.path.insert(0, GOLDEN)
from make_zipf_offsets import capped_zipf_targets  # noqa: E402


def test_capped_targets():
    t = capped_zipf_targets(8192, 6, 160)
    assert abs(t.sum() - 8192 * 6) < 1e-6
    assert t.max() == 8192 and np.all(np.diff(t) <= 1e-9)
    # the uncapped head would need more tokens than exist (the recipe's point)
    w = np.arange(1, 161) ** -1.1
    assert 8192 * 6 * w[0] / w.sum() > 8192


def test_stored_offsets_reproduce_loads():
    cfg = recipes.CONFIGS["v2_bf16_zipf"]
    offs = np.loadtxt(os.path.join(GOLDEN, "zipf_offsets_v2_bf16_zipf.txt"))
    tl = np.loadtxt(os.path.join(GOLDEN, "zipf_loads_v2_bf16_zipf.txt"))
    r = mo.route(recipes.host_x(cfg), recipes.host_router(cfg, offs), None, gate="softmax",
                 top_k=cfg.top_k)
    loads = np.bincount(r["idx"].reshape(-1), minlength=cfg.n_routed)
    assert np.array_equal(loads, tl[:, 1])
    assert np.max(np.abs(loads - tl[:, 0]) / tl[:, 0]) <= 0.05
    assert loads.max() / loads.mean() > 25 and loads.min() / loads.mean() < 0.15
