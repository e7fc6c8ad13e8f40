"""CPU tests of the routing comparison used by the GPU parity tests: the
selected set is compared exactly outside near-ties, and the order of two
picks whose keys lie within the tie bound may go either way, while every
other swap still fails."""
import numpy as np
import pytest

from oracle import moe_oracle as mo

from gpu_layer import check_routing


class Cfg:
    T, n_routed, renorm, route_scale = 3, 6, False, 1.0


def make_ref():
    key = np.array([
        [0.90, 0.80, 0.70, 0.10, 0.05, 0.01],
        [0.50, 0.50 + 2e-8, 0.20, 0.10, 0.05, 0.01],   # experts 0 and 1 tie within the bound
        [0.10, 0.20, 0.30, 0.40, 0.95, 0.60],
    ])
    idx = np.argsort(-key, axis=1, kind="stable")[:, :3]
    return {"key": key, "s": key.copy(), "idx": idx,
            "kgap": np.full(3, 0.05), "ggap": np.full(3, 1.0)}


def counts_of(idx):
    return np.bincount(idx.reshape(-1), minlength=Cfg.n_routed)


def weights_of(ref, idx):
    return mo.gate_weights(ref["s"], idx, False, 1.0)


def test_exact_selection_passes():
    ref = make_ref()
    g = ref["idx"].copy()
    check_routing(Cfg, ref, g, weights_of(ref, g), counts_of(g))


def test_equal_keys_may_swap():
    ref = make_ref()
    g = ref["idx"].copy()
    assert list(g[1, :2]) == [1, 0]
    g[1, :2] = [0, 1]          # lower index first, as fp32 equal keys would give
    check_routing(Cfg, ref, g, weights_of(ref, g), counts_of(g))


def test_distinct_keys_may_not_swap():
    ref = make_ref()
    g = ref["idx"].copy()
    g[0, :2] = g[0, 1::-1]     # 0.90 and 0.80 swapped
    with pytest.raises(AssertionError):
        check_routing(Cfg, ref, g, weights_of(ref, g), counts_of(g))


def test_other_set_fails_even_with_a_tie():
    ref = make_ref()
    g = ref["idx"].copy()
    g[1, 2] = 3                # a different third expert
    with pytest.raises(AssertionError):
        check_routing(Cfg, ref, g, weights_of(ref, g), counts_of(g))
