"""Pins of the oracle's load-balance rows: the bias update rule and the f_i,
P_i routing statistics."""
import numpy as np
import pytest

from oracle import moe_oracle as mo


def test_bias_update_directions_and_size():
    b = np.array([0.1, -0.05, 0.0, 0.02], np.float32)
    counts = np.array([10, 2, 4, 8])          # mean 6
    out = mo.bias_update(b, counts, 0.001)
    assert out.dtype == np.float32
    assert out[0] == np.float32(np.float32(0.1) - np.float32(0.001))    # overloaded: down
    assert out[3] == np.float32(np.float32(0.02) - np.float32(0.001))
    assert out[1] == np.float32(np.float32(-0.05) + np.float32(0.001))  # underloaded: up
    assert out[2] == np.float32(np.float32(0.0) + np.float32(0.001))


def test_bias_update_balanced_and_zero_rate():
    b = np.linspace(-0.1, 0.1, 8).astype(np.float32)
    assert np.array_equal(mo.bias_update(b, np.full(8, 5), 0.001), b)   # every load at the mean
    assert np.array_equal(mo.bias_update(b, np.arange(8), 0.0), b)      # gamma = 0 later in training


def test_bias_update_steers_selection_toward_balance():
    # Repeated updates with the loads of the oracle's own routing lower the
    # maximum load of a skewed router (sigmoid gating, bias in the key only).
    rng = np.random.default_rng(0)
    T, N, K = 2000, 16, 2
    logits = rng.normal(size=(T, N)) + np.linspace(1.0, -1.0, N)   # skewed towards low indices
    s = mo.affinity(logits, "sigmoid")
    b = np.zeros(N, np.float32)
    idx, _, _ = mo.select_experts(s, b, K)
    first = np.bincount(idx.reshape(-1), minlength=N).max()
    for _ in range(300):
        idx, _, _ = mo.select_experts(s, b, K)
        b = mo.bias_update(b, np.bincount(idx.reshape(-1), minlength=N), 0.01)
    last = np.bincount(idx.reshape(-1), minlength=N).max()
    assert last < 0.6 * first
    # the weights still come from the unbiased affinities
    g = mo.gate_weights(s, idx, True, 1.0)
    np.testing.assert_allclose(g.sum(1), 1.0, atol=1e-12)


def test_balance_stats_closed_forms():
    rng = np.random.default_rng(1)
    T, N, K, L = 48, 8, 3, 12
    s = mo.affinity(rng.normal(size=(T, N)), "softmax")
    idx, _, _ = mo.select_experts(s, None, K)
    f, P = mo.balance_stats(s, idx, L)
    assert f.shape == (T // L, N)
    np.testing.assert_allclose(f.sum(1), K)               # each token picks K experts
    np.testing.assert_allclose(P.sum(1), 1.0, atol=1e-12)  # softmax rows sum to 1
    # literal counting for one sequence
    q = 2
    want_f = [sum(1 for t in range(q * L, (q + 1) * L) if e in idx[t]) / L for e in range(N)]
    np.testing.assert_allclose(f[q], want_f)
    np.testing.assert_allclose(P[q], [np.mean([s[t, e] for t in range(q * L, (q + 1) * L)])
                                      for e in range(N)], rtol=1e-13)
    # the batch statistics are the means of the per-sequence ones
    fb, Pb = mo.balance_stats(s, idx, T)
    np.testing.assert_allclose(fb[0], f.mean(0))
    np.testing.assert_allclose(Pb[0], P.mean(0), rtol=1e-13)
    # uniform affinities and a round-robin selection give f_i = K/N, P_i = 1/N
    su = np.full((T, N), 1.0 / N)
    iu = np.array([[(t * K + k) % N for k in range(K)] for t in range(T)])
    fu, Pu = mo.balance_stats(su, iu, T)
    np.testing.assert_allclose(fu[0], K / N)
    np.testing.assert_allclose(Pu[0], 1.0 / N)
    with pytest.raises(ValueError):
        mo.balance_stats(s, idx, 7)
