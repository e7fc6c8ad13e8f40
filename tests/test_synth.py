"""The seeded input generator: determinism, block regeneration, distributions,
and (on a GPU) bit-identity of the host and device implementations."""
import numpy as np
import pytest

import synth
from synth import recipes


def test_host_fill_is_deterministic_and_blockwise():
    a = synth.host_normal(10000, 0.02, 0, synth.TID_WGU)
    b = synth.host_normal(10000, 0.02, 0, synth.TID_WGU)
    np.testing.assert_array_equal(a, b)
    # any block regenerates on its own
    c = synth.host_normal(300, 0.02, 0, synth.TID_WGU, offset=4321)
    np.testing.assert_array_equal(c, a[4321:4621])
    # different tensor ids and seeds give different streams
    assert not np.array_equal(a, synth.host_normal(10000, 0.02, 0, synth.TID_WD))
    assert not np.array_equal(a, synth.host_normal(10000, 0.02, 1, synth.TID_WGU))


def test_threads_do_not_change_values():
    L = synth.lib()
    n = 1 << 18
    one = np.empty(n, np.float32)
    many = np.empty(n, np.float32)
    sc = synth.normal_scale(1.0)
    L.syn_host_normal_f32(one.ctypes.data, n, 3, 0, 0, sc, 1)
    L.syn_host_normal_f32(many.ctypes.data, n, 3, 0, 0, sc, 7)
    np.testing.assert_array_equal(one, many)


def test_normal_moments_and_range():
    v = synth.host_normal(1 << 20, 1.0, 0, synth.TID_X).astype(np.float64)
    assert abs(v.mean()) < 5e-3
    assert abs(v.std() - 1.0) < 5e-3
    assert np.abs(v).max() <= 2 * np.sqrt(3.0) + 1e-6       # Irwin-Hall(4) support
    # kurtosis of Irwin-Hall(4) is 3 - 6/(5*4) = 2.7
    k = np.mean(v ** 4) / np.mean(v ** 2) ** 2
    assert abs(k - 2.7) < 0.02


def test_uniform_range():
    u = synth.host_uniform(1 << 16, -0.1, 0.1, 0, synth.TID_BIAS).astype(np.float64)
    assert u.min() >= -0.1 - 1e-7 and u.max() < 0.1
    assert abs(u.mean()) < 2e-3


def test_bf16_rounding_is_nearest_even():
    import torch
    f = synth.host_normal(1 << 14, 0.02, 0, synth.TID_WGU)
    bits = synth.host_normal(1 << 14, 0.02, 0, synth.TID_WGU, bf16=True)
    want = torch.from_numpy(f).to(torch.bfloat16).view(torch.int16).numpy().view(np.uint16)
    np.testing.assert_array_equal(bits, want)


def test_recipes_shapes():
    c = recipes.CONFIGS["v3_bf16"]
    assert (c.T, c.d, c.n_shared, c.n_routed, c.top_k, c.inter) == (16384, 7168, 1, 256, 8, 2048)
    assert c.expert_gemm_flops() == pytest.approx(12.99e12, rel=1e-3)
    small = recipes.small_variant(c, T=256, d=512, inter=256)
    wg, wu, wd = recipes.host_expert(small, 3)
    assert wg.shape == (256, 512) and wd.shape == (512, 256)


@pytest.mark.gpu
def test_device_matches_host_bit_for_bit():
    import torch
    n = (1 << 20) + 7
    for bf in (False, True):
        t = torch.empty(n, dtype=torch.bfloat16 if bf else torch.float32, device="cuda")
        synth.dev_fill_normal(t, 0.02, 0, synth.TID_WGU, offset=12345)
        h = synth.host_normal(n, 0.02, 0, synth.TID_WGU, offset=12345, bf16=bf)
        got = t.view(torch.int16).cpu().numpy().view(np.uint16) if bf else t.cpu().numpy()
        np.testing.assert_array_equal(got, h)
    u = torch.empty(1000, dtype=torch.float32, device="cuda")
    synth.dev_fill_uniform(u, -0.1, 0.1, 0, synth.TID_BIAS)
    np.testing.assert_array_equal(u.cpu().numpy(), synth.host_uniform(1000, -0.1, 0.1, 0,
                                                                      synth.TID_BIAS))


@pytest.mark.gpu
def test_device_recipe_matches_host_recipe():
    import torch
    for name in ("tiny_f32", "dsmoe16b_bf16"):
        cfg = recipes.CONFIGS[name]
        if name == "dsmoe16b_bf16":
            cfg = recipes.small_variant(cfg, T=256, d=256, inter=128, n_routed=8)
        dev = recipes.device_inputs(cfg)
        np.testing.assert_array_equal(dev["x"].double().cpu().numpy(), recipes.host_x(cfg))
        np.testing.assert_array_equal(dev["w_r"].double().cpu().numpy(), recipes.host_router(cfg))
        for e in (0, cfg.n_experts - 1):
            wg, wu, wd = recipes.host_expert(cfg, e)
            gu = dev["w_gu"][e].double().cpu().numpy()
            np.testing.assert_array_equal(gu[:cfg.inter], wg)
            np.testing.assert_array_equal(gu[cfg.inter:], wu)
            np.testing.assert_array_equal(dev["w_down"][e].double().cpu().numpy(), wd)
