"""Pins of the oracle's GroupNorm epilogue (the x070 ln_x: RWKV-7 G0 7.2B walkthrough,
lshu.cn/news/198401, section 7.1) against the library routine and the properties it must have."""

import numpy as np
import torch

import oracle


def test_matches_torch_group_norm_in_float64():
    g = np.random.default_rng(11)
    T, H, N = 37, 5, 64
    y = g.normal(0.0, 3.0, size=(T, H, N))
    w = g.uniform(0.5, 1.5, size=(H, N))
    b = g.normal(size=(H, N))
    got = oracle.group_norm_heads(y, w, b)
    ref = torch.nn.functional.group_norm(torch.from_numpy(y.reshape(T, H * N)), H,
                                         torch.from_numpy(w.reshape(-1)), torch.from_numpy(b.reshape(-1)),
                                         eps=64e-5).numpy().reshape(T, H, N)
    assert np.max(np.abs(got - ref)) < 1e-12


def test_unit_weight_gives_zero_mean_and_the_eps_shrunk_unit_variance():
    g = np.random.default_rng(12)
    y = g.normal(2.0, 0.7, size=(9, 3, 64))
    out = oracle.group_norm_heads(y)
    assert np.max(np.abs(out.mean(axis=-1))) < 1e-13
    var = ((y - y.mean(axis=-1, keepdims=True)) ** 2).mean(axis=-1)
    assert np.max(np.abs((out ** 2).mean(axis=-1) - var / (var + oracle.LN_EPS))) < 1e-12


def test_constant_rows_map_to_the_bias_and_scale_invariance():
    y = np.full((2, 4, 64), 3.25)
    b = np.arange(4 * 64, dtype=np.float64).reshape(4, 64) * 0.01
    assert np.max(np.abs(oracle.group_norm_heads(y, None, b) - b)) < 1e-15
    g = np.random.default_rng(13)
    z = g.normal(size=(6, 2, 64)) * 50.0  # var >> eps: scaling y leaves the output (almost) unchanged
    assert np.max(np.abs(oracle.group_norm_heads(z) - oracle.group_norm_heads(4.0 * z + 1.0))) < 1e-6
