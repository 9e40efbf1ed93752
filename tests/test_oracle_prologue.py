"""Pins of the oracle's model-native operand prologue (RWKV-7 G0 7.2B walkthrough,
lshu.cn/news/198401, section 7.1), each against something other than its own formula."""

import numpy as np
import pytest
import torch

import oracle
import wkv7_inputs as wi


def _rng(seed):
    return np.random.default_rng(seed)


def test_decay_matches_the_printed_generator_constant():
    # The pages give the decay as exp(-exp(-softplus(-x) - 0.5)); the configs print it as
    # exp(-0.606531 * sigmoid(z)).  The two agree up to the six printed digits of e^-0.5.
    z = _rng(1).normal(0.0, 2.0, size=(4, 64))
    w, _, _ = oracle.x070_prologue(z, np.ones_like(z), np.zeros_like(z), None)
    w_cfg = np.exp(-wi.DECAY_SCALE / (1.0 + np.exp(-z)))
    assert np.max(np.abs(w / w_cfg - 1.0)) < 2e-6


def test_decay_range_and_limits():
    # softly clamped pre-activation (-inf, -0.5]: decay in (exp(-e^-0.5), 1), monotone decreasing in x
    x = np.linspace(-40.0, 40.0, 2001)[None, :].repeat(1, 0)
    w, _, _ = oracle.x070_prologue(x, np.ones((1, 2001)), np.zeros((1, 2001)), None)
    lo = np.exp(-np.exp(-0.5))
    assert np.all(w >= lo) and np.all(w <= 1.0)
    mid = np.abs(x[0]) <= 20.0
    assert np.all(w[0, mid] > lo) and np.all(w[0, mid] < 1.0)
    assert np.all(np.diff(w[0]) <= 0)
    assert abs(w[0, 0] - 1.0) < 1e-15 and abs(w[0, -1] - lo) < 1e-15


def test_kk_is_the_unit_key_and_scale_free():
    g = _rng(2)
    k = g.normal(size=(3, 5, 64))
    kk_w = g.uniform(0.5, 1.5, size=(5, 64))
    _, a, b = oracle.x070_prologue(np.zeros_like(k), k, np.zeros_like(k), kk_w)
    assert np.max(np.abs(np.linalg.norm(a, axis=-1) - 1.0)) < 1e-14
    # sigmoid(0) = 1/2 on every channel: b = -a / 2
    assert np.max(np.abs(b + 0.5 * a)) < 1e-15
    # a positive common factor on k_k does not change kk
    _, a2, _ = oracle.x070_prologue(np.zeros_like(k), k, np.zeros_like(k), 3.7 * kk_w)
    assert np.max(np.abs(a2 - a)) < 1e-14
    # with k_k = 1 a unit key is returned as it is (a = -k)
    ku = k / np.linalg.norm(k, axis=-1, keepdims=True)
    _, a3, _ = oracle.x070_prologue(np.zeros_like(k), ku, np.zeros_like(k), None)
    assert np.max(np.abs(a3 + ku)) < 1e-15


def test_zero_key_gives_zero_operands():
    k = np.zeros((2, 64))
    _, a, b = oracle.x070_prologue(np.zeros_like(k), k, np.ones_like(k), None)
    assert np.all(a == 0.0) and np.all(b == 0.0)


def test_model_native_equals_the_recurrence_on_the_generator_operands():
    # Build inputs for which the prologue must reproduce the configs' operands exactly:
    # k = unit kh, k_k = 1, xw = z, xa = logit(alpha)  ->  w = exp(-e^-0.5 sigmoid(z)), a = -kh,
    # b = kh * alpha.  The fused oracle then equals the plain one up to the printed 0.606531.
    g = _rng(3)
    shp = (2, 40, 3, 64)
    r, v = g.normal(size=shp), g.normal(size=shp)
    kh = g.normal(size=shp)
    kh /= np.linalg.norm(kh, axis=-1, keepdims=True)
    z = g.normal(size=shp)
    alpha = g.uniform(0.05, 0.95, size=shp)
    s0 = g.normal(0.0, 0.1, size=(2, 3, 64, 64))
    y1, s1 = oracle.wkv7_model_native(r, z, kh, v, np.log(alpha / (1.0 - alpha)), None, s0)
    w = np.exp(-wi.DECAY_SCALE / (1.0 + np.exp(-z)))
    y2, s2 = oracle.wkv7(r, w, kh, v, -kh, kh * alpha, s0)
    assert np.max(np.abs(y1 - y2)) / np.max(np.abs(y2)) < 2e-5
    assert np.max(np.abs(s1 - s2)) / np.max(np.abs(s2)) < 2e-5


def test_generator_draw_model_native_shapes():
    d = wi.draw_model_native(2, 3, 4, seed=9, s0_std=0.1)
    for nm in ("r", "xw", "k", "v", "xa"):
        assert d[nm].shape == (2, 3, 4, 64) and d[nm].dtype == torch.bfloat16
    assert d["k_k"].shape == (4, 64) and d["k_k"].dtype == torch.float32
    assert d["s0"].shape == (2, 4, 64, 64)
