"""GPU parity of the model-native entry points (operand prologue fused into the kernels) against the
float64 oracle (prologue + recurrence), through the C ABI.

Bar: 5e-3 of max|oracle| (bf16 inputs and y, float32 state), as for the other bf16 entry points.
"""

import numpy as np
import pytest
import torch

import oracle
import rwkv_delta_rule_b200 as rk
import wkv7_inputs as wi
from helpers import TOL_BF16, need_cuda, rel_err

pytestmark = pytest.mark.gpu

NATIVE = ("r", "xw", "k", "v", "xa")


@pytest.fixture(autouse=True)
def _cuda():
    need_cuda()
    rk.load_library()
    yield
    assert rk.rwkv7_get_last_error() == 0


def _oracle(d, k_k, s0):
    return oracle.wkv7_model_native(*[d[n + "_f32"] for n in ("r", "xw", "k", "v", "xa")], k_k, s0)


PATHS = [pytest.param(rk.RWKV7_PATH_SCAN, id="scan"), pytest.param(rk.RWKV7_PATH_CHUNK, id="chunk")]


@pytest.mark.parametrize("path", PATHS)
@pytest.mark.parametrize("T", [1, 33, 64, 65, 127, 128, 129, 257])
def test_prefill_model_native(T, path):
    d = wi.draw_model_native(2, T, 3, seed=300 + T, s0_std=0.1)
    yo, so = _oracle(d, d["k_k"], d["s0"])
    dev = {n: d[n].cuda() for n in NATIVE}
    y, s = rk.prefill_model_native(*[dev[n] for n in NATIVE], d["k_k"].cuda(), d["s0"].cuda(), path=path)
    torch.cuda.synchronize()
    assert rel_err(y, yo) <= TOL_BF16
    assert rel_err(s, so) <= TOL_BF16


@pytest.mark.parametrize("path", PATHS)
def test_prefill_model_native_without_key_scale_and_state(path):
    d = wi.draw_model_native(1, 192, 2, seed=401)
    yo, so = _oracle(d, None, None)
    dev = {n: d[n].cuda() for n in NATIVE}
    y, s = rk.prefill_model_native(*[dev[n] for n in NATIVE], None, None, path=path)
    torch.cuda.synchronize()
    assert rel_err(y, yo) <= TOL_BF16
    assert rel_err(s, so) <= TOL_BF16


@pytest.mark.parametrize("sched", [rk.RWKV7_SCHED_PAIR, rk.RWKV7_SCHED_TASKS, rk.RWKV7_SCHED_PIPE],
                         ids=["pair", "tasks", "pipe"])
@pytest.mark.parametrize("T", [64, 65, 200, 1000])
def test_prefill_model_native_every_schedule(T, sched):
    """Every chunked schedule with model-native inputs, across one chunk, ragged tails and many chunks
    (the decays and learning rates are formed ahead of the chunk that uses them)."""
    d = wi.draw_model_native(2, T, 3, seed=420 + T, s0_std=0.1)
    yo, so = _oracle(d, d["k_k"], d["s0"])
    dev = {n: d[n].cuda() for n in NATIVE}
    y, s = rk.prefill_ext(dev["r"], dev["xw"], dev["k"], dev["v"], dev["xa"], None, d["s0"].cuda(),
                          path=rk.RWKV7_PATH_CHUNK, model_native=True, k_k=d["k_k"].cuda(), schedule=sched)
    torch.cuda.synchronize()
    assert rel_err(y, yo) <= TOL_BF16
    assert rel_err(s, so) <= TOL_BF16


@pytest.mark.parametrize("z_mean", [-3.0, 3.0])
def test_prefill_model_native_decay_regimes(z_mean):
    d = wi.draw_model_native(2, 320, 2, seed=410, z_mean=z_mean, s0_std=0.1)
    yo, so = _oracle(d, d["k_k"], d["s0"])
    dev = {n: d[n].cuda() for n in NATIVE}
    y, s = rk.prefill_model_native(*[dev[n] for n in NATIVE], d["k_k"].cuda(), d["s0"].cuda())
    torch.cuda.synchronize()
    assert rel_err(y, yo) <= TOL_BF16
    assert rel_err(s, so) <= TOL_BF16


def test_zero_keys_are_finite():
    # k = 0 on some tokens: kk = 0 there (the normalisation's 1e-12 floor), so a = b = 0
    d = wi.draw_model_native(1, 130, 2, seed=420, s0_std=0.1)
    d["k"][:, 5:9] = 0
    d["k_f32"] = d["k"].float()
    yo, so = _oracle(d, d["k_k"], d["s0"])
    dev = {n: d[n].cuda() for n in NATIVE}
    for path in (rk.RWKV7_PATH_SCAN, rk.RWKV7_PATH_CHUNK):
        y, s = rk.prefill_model_native(*[dev[n] for n in NATIVE], d["k_k"].cuda(), d["s0"].cuda(), path=path)
        torch.cuda.synchronize()
        assert torch.isfinite(y.float()).all() and torch.isfinite(s).all()
        assert rel_err(y, yo) <= TOL_BF16
        assert rel_err(s, so) <= TOL_BF16


def test_decode_model_native_steps_equal_oracle():
    T = 24
    d = wi.draw_model_native(3, T, 4, seed=430, s0_std=0.1)
    yo, so = _oracle(d, d["k_k"], d["s0"])
    dev = {n: d[n].cuda() for n in NATIVE}
    state = d["s0"].cuda().clone()
    kk = d["k_k"].cuda()
    ys = []
    for t in range(T):
        ys.append(rk.decode_model_native_(*[dev[n][:, t].contiguous() for n in NATIVE], kk, state))
    torch.cuda.synchronize()
    y = torch.stack(ys, dim=1)
    assert rel_err(y, yo) <= TOL_BF16
    assert rel_err(state, so) <= TOL_BF16


def test_decode_model_native_rejects_bad_shapes():
    d = wi.draw_model_native(2, 1, 2, seed=440)
    dev = {n: d[n][:, 0].cuda() for n in NATIVE}
    state = torch.zeros((2, 2, 64, 64), device="cuda")
    with pytest.raises(ValueError):
        rk.decode_model_native_(*[dev[n] for n in NATIVE], torch.ones((3, 64), device="cuda"), state)
