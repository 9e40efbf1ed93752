"""GPU parity of the reduced-precision decode (state stored as bfloat16) against the bfloat16-state
oracle (``oracle.decode_step_bf16_state``: the float64 step, rounded to nearest even), through the
C ABI.

Bars, from the arithmetic: the GPU computes the step in float32 and rounds; the oracle computes it in
float64 and rounds.  The two pre-rounding values differ by the float32 evaluation error of
S w + (S a) b + v k, at most about 64 * 2^-24 of the terms' magnitudes M = |S||w| + (|S||a|) |b| + |v||k|
(the 64-term dot product dominates); they round to the same bfloat16 value unless that error reaches
a rounding boundary.  So after one step every element is within one bfloat16 ulp (2^-7 of the
element) plus 2^-18 M of the oracle, and elements that differ at all are rare.  y is a bf16 output of
float32 arithmetic: the usual 5e-3 of max|y|.  Over several steps a one-ulp difference is carried
forward (the state update is a contraction for these inputs), so multi-step runs are held to 2^-7 of
max|state| against the oracle's own bfloat16-state trajectory.
"""

import numpy as np
import pytest
import torch

import oracle
import rwkv_delta_rule_b200 as rk
import wkv7_inputs as wi
from helpers import OPS, TOL_BF16, need_cuda, rel_err

pytestmark = pytest.mark.gpu


@pytest.fixture(autouse=True)
def _cuda():
    need_cuda()
    rk.load_library()
    yield
    assert rk.rwkv7_get_last_error() == 0


def _bf16_state(s0):
    return s0.to(torch.bfloat16)


def test_one_step_rounds_like_the_oracle():
    B, H = 64, 16
    d = wi.draw(B, 1, H, seed=900, s0_std=0.1)
    s = _bf16_state(d["s0"])
    ops = [d[n + "_f32"][:, 0] for n in OPS]
    yo, so = oracle.decode_step_bf16_state(*ops, s.to(torch.float64))
    st = s.cuda().clone()
    y = torch.empty((B, H, 64), dtype=torch.bfloat16, device="cuda")
    rk.rwkv7_wkv_decode_bf16_bf16state(*[d[n][:, 0].contiguous().cuda() for n in OPS], st, y)
    torch.cuda.synchronize()
    got = st.cpu().to(torch.float64).numpy()
    diff = got != so
    assert diff.mean() < 1e-3, diff.mean()
    S = np.abs(s.to(torch.float64).numpy())
    w, k, v, a, b = [np.abs(d[n + "_f32"][:, 0].numpy().astype(np.float64)) for n in ("w", "k", "v", "a", "b")]
    sa = np.einsum("bhij,bhj->bhi", S, a)
    M = S * w[:, :, None, :] + sa[..., None] * b[:, :, None, :] + v[..., None] * k[:, :, None, :]
    assert np.all(np.abs(got - so) <= 2.0 ** -7 * np.abs(so) + 2.0 ** -18 * M)
    assert rel_err(y, yo) <= TOL_BF16


def test_steps_track_the_bf16_state_oracle():
    B, H, T = 4, 8, 24
    d = wi.draw(B, T, H, seed=910, s0_std=0.1)
    s_or = oracle.round_bf16(d["s0"].numpy())
    st = _bf16_state(d["s0"]).cuda()
    y = torch.empty((B, H, 64), dtype=torch.bfloat16, device="cuda")
    for t in range(T):
        ops = [d[n + "_f32"][:, t] for n in OPS]
        yo, s_or = oracle.decode_step_bf16_state(*ops, s_or)
        rk.rwkv7_wkv_decode_bf16_bf16state(*[d[n][:, t].contiguous().cuda() for n in OPS], st, y)
        torch.cuda.synchronize()
        assert rel_err(y, yo) <= TOL_BF16, t
    assert rel_err(st.to(torch.float32), s_or) <= 2.0 ** -7


def test_drift_from_the_float32_state_is_bounded():
    # the reduced-precision state against the full-precision recurrence over 256 steps: a property of
    # the method (rounding every step), recorded here with its measured size as the bound's basis
    B, H, T = 2, 4, 256
    d = wi.draw(B, T, H, seed=920, s0_std=0.1)
    yo, so = oracle.wkv7(*[d[n + "_f32"] for n in OPS], oracle.round_bf16(d["s0"].numpy()))
    st = _bf16_state(d["s0"]).cuda()
    y = torch.empty((B, H, 64), dtype=torch.bfloat16, device="cuda")
    ys = []
    for t in range(T):
        rk.rwkv7_wkv_decode_bf16_bf16state(*[d[n][:, t].contiguous().cuda() for n in OPS], st, y)
        ys.append(y.clone())
    torch.cuda.synchronize()
    err_s = rel_err(st.to(torch.float32), so)
    err_y = rel_err(torch.stack(ys, dim=1), yo)
    print(f"bf16-state drift after {T} steps: state {err_s:.2e}, y {err_y:.2e}")
    assert err_s <= 2e-2 and err_y <= 2e-2


def test_rejects_a_float32_state():
    d = wi.draw(1, 1, 2, seed=930)
    with pytest.raises(ValueError):
        rk.rwkv7_wkv_decode_bf16_bf16state(*[d[n][:, 0].contiguous().cuda() for n in OPS],
                                           torch.zeros((1, 2, 64, 64), device="cuda"),
                                           torch.empty((1, 2, 64), dtype=torch.bfloat16, device="cuda"))
