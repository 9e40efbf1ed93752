"""GPU parity of the fused ln_x GroupNorm epilogue (one group per head, eps 64e-5) against the float64
oracle (recurrence, then ``oracle.group_norm_heads``), through the C ABI's option entry points.

The normalised output is O(1) per token, so the bf16 bar (5e-3 of max|oracle|) covers the output's
own bf16 rounding (2^-9 of an element) plus the recurrence's float32 / tensor-core error divided by
each token's channel standard deviation.  The state is not touched by the epilogue: it must be
bit-identical to the run without it.
"""

import numpy as np
import pytest
import torch

import oracle
import rwkv_delta_rule_b200 as rk
import wkv7_inputs as wi
from helpers import OPS, TOL_BF16, need_cuda, oracle_ops, rel_err, to_dev

pytestmark = pytest.mark.gpu

NATIVE = ("r", "xw", "k", "v", "xa")
PATHS = [pytest.param(rk.RWKV7_PATH_SCAN, id="scan"), pytest.param(rk.RWKV7_PATH_CHUNK, id="chunk")]


@pytest.fixture(autouse=True)
def _cuda():
    need_cuda()
    rk.load_library()
    yield
    assert rk.rwkv7_get_last_error() == 0


def _ln(H, seed):
    p = wi.draw_group_norm(H, seed=seed)
    return p["ln_w"], p["ln_b"]


@pytest.mark.parametrize("path", PATHS)
@pytest.mark.parametrize("T", [1, 31, 64, 65, 129, 257])
def test_prefill_group_norm(T, path):
    d = wi.draw(2, T, 3, seed=500 + T, s0_std=0.1)
    ln_w, ln_b = _ln(3, 501 + T)
    yo, so = oracle.wkv7(*oracle_ops(d), d["s0"])
    zo = oracle.group_norm_heads(yo, ln_w, ln_b)
    dv = to_dev(d)
    y, s = rk.prefill_ext(*[dv[n] for n in OPS], dv["s0"], path=path, group_norm=True, ln_w=ln_w.cuda(),
                          ln_b=ln_b.cuda())
    torch.cuda.synchronize()
    assert rel_err(y, zo) <= TOL_BF16
    assert rel_err(s, so) <= TOL_BF16


@pytest.mark.parametrize("path", PATHS)
def test_prefill_group_norm_default_affine(path):
    d = wi.draw(1, 200, 2, seed=520)
    yo, so = oracle.wkv7(*oracle_ops(d), None)
    zo = oracle.group_norm_heads(yo)
    dv = to_dev(d)
    y, s = rk.prefill_ext(*[dv[n] for n in OPS], None, path=path, group_norm=True)
    torch.cuda.synchronize()
    assert rel_err(y, zo) <= TOL_BF16
    assert rel_err(s, so) <= TOL_BF16


@pytest.mark.parametrize("path", PATHS)
def test_prefill_group_norm_with_model_native_inputs(path):
    d = wi.draw_model_native(2, 190, 3, seed=530, s0_std=0.1)
    ln_w, ln_b = _ln(3, 531)
    yo, so = oracle.wkv7_model_native(*[d[n + "_f32"] for n in NATIVE], d["k_k"], d["s0"])
    zo = oracle.group_norm_heads(yo, ln_w, ln_b)
    dev = {n: d[n].cuda() for n in NATIVE}
    y, s = rk.prefill_ext(dev["r"], dev["xw"], dev["k"], dev["v"], dev["xa"], None, d["s0"].cuda(), path=path,
                          model_native=True, k_k=d["k_k"].cuda(), group_norm=True, ln_w=ln_w.cuda(),
                          ln_b=ln_b.cuda())
    torch.cuda.synchronize()
    assert rel_err(y, zo) <= TOL_BF16
    assert rel_err(s, so) <= TOL_BF16


@pytest.mark.parametrize("path", PATHS + [pytest.param(rk.RWKV7_PATH_AUTO, id="auto")])
def test_state_unchanged_by_group_norm(path):
    d = wi.draw(2, 321, 2, seed=540, s0_std=0.1)
    ln_w, ln_b = _ln(2, 541)
    dv = to_dev(d)
    y0, s0 = rk.prefill_ext(*[dv[n] for n in OPS], dv["s0"], path=path)
    y1, s1 = rk.prefill_ext(*[dv[n] for n in OPS], dv["s0"], path=path, group_norm=True, ln_w=ln_w.cuda(),
                            ln_b=ln_b.cuda())
    torch.cuda.synchronize()
    assert torch.equal(s0, s1)
    # the un-normalised output of the option entry point is the plain entry point's, bit for bit
    yp, sp = rk.prefill(*[dv[n] for n in OPS], dv["s0"], path=path)
    torch.cuda.synchronize()
    assert torch.equal(y0, yp) and torch.equal(s0, sp)


@pytest.mark.parametrize("path", PATHS)
def test_zero_output_normalises_to_bias(path):
    # v = 0 and a zero state keep y = 0 everywhere; (0 - 0) / sqrt(0 + eps) * w + b = b exactly
    d = wi.draw(1, 130, 2, seed=550)
    ln_w, ln_b = _ln(2, 551)
    dv = to_dev(d)
    dv["v"] = torch.zeros_like(dv["v"])
    y, s = rk.prefill_ext(*[dv[n] for n in OPS], None, path=path, group_norm=True, ln_w=ln_w.cuda(),
                          ln_b=ln_b.cuda())
    torch.cuda.synchronize()
    expect = ln_b.to(torch.bfloat16).expand(1, 130, 2, 64)
    assert torch.equal(y.cpu(), expect)
    assert torch.count_nonzero(s) == 0


@pytest.mark.parametrize("native", [False, True], ids=["plain", "native"])
def test_decode_group_norm_steps_equal_oracle(native):
    T, B, H = 20, 3, 4
    ln_w, ln_b = _ln(H, 561)
    if native:
        d = wi.draw_model_native(B, T, H, seed=560, s0_std=0.1)
        yo, so = oracle.wkv7_model_native(*[d[n + "_f32"] for n in NATIVE], d["k_k"], d["s0"])
        names = ("r", "xw", "k", "v", "xa")
        kk = d["k_k"].cuda()
    else:
        d = wi.draw(B, T, H, seed=560, s0_std=0.1)
        yo, so = oracle.wkv7(*oracle_ops(d), d["s0"])
        names = OPS
        kk = None
    zo = oracle.group_norm_heads(yo, ln_w, ln_b)
    dev = {n: d[n].cuda() for n in names}
    state = d["s0"].cuda().clone()
    lw, lb = ln_w.cuda(), ln_b.cuda()
    ys = []
    for t in range(T):
        ops = [dev[n][:, t].contiguous() for n in names]
        if native:
            ops.append(None)
        ys.append(rk.decode_ext_(*ops, state, model_native=native, k_k=kk, group_norm=True, ln_w=lw, ln_b=lb))
    torch.cuda.synchronize()
    y = torch.stack(ys, dim=1)
    assert rel_err(y, zo) <= TOL_BF16
    assert rel_err(state, so) <= TOL_BF16


def test_group_norm_rejects_bad_parameter_shapes():
    d = wi.draw(1, 8, 2, seed=570)
    dv = to_dev(d)
    with pytest.raises(ValueError):
        rk.prefill_ext(*[dv[n] for n in OPS], None, group_norm=True, ln_w=torch.ones((3, 64), device="cuda"))
    with pytest.raises(ValueError):
        rk.prefill_ext(*[dv[n] for n in OPS], None, group_norm=True,
                       ln_b=torch.zeros((2, 64), device="cuda", dtype=torch.float64))
