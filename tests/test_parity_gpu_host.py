"""GPU parity of the host-buffer prefill (``rwkv7_wkv_prefill_host_bf16``: operands and results in
host memory, staged through device buffers batch slice by batch slice with the copies of one slice
overlapping the compute of another) against the float64 oracle and against the device entry point,
through the C ABI.  Bars as for the device call: 5e-3 of max|oracle| for bf16 operands; the scan
path, whose rows are independent, must match the device call bit for bit."""

import pytest
import torch

import oracle
import rwkv_delta_rule_b200 as rk
import wkv7_inputs as wi
from helpers import OPS, TOL_BF16, need_cuda, oracle_ops, rel_err, to_dev

pytestmark = pytest.mark.gpu


@pytest.fixture(autouse=True)
def _cuda():
    need_cuda()
    rk.load_library()
    yield
    assert rk.rwkv7_get_last_error() == 0


def _host_call(d, path, with_s0=True, slices=0, pinned=True):
    B, T, H, N = d["r"].shape
    pin = (lambda t: t.pin_memory()) if pinned else (lambda t: t.clone())
    host = {n: pin(d[n].contiguous()) for n in OPS}
    s_in = pin(d["s0"]) if with_s0 else None
    y = pin(torch.empty((B, T, H, N), dtype=torch.bfloat16))
    s_out = pin(torch.empty((B, H, N, N)))
    dev = {n: torch.empty((B, T, H, N), dtype=torch.bfloat16, device="cuda") for n in OPS + ("y",)}
    dev["s_in"] = torch.empty((B, H, N, N), device="cuda")
    dev["s_out"] = torch.empty((B, H, N, N), device="cuda")
    rk.rwkv7_wkv_prefill_host_bf16(path, *[host[n] for n in OPS], s_in, y, s_out, dev, slices=slices)
    torch.cuda.synchronize()
    return y, s_out


def _device_call(d, path, with_s0=True):
    dv = to_dev(d)
    y, s = rk.prefill(*[dv[n] for n in OPS], dv["s0"] if with_s0 else None, path=path)
    torch.cuda.synchronize()
    return y.cpu(), s.cpu()


@pytest.mark.parametrize("path", [rk.RWKV7_PATH_CHUNK, rk.RWKV7_PATH_SCAN])
@pytest.mark.parametrize("slices", [0, 1, 2, 5])
def test_host_prefill_matches_oracle_and_device_call(path, slices):
    d = wi.draw(5, 200, 3, seed=960 + slices, s0_std=0.1)
    yo, so = oracle.wkv7(*oracle_ops(d), d["s0"])
    y, s = _host_call(d, path, slices=slices)
    assert rel_err(y, yo) <= TOL_BF16
    assert rel_err(s, so) <= TOL_BF16
    yd, sd = _device_call(d, path)
    if path == rk.RWKV7_PATH_SCAN:
        assert torch.equal(y, yd) and torch.equal(s, sd)
    else:
        assert rel_err(y, yd.float().numpy()) <= 1e-2 and rel_err(s, sd.numpy()) <= 1e-2


def test_host_prefill_zero_state_and_pageable_buffers():
    d = wi.draw(3, 130, 2, seed=970)
    yo, so = oracle.wkv7(*oracle_ops(d), None)
    y, s = _host_call(d, rk.RWKV7_PATH_AUTO, with_s0=False, slices=3, pinned=False)
    assert rel_err(y, yo) <= TOL_BF16
    assert rel_err(s, so) <= TOL_BF16


def test_host_prefill_empty_sequence_copies_the_state():
    d = wi.draw(2, 1, 2, seed=975, s0_std=0.1)
    e = {n: d[n][:, :0].contiguous() for n in OPS}
    e["s0"] = d["s0"]
    y, s = _host_call(e, rk.RWKV7_PATH_AUTO, slices=2)
    assert torch.equal(s, d["s0"])
    assert y.numel() == 0


@pytest.mark.slow
def test_host_prefill_at_the_d768_shape_equals_the_device_call():
    # the bench's end-to-end call (B8 T4096 H12, default slices): the same kernels on batch slices,
    # so every element equals the device-buffer call's (a pair's arithmetic does not depend on the
    # other pairs of its launch), and sampled pairs match the oracle
    case = wi.CASES["prefill_d768_b8_t4096"]
    d = wi.draw_case(case)
    y, s = _host_call(d, rk.RWKV7_PATH_AUTO)
    yd, sd = _device_call(d, rk.RWKV7_PATH_AUTO)
    assert torch.equal(y, yd) and torch.equal(s, sd)
    for b, h in ((0, 0), (7, 11)):
        sub = [x[b:b + 1, :, h:h + 1] for x in oracle_ops(d)]
        yo, so = oracle.wkv7(*sub, d["s0"][b:b + 1, h:h + 1])
        assert rel_err(y[b:b + 1, :, h:h + 1], yo) <= TOL_BF16
        assert rel_err(s[b:b + 1, h:h + 1], so) <= TOL_BF16
