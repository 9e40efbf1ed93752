"""Failure detection and output bounds on the GPU, in forms that fault and hang nothing.

* A device wait that runs out: through the library's test hook, every wait of the chunked kernel is
  bounded to a few thousand polls and one (b, h) pair's first chunk keeps its chain flag down in the
  task-parallel schedule, so the next chunk of that pair waits on a flag that nothing raises.  The
  launch must return, rwkv7_get_last_error() must report RWKV7_ERR_TIMEOUT once (and then OK), and
  the launches after it, on every flag slot, must match the float64 oracle again.  With a bound of 32
  polls, ordinary waits give up early on both schedules: the launch must still return cleanly.
* Guard bands: y and s_out sit inside larger buffers filled with a canary bit pattern.  After ragged
  batches (empty rows, rows of 1, 63, 65, 70 and 130 tokens, rows whose offsets leave [0, total_T],
  tokens that belong to no row) and dense calls with ragged tail chunks, every byte outside what the
  call may write still holds the canary, rows that are skipped keep the canary in y and s_out, an
  empty row's final state equals its initial state, and everything else matches the oracle
  (max|gpu - oracle| / max|oracle| <= 5e-3, the bf16 bar).
The ragged batch is the long-context workload's per-row-length batch in small (the 7.2B-width
configuration with T_b ~ U(1024, 16384)); the recurrence is the x070 update of the RWKV-7 G0 7.2B
walkthrough (lshu.cn/news/198401), section 7.1.
"""

import time

import numpy as np
import pytest
import torch

import oracle
import rwkv_delta_rule_b200 as rk
import wkv7_inputs as wi
from helpers import OPS, TOL_BF16, need_cuda, oracle_ops, rel_err, to_dev

pytestmark = pytest.mark.gpu

ERR_TIMEOUT = 4
N = 64
GUARD = 4096                    # guard elements on each side (a multiple of 8: keeps 16-byte alignment)
CANARY_BF16 = 0x7E5A            # bit patterns the kernels never produce from these inputs
CANARY_F32 = 0x7F7A5A5A


@pytest.fixture(autouse=True)
def _cuda():
    need_cuda()
    rk.load_library()
    assert rk.rwkv7_get_last_error() == 0
    yield
    rk.rwkv7_test_set_wait_hooks(0, -1)


# ---- a device wait that runs out -----------------------------------------------------------------

def _tasks_call(dv, y, s_out):
    rk.rwkv7_wkv_prefill_ext_bf16(rk.RWKV7_PATH_CHUNK, *[dv[n] for n in OPS], dv["s0"], y, s_out,
                                  schedule=rk.RWKV7_SCHED_TASKS)


def test_chain_wait_runs_out_reports_timeout_and_recovers():
    B, T, H = 1, 512, 4  # 4 pairs x 8 chunks: pair 0's chunks 1..7 wait on a flag that stays down
    d = wi.draw(B, T, H, seed=4242, s0_std=0.1)
    yo, so = oracle.wkv7(*oracle_ops(d), d["s0"])
    dv = to_dev(d)
    y = torch.empty(B, T, H, N, dtype=torch.bfloat16, device="cuda")
    s_out = torch.empty(B, H, N, N, device="cuda")

    rk.rwkv7_test_set_wait_hooks(1 << 12, 0)
    t0 = time.monotonic()
    try:
        _tasks_call(dv, y, s_out)
        torch.cuda.synchronize()
        elapsed = time.monotonic() - t0
        st = rk.rwkv7_get_last_error()
    finally:
        rk.rwkv7_test_set_wait_hooks(0, -1)
    assert st == ERR_TIMEOUT, rk.rwkv7_status_string(st)
    assert "timed out" in rk.rwkv7_status_string(st)
    assert elapsed < 30.0
    assert rk.rwkv7_get_last_error() == 0  # read once, then cleared

    # the context is usable and the chain flags are clear: four launches in a row cover every slot
    for i in range(4):
        y.zero_()
        s_out.zero_()
        _tasks_call(dv, y, s_out)
        torch.cuda.synchronize()
        assert rk.rwkv7_get_last_error() == 0, i
        assert rel_err(y, yo) <= TOL_BF16, i
        assert rel_err(s_out, so) <= TOL_BF16, i


@pytest.mark.parametrize("sched", [rk.RWKV7_SCHED_PAIR, rk.RWKV7_SCHED_TASKS])
def test_waits_that_give_up_early_abort_cleanly(sched):
    """With every wait bounded to 32 polls, ordinary waits (MMA completions, tile loads) give up before
    the hardware is done: whichever wait runs out first, the CTA must abort, drain what it issued and
    return; the call reports OK or TIMEOUT, and the next launch with the production bound is exact."""
    B, T, H = 2, 640, 3
    d = wi.draw(B, T, H, seed=4244, s0_std=0.1)
    yo, so = oracle.wkv7(*oracle_ops(d), d["s0"])
    dv = to_dev(d)
    y = torch.empty(B, T, H, N, dtype=torch.bfloat16, device="cuda")
    s_out = torch.empty(B, H, N, N, device="cuda")
    rk.rwkv7_test_set_wait_hooks(32, -1)
    t0 = time.monotonic()
    try:
        rk.rwkv7_wkv_prefill_ext_bf16(rk.RWKV7_PATH_CHUNK, *[dv[n] for n in OPS], dv["s0"], y, s_out,
                                      schedule=sched)
        torch.cuda.synchronize()
        elapsed = time.monotonic() - t0
        st = rk.rwkv7_get_last_error()
    finally:
        rk.rwkv7_test_set_wait_hooks(0, -1)
    assert st in (0, ERR_TIMEOUT), rk.rwkv7_status_string(st)
    assert elapsed < 30.0
    assert rk.rwkv7_get_last_error() == 0
    rk.rwkv7_wkv_prefill_ext_bf16(rk.RWKV7_PATH_CHUNK, *[dv[n] for n in OPS], dv["s0"], y, s_out, schedule=sched)
    torch.cuda.synchronize()
    assert rk.rwkv7_get_last_error() == 0
    assert rel_err(y, yo) <= TOL_BF16 and rel_err(s_out, so) <= TOL_BF16


@pytest.mark.parametrize("sched", [rk.RWKV7_SCHED_PAIR, rk.RWKV7_SCHED_TASKS])
def test_model_native_waits_that_give_up_early_abort_cleanly(sched):
    """The same with model-native inputs, where warps 0-3 hand the next chunk's rates, key norms and
    V^T to warps 4-7 through a wait of its own: it too gives up, the CTA aborts and returns, and the
    next launch is exact (against the float64 prologue and recurrence)."""
    B, T, H = 2, 640, 3
    d = wi.draw_model_native(B, T, H, seed=4245, s0_std=0.1)
    names = ("r", "xw", "k", "v", "xa")
    yo, so = oracle.wkv7_model_native(*[d[n + "_f32"] for n in names], d["k_k"], d["s0"])
    dv = {n: d[n].cuda() for n in names}
    kk, s0 = d["k_k"].cuda(), d["s0"].cuda()
    y = torch.empty(B, T, H, N, dtype=torch.bfloat16, device="cuda")
    s_out = torch.empty(B, H, N, N, device="cuda")

    def call():
        rk.rwkv7_wkv_prefill_ext_bf16(rk.RWKV7_PATH_CHUNK, dv["r"], dv["xw"], dv["k"], dv["v"], dv["xa"], None, s0,
                                      y, s_out, model_native=True, k_k=kk, schedule=sched)

    rk.rwkv7_test_set_wait_hooks(32, -1)
    t0 = time.monotonic()
    try:
        call()
        torch.cuda.synchronize()
        elapsed = time.monotonic() - t0
        st = rk.rwkv7_get_last_error()
    finally:
        rk.rwkv7_test_set_wait_hooks(0, -1)
    assert st in (0, ERR_TIMEOUT), rk.rwkv7_status_string(st)
    assert elapsed < 30.0
    assert rk.rwkv7_get_last_error() == 0
    call()
    torch.cuda.synchronize()
    assert rk.rwkv7_get_last_error() == 0
    assert rel_err(y, yo) <= TOL_BF16 and rel_err(s_out, so) <= TOL_BF16


def test_hook_defaults_leave_every_schedule_exact():
    """With the hooks at their defaults (and after being set and reset) nothing times out."""
    rk.rwkv7_test_set_wait_hooks(1 << 12, 0)
    rk.rwkv7_test_set_wait_hooks(0, -1)
    B, T, H = 2, 300, 3
    d = wi.draw(B, T, H, seed=4243, s0_std=0.1)
    yo, so = oracle.wkv7(*oracle_ops(d), d["s0"])
    dv = to_dev(d)
    for sched in (rk.RWKV7_SCHED_PAIR, rk.RWKV7_SCHED_TASKS, rk.RWKV7_SCHED_PIPE):
        y, s = rk.prefill_ext(*[dv[n] for n in OPS], dv["s0"], path=rk.RWKV7_PATH_CHUNK, schedule=sched)
        torch.cuda.synchronize()
        assert rk.rwkv7_get_last_error() == 0, sched
        assert rel_err(y, yo) <= TOL_BF16 and rel_err(s, so) <= TOL_BF16, sched


# ---- guard bands ------------------------------------------------------------------------------------

def _guarded(n, dtype):
    """A buffer of n elements with GUARD canary elements on each side: (full buffer, inner view)."""
    if dtype == torch.bfloat16:
        buf = torch.full((n + 2 * GUARD,), CANARY_BF16, dtype=torch.int16, device="cuda")
        return buf, buf[GUARD:GUARD + n].view(torch.bfloat16)
    buf = torch.full((n + 2 * GUARD,), CANARY_F32, dtype=torch.int32, device="cuda")
    return buf, buf[GUARD:GUARD + n].view(torch.float32)


def _canary(buf):
    return CANARY_BF16 if buf.dtype == torch.int16 else CANARY_F32


def _guards_intact(buf):
    c = _canary(buf)
    return bool((buf[:GUARD] == c).all()) and bool((buf[-GUARD:] == c).all())


def _is_canary(buf_slice):
    return bool((buf_slice == _canary(buf_slice)).all())


# rows 0..5 are valid (lengths 0, 70, 1, 130, 63, 65); tokens 329..335 belong to no row; row 6 ends
# past total_T and row 7 ends before it starts, so both are skipped
LENGTHS = [0, 70, 1, 130, 63, 65]
TOTAL = 336


def _cu():
    cu = [0]
    for L in LENGTHS:
        cu.append(cu[-1] + L)
    cu += [cu[-1] + 50, 100]
    return cu  # [0, 0, 70, 71, 201, 264, 329, 379, 100]


@pytest.mark.parametrize("H", [2, 16])  # 16 and 128 pairs: AUTO takes the task-parallel and the one-CTA-per-pair schedule
@pytest.mark.parametrize("path", [rk.RWKV7_PATH_AUTO, rk.RWKV7_PATH_SCAN, rk.RWKV7_PATH_CHUNK])
def test_varlen_guard_bands_and_skipped_rows(path, H):
    cu = _cu()
    Bn = len(cu) - 1
    d = wi.draw(1, TOTAL, H, seed=4300 + H, s0_std=0.1)
    ops = {n: d[n][0].to("cuda") for n in OPS}
    g = torch.Generator().manual_seed(4301 + H)
    s_in = (torch.randn((Bn, H, N, N), generator=g) * 0.1).contiguous()
    cu_dev = torch.tensor(cu, dtype=torch.int32, device="cuda")

    ybuf, y = _guarded(TOTAL * H * N, torch.bfloat16)
    sbuf, s_out = _guarded(Bn * H * N * N, torch.float32)
    y = y.view(TOTAL, H, N)
    s_out = s_out.view(Bn, H, N, N)
    rk.rwkv7_wkv_prefill_varlen_bf16(path, cu_dev, max(LENGTHS), *[ops[n] for n in OPS], s_in.cuda(), y, s_out)
    torch.cuda.synchronize()
    assert rk.rwkv7_get_last_error() == 0

    assert _guards_intact(ybuf) and _guards_intact(sbuf)
    y_bits = ybuf[GUARD:GUARD + TOTAL * H * N].view(TOTAL, H, N)
    s_bits = sbuf[GUARD:GUARD + Bn * H * N * N].view(Bn, H, N, N)
    assert _is_canary(y_bits[cu[len(LENGTHS)]:])      # tokens of no row
    for b in (6, 7):                                    # skipped rows
        assert _is_canary(s_bits[b])
    assert torch.equal(s_out[0].cpu(), s_in[0])        # an empty row's end state is its start state
    for b in range(1, len(LENGTHS)):
        lo, hi = cu[b], cu[b + 1]
        sl = [d[n + "_f32"][:, lo:hi] for n in OPS]
        yo, so = oracle.wkv7(*sl, s_in[b:b + 1])
        assert rel_err(y[lo:hi], yo[0]) <= TOL_BF16, b
        assert rel_err(s_out[b], so[0]) <= TOL_BF16, b


@pytest.mark.parametrize("sched", [None, rk.RWKV7_SCHED_PAIR, rk.RWKV7_SCHED_TASKS, rk.RWKV7_SCHED_PIPE])
@pytest.mark.parametrize("T", [65, 130, 191])
def test_dense_ragged_tail_guard_bands(T, sched):
    B, H = 2, 3
    d = wi.draw(B, T, H, seed=4400 + T, s0_std=0.1)
    yo, so = oracle.wkv7(*oracle_ops(d), d["s0"])
    dv = to_dev(d)
    ybuf, y = _guarded(B * T * H * N, torch.bfloat16)
    sbuf, s_out = _guarded(B * H * N * N, torch.float32)
    y = y.view(B, T, H, N)
    s_out = s_out.view(B, H, N, N)
    if sched is None:
        rk.rwkv7_wkv_prefill_bf16_path(rk.RWKV7_PATH_SCAN, *[dv[n] for n in OPS], dv["s0"], y, s_out)
    else:
        rk.rwkv7_wkv_prefill_ext_bf16(rk.RWKV7_PATH_CHUNK, *[dv[n] for n in OPS], dv["s0"], y, s_out,
                                      schedule=sched)
    torch.cuda.synchronize()
    assert rk.rwkv7_get_last_error() == 0
    assert _guards_intact(ybuf) and _guards_intact(sbuf)
    assert rel_err(y, yo) <= TOL_BF16 and rel_err(s_out, so) <= TOL_BF16


def test_decode_guard_bands():
    B, H = 5, 3
    d = wi.draw(B, 1, H, seed=4500, s0_std=0.1)
    yo, so = oracle.wkv7(*oracle_ops(d), d["s0"])
    ops = {n: d[n][:, 0].contiguous().cuda() for n in OPS}
    ybuf, y = _guarded(B * H * N, torch.bfloat16)
    sbuf, s = _guarded(B * H * N * N, torch.float32)
    y = y.view(B, H, N)
    s = s.view(B, H, N, N)
    s.copy_(d["s0"].cuda())
    rk.rwkv7_wkv_decode_bf16(*[ops[n] for n in OPS], s, y)
    torch.cuda.synchronize()
    assert rk.rwkv7_get_last_error() == 0
    assert _guards_intact(ybuf) and _guards_intact(sbuf)
    assert rel_err(y, yo[:, 0]) <= TOL_BF16 and rel_err(s, so) <= TOL_BF16
