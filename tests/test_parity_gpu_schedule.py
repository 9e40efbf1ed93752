"""GPU parity of the chunked prefill under its three schedules of work -- one CTA per (b, h); every chunk
a task spread over all SMs with the state handed between CTAs through s_out; and the warp-specialised
pipeline (one persistent CTA per SM, three chunks in flight) -- against the float64 oracle, through the
C ABI's option entry point.

Shapes cover fewer pairs than SMs, more pairs than SMs (several tasks per CTA, and CTAs whose next
chunk is held by another CTA in the same round), ragged last chunks, one-chunk sequences, a zero and
a given initial state, in-place state, the model-native / GroupNorm variants, and the automatic
choice with more pairs than SMs (a partial last wave).
"""

import numpy as np
import pytest
import torch

import oracle
import rwkv_delta_rule_b200 as rk
import wkv7_inputs as wi
from helpers import OPS, TOL_BF16, need_cuda, oracle_ops, rel_err, to_dev

pytestmark = pytest.mark.gpu

SCHEDS = [pytest.param(rk.RWKV7_SCHED_PAIR, id="pair"), pytest.param(rk.RWKV7_SCHED_TASKS, id="tasks"),
          pytest.param(rk.RWKV7_SCHED_PIPE, id="pipe")]


@pytest.fixture(autouse=True)
def _cuda():
    need_cuda()
    rk.load_library()
    yield
    assert rk.rwkv7_get_last_error() == 0


def _run(d, sched, s0=True, **kw):
    dv = to_dev(d)
    y, s = rk.prefill_ext(*[dv[n] for n in OPS], dv["s0"] if s0 else None, path=rk.RWKV7_PATH_CHUNK,
                          schedule=sched, **kw)
    torch.cuda.synchronize()
    return y, s


@pytest.mark.parametrize("sched", SCHEDS)
@pytest.mark.parametrize("B,T,H", [(1, 64, 1), (2, 257, 3), (1, 1000, 2), (3, 130, 5), (2, 65, 80)])
def test_schedules_match_oracle(B, T, H, sched):
    d = wi.draw(B, T, H, seed=700 + 7 * B + T + H, s0_std=0.1)
    yo, so = oracle.wkv7(*oracle_ops(d), d["s0"])
    y, s = _run(d, sched)
    assert rel_err(y, yo) <= TOL_BF16
    assert rel_err(s, so) <= TOL_BF16


@pytest.mark.parametrize("sched", SCHEDS)
def test_schedules_zero_initial_state_and_slow_decay(sched):
    d = wi.draw(2, 700, 3, seed=720, z_mean=-3.0)
    yo, so = oracle.wkv7(*oracle_ops(d), None)
    y, s = _run(d, sched, s0=False)
    assert rel_err(y, yo) <= TOL_BF16
    assert rel_err(s, so) <= TOL_BF16


@pytest.mark.parametrize("sched", SCHEDS)
def test_schedules_in_place_state(sched):
    d = wi.draw(2, 300, 3, seed=730, s0_std=0.1)
    yo, so = oracle.wkv7(*oracle_ops(d), d["s0"])
    dv = to_dev(d)
    st = dv["s0"].clone()
    y = torch.empty_like(dv["r"])
    rk.rwkv7_wkv_prefill_ext_bf16(rk.RWKV7_PATH_CHUNK, *[dv[n] for n in OPS], st, y, st, schedule=sched)
    torch.cuda.synchronize()
    assert rel_err(y, yo) <= TOL_BF16
    assert rel_err(st, so) <= TOL_BF16


def test_many_pairs_sampled():
    # 16 x 24 = 384 pairs over the SMs: several tasks per CTA, chained through s_out; checked on sampled
    # pairs against the oracle, and against the one-CTA-per-pair schedule everywhere
    B, T, H = 16, 512, 24
    d = wi.draw(B, T, H, seed=740, s0_std=0.1)
    y2, s2 = _run(d, rk.RWKV7_SCHED_TASKS)
    y1, s1 = _run(d, rk.RWKV7_SCHED_PAIR)
    y0, s0 = _run(d, rk.RWKV7_SCHED_AUTO)
    y3, s3 = _run(d, rk.RWKV7_SCHED_PIPE)
    rng = np.random.default_rng(741)
    for _ in range(4):
        b, h = int(rng.integers(B)), int(rng.integers(H))
        sub = {n: d[n + "_f32"][b:b + 1, :, h:h + 1] for n in OPS}
        yo, so = oracle.wkv7(*[sub[n] for n in OPS], d["s0"][b:b + 1, h:h + 1])
        assert rel_err(y2[b:b + 1, :, h:h + 1], yo) <= TOL_BF16
        assert rel_err(s2[b:b + 1, h:h + 1], so) <= TOL_BF16
    assert rel_err(y2, y1.float().cpu().numpy()) <= 1e-2
    assert rel_err(s2, s1.cpu().numpy()) <= 1e-2
    assert rel_err(y0, y1.float().cpu().numpy()) <= 1e-2
    assert rel_err(s0, s1.cpu().numpy()) <= 1e-2
    assert rel_err(y3, y1.float().cpu().numpy()) <= 1e-2
    assert rel_err(s3, s1.cpu().numpy()) <= 1e-2
    for _ in range(4):
        b, h = int(rng.integers(B)), int(rng.integers(H))
        sub = {n: d[n + "_f32"][b:b + 1, :, h:h + 1] for n in OPS}
        yo, so = oracle.wkv7(*[sub[n] for n in OPS], d["s0"][b:b + 1, h:h + 1])
        assert rel_err(y3[b:b + 1, :, h:h + 1], yo) <= TOL_BF16
        assert rel_err(s3[b:b + 1, h:h + 1], so) <= TOL_BF16


@pytest.mark.parametrize("sched", SCHEDS)
def test_schedules_model_native_and_group_norm(sched):
    d = wi.draw_model_native(2, 200, 3, seed=750, s0_std=0.1)
    ln = wi.draw_group_norm(3, seed=751)
    nat = ("r", "xw", "k", "v", "xa")
    yo, so = oracle.wkv7_model_native(*[d[n + "_f32"] for n in nat], d["k_k"], d["s0"])
    zo = oracle.group_norm_heads(yo, ln["ln_w"], ln["ln_b"])
    dev = {n: d[n].cuda() for n in nat}
    y, s = rk.prefill_ext(dev["r"], dev["xw"], dev["k"], dev["v"], dev["xa"], None, d["s0"].cuda(),
                          path=rk.RWKV7_PATH_CHUNK, model_native=True, k_k=d["k_k"].cuda(), group_norm=True,
                          ln_w=ln["ln_w"].cuda(), ln_b=ln["ln_b"].cuda(), schedule=sched)
    torch.cuda.synchronize()
    assert rel_err(y, zo) <= TOL_BF16
    assert rel_err(s, so) <= TOL_BF16


def test_repeated_launches_reuse_flag_slots():
    # more launches than flag slots, back to back on one stream: every one starts from fresh flags
    d = wi.draw(1, 400, 2, seed=760, s0_std=0.1)
    yo, so = oracle.wkv7(*oracle_ops(d), d["s0"])
    dv = to_dev(d)
    for _ in range(9):
        y, s = rk.prefill_ext(*[dv[n] for n in OPS], dv["s0"], path=rk.RWKV7_PATH_CHUNK,
                              schedule=rk.RWKV7_SCHED_TASKS)
    torch.cuda.synchronize()
    assert rel_err(y, yo) <= TOL_BF16
    assert rel_err(s, so) <= TOL_BF16


@pytest.mark.parametrize("B,T,H", [(2, 200, 80), (1, 130, 300)])
def test_auto_with_a_partial_last_wave(B, T, H):
    # more pairs than SMs (160 and 300 pairs on 148 SMs): the automatic choice, against the oracle and
    # against the explicit one-CTA-per-pair schedule
    d = wi.draw(B, T, H, seed=790 + H, s0_std=0.1)
    yo, so = oracle.wkv7(*oracle_ops(d), d["s0"])
    y, s = _run(d, rk.RWKV7_SCHED_AUTO)
    assert rel_err(y, yo) <= TOL_BF16
    assert rel_err(s, so) <= TOL_BF16
    yp, sp = _run(d, rk.RWKV7_SCHED_PAIR)
    assert rel_err(y, yp.float().cpu().numpy()) <= 1e-2
    assert rel_err(s, sp.cpu().numpy()) <= 1e-2


def test_auto_with_a_partial_last_wave_saves_every_checkpoint():
    B, T, H = 2, 200, 80
    d = wi.draw(B, T, H, seed=795, s0_std=0.1)
    dv = to_dev(d)
    y, s_out, states = rk.prefill_save(*[dv[n] for n in OPS], dv["s0"], path=rk.RWKV7_PATH_CHUNK)
    torch.cuda.synchronize()
    assert torch.equal(states[:, :, 0].cpu(), d["s0"])
    for c in range(1, rk.n_checkpoints(T)):
        sub = [x[:, :64 * c] for x in oracle_ops(d)]
        _, so = oracle.wkv7(*sub, d["s0"])
        assert rel_err(states[:, :, c], so) <= TOL_BF16


def test_schedule_value_is_checked():
    d = wi.draw(1, 64, 1, seed=770)
    dv = to_dev(d)
    with pytest.raises(rk.Rwkv7Error):
        rk.prefill_ext(*[dv[n] for n in OPS], None, path=rk.RWKV7_PATH_CHUNK, schedule=4)


def test_graph_replays_start_from_fresh_flags():
    # a captured launch replays with the same epoch: each replay must still order its own chunks
    B, T, H = 2, 300, 3
    static = {n: torch.empty((B, T, H, 64), dtype=torch.bfloat16, device="cuda") for n in OPS}
    s0 = torch.empty((B, H, 64, 64), device="cuda")
    y = torch.empty((B, T, H, 64), dtype=torch.bfloat16, device="cuda")
    s_out = torch.empty_like(s0)

    def run():
        rk.rwkv7_wkv_prefill_ext_bf16(rk.RWKV7_PATH_CHUNK, *[static[n] for n in OPS], s0, y, s_out,
                                      schedule=rk.RWKV7_SCHED_TASKS)

    d = wi.draw(B, T, H, seed=780, s0_std=0.1)
    for n in OPS:
        static[n].copy_(d[n])
    s0.copy_(d["s0"])
    side = torch.cuda.Stream()
    side.wait_stream(torch.cuda.current_stream())
    with torch.cuda.stream(side):
        run()
    torch.cuda.current_stream().wait_stream(side)
    g = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g):
        run()
    for seed in (781, 782, 783):
        d = wi.draw(B, T, H, seed=seed, s0_std=0.1)
        for n in OPS:
            static[n].copy_(d[n])
        s0.copy_(d["s0"])
        g.replay()
        torch.cuda.synchronize()
        yo, so = oracle.wkv7(*oracle_ops(d), d["s0"])
        assert rel_err(y, yo) <= TOL_BF16, seed
        assert rel_err(s_out, so) <= TOL_BF16, seed


def test_concurrent_launches_on_separate_streams():
    # launches running at once take different flag slots
    runs = []
    for i, seed in enumerate((790, 791, 792)):
        d = wi.draw(2, 260, 3, seed=seed, s0_std=0.1)
        dv = to_dev(d)
        y = torch.empty_like(dv["r"])
        s_out = torch.empty_like(dv["s0"])
        runs.append((d, dv, y, s_out, torch.cuda.Stream()))
    torch.cuda.synchronize()
    for d, dv, y, s_out, st in runs:
        with torch.cuda.stream(st):
            rk.rwkv7_wkv_prefill_ext_bf16(rk.RWKV7_PATH_CHUNK, *[dv[n] for n in OPS], dv["s0"], y, s_out,
                                          schedule=rk.RWKV7_SCHED_TASKS)
    torch.cuda.synchronize()
    for d, dv, y, s_out, st in runs:
        yo, so = oracle.wkv7(*oracle_ops(d), d["s0"])
        assert rel_err(y, yo) <= TOL_BF16
        assert rel_err(s_out, so) <= TOL_BF16
