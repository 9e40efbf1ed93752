"""GPU parity of the prefill across the decay domain [0, 1] against the float64 oracle.

The chunked form divides by the product of up to 64 consecutive decays.  The model's decays lie in
[0.5452, 1) (RWKV-7 G0 7.2B walkthrough, lshu.cn/news/198401, section 7.1), but the recurrence takes any
w in [0, 1], so the kernels are checked on decays the model never produces:
  * w ~ U(0.27, 0.55): every chunked schedule stays inside its factorised range and matches the oracle;
  * w ~ U(0.02, 0.27), w = 0 in places, and a long sequence with a stretch of fast decays: every
    chunked schedule runs a chunk outside its factorised range token by token in float32, so all of
    them, AUTO and the sequential scan match the oracle (model-native inputs never leave the range;
    they would report RWKV7_ERR_DOMAIN);
  * w = 1 everywhere (no decay at all).
Bars as for every bf16 parity test: max|gpu - oracle| / max|oracle| <= 5e-3 for y and the end state.
"""

import numpy as np
import pytest
import torch

import oracle
import rwkv_delta_rule_b200 as rk
import wkv7_inputs as wi
from helpers import OPS, TOL_BF16, need_cuda, oracle_ops, rel_err, to_dev

pytestmark = pytest.mark.gpu

ERR_DOMAIN = 6


@pytest.fixture(autouse=True)
def _cuda():
    need_cuda()
    rk.load_library()
    assert rk.rwkv7_get_last_error() == 0
    yield


def _draw(B, T, H, seed, wfun):
    """The config generator's inputs with the decay replaced by wfun(generator, shape), rounded to bf16."""
    d = wi.draw(B, T, H, seed=seed, s0_std=0.1)
    g = torch.Generator().manual_seed(seed + 1)
    w = wfun(g, d["w"].shape).to(torch.bfloat16)
    d["w"], d["w_f32"] = w, w.float()
    return d


def _uniform(lo, hi):
    return lambda g, shape: lo + (hi - lo) * torch.rand(shape, generator=g)


def _chunk(d, sched, path=rk.RWKV7_PATH_CHUNK):
    dv = to_dev(d)
    y, s = rk.prefill_ext(*[dv[n] for n in OPS], dv["s0"], path=path, schedule=sched)
    torch.cuda.synchronize()
    return y, s, rk.rwkv7_get_last_error()


@pytest.mark.parametrize("sched", [rk.RWKV7_SCHED_PAIR, rk.RWKV7_SCHED_TASKS, rk.RWKV7_SCHED_PIPE])
@pytest.mark.parametrize("B,T,H", [(1, 300, 2), (2, 1000, 3)])
def test_moderate_decay_every_chunk_schedule(B, T, H, sched):
    d = _draw(B, T, H, 900 + T, _uniform(0.27, 0.55))
    yo, so = oracle.wkv7(*oracle_ops(d), d["s0"])
    y, s, st = _chunk(d, sched)
    assert st == 0
    assert rel_err(y, yo) <= TOL_BF16
    assert rel_err(s, so) <= TOL_BF16


@pytest.mark.parametrize("B,T,H", [(1, 300, 2), (2, 130, 3)])
def test_fast_decay(B, T, H):
    d = _draw(B, T, H, 910 + T, _uniform(0.02, 0.27))
    yo, so = oracle.wkv7(*oracle_ops(d), d["s0"])
    y, s, st = _chunk(d, rk.RWKV7_SCHED_PIPE)
    assert st == 0
    assert rel_err(y, yo) <= TOL_BF16
    assert rel_err(s, so) <= TOL_BF16
    y, s, st = _chunk(d, rk.RWKV7_SCHED_AUTO, path=rk.RWKV7_PATH_SCAN)
    assert st == 0
    assert rel_err(y, yo) <= TOL_BF16
    assert rel_err(s, so) <= TOL_BF16
    # the other chunked schedules cannot factorise these chunks either: they run them token by token
    for sched in (rk.RWKV7_SCHED_AUTO, rk.RWKV7_SCHED_PAIR, rk.RWKV7_SCHED_TASKS):
        y, s, st = _chunk(d, sched)
        assert st == 0, sched
        assert rel_err(y, yo) <= TOL_BF16, sched
        assert rel_err(s, so) <= TOL_BF16, sched


def test_zero_decay_in_places():
    def wfun(g, shape):
        w = 0.55 + 0.45 * torch.rand(shape, generator=g)
        return torch.where(torch.rand(shape, generator=g) < 0.01, torch.zeros(shape), w)

    d = _draw(1, 257, 2, 920, wfun)
    yo, so = oracle.wkv7(*oracle_ops(d), d["s0"])
    for sched in (rk.RWKV7_SCHED_PIPE, rk.RWKV7_SCHED_PAIR, rk.RWKV7_SCHED_TASKS):
        y, s, st = _chunk(d, sched)
        assert st == 0, sched
        assert rel_err(y, yo) <= TOL_BF16, sched
        assert rel_err(s, so) <= TOL_BF16, sched


def test_long_sequence_with_a_stretch_of_fast_decay():
    # T = 4096: model decays, except tokens 700..1400 (chunks 10..21) with w ~ U(0.02, 0.27)
    def wfun(g, shape):
        w = 0.5452 + 0.4548 * torch.rand(shape, generator=g)
        w[:, 700:1400] = 0.02 + 0.25 * torch.rand(w[:, 700:1400].shape, generator=g)
        return w

    d = _draw(1, 4096, 2, 930, wfun)
    yo, so = oracle.wkv7(*oracle_ops(d), d["s0"])
    for sched in (rk.RWKV7_SCHED_PIPE, rk.RWKV7_SCHED_AUTO, rk.RWKV7_SCHED_PAIR, rk.RWKV7_SCHED_TASKS):
        y, s, st = _chunk(d, sched)
        assert st == 0, sched
        assert rel_err(y, yo) <= TOL_BF16, sched
        assert rel_err(s, so) <= TOL_BF16, sched


@pytest.mark.parametrize("sched", [rk.RWKV7_SCHED_PAIR, rk.RWKV7_SCHED_TASKS])
def test_fast_decay_with_options_and_checkpoints(sched):
    # the token-by-token path with the GroupNorm epilogue, and the checkpointing forward's saved states
    def wfun(g, shape):
        w = 0.5452 + 0.4548 * torch.rand(shape, generator=g)
        w[:, 64:192] = 0.02 + 0.25 * torch.rand(w[:, 64:192].shape, generator=g)
        return w

    d = _draw(2, 300, 3, 950, wfun)
    yo, so = oracle.wkv7(*oracle_ops(d), d["s0"])
    ln = wi.draw_group_norm(3, seed=951)
    yn = oracle.group_norm_heads(yo, ln["ln_w"], ln["ln_b"])
    dv = to_dev(d)
    y, s = rk.prefill_ext(*[dv[n] for n in OPS], dv["s0"], path=rk.RWKV7_PATH_CHUNK, group_norm=True,
                          ln_w=ln["ln_w"].cuda(), ln_b=ln["ln_b"].cuda(), schedule=sched)
    torch.cuda.synchronize()
    assert rk.rwkv7_get_last_error() == 0
    assert rel_err(y, yn) <= TOL_BF16
    assert rel_err(s, so) <= TOL_BF16
    if sched == rk.RWKV7_SCHED_PAIR:
        return
    # checkpoints: the state before every 64th token (the chunked forward saves them on the tasks schedule)
    y2, s2, states = rk.prefill_save(*[dv[n] for n in OPS], dv["s0"], path=rk.RWKV7_PATH_CHUNK)
    torch.cuda.synchronize()
    assert rk.rwkv7_get_last_error() == 0
    assert rel_err(y2, yo) <= TOL_BF16
    for c in range(states.shape[2]):
        t = 64 * c
        if t == 0:
            ref = d["s0"].numpy()
        else:
            _, ref = oracle.wkv7(*[d[n + "_f32"][:, :t] for n in OPS], d["s0"])
        assert rel_err(states[:, :, c], ref) <= TOL_BF16, c


@pytest.mark.parametrize("sched", [rk.RWKV7_SCHED_AUTO, rk.RWKV7_SCHED_PIPE])
def test_no_decay(sched):
    d = _draw(2, 200, 2, 940, lambda g, shape: torch.ones(shape))
    yo, so = oracle.wkv7(*oracle_ops(d), d["s0"])
    y, s, st = _chunk(d, sched)
    assert st == 0
    assert rel_err(y, yo) <= TOL_BF16
    assert rel_err(s, so) <= TOL_BF16


def test_fast_decay_checkpoints_one_cta_per_pair():
    # 120 (b, h) pairs: AUTO takes one CTA per pair for the checkpointing forward; chunks 1..2 of every
    # sequence run token by token, and the saved states and y match the oracle on sampled pairs
    def wfun(g, shape):
        w = 0.5452 + 0.4548 * torch.rand(shape, generator=g)
        w[:, 64:192] = 0.02 + 0.25 * torch.rand(w[:, 64:192].shape, generator=g)
        return w

    B, T, H = 2, 260, 60
    d = _draw(B, T, H, 960, wfun)
    dv = to_dev(d)
    y, s_out, states = rk.prefill_save(*[dv[n] for n in OPS], dv["s0"], path=rk.RWKV7_PATH_CHUNK)
    torch.cuda.synchronize()
    assert rk.rwkv7_get_last_error() == 0
    for (b, h) in ((0, 0), (1, 59), (0, 31), (1, 7)):
        ops = [d[n + "_f32"][b:b + 1, :, h:h + 1] for n in OPS]
        s0 = d["s0"][b:b + 1, h:h + 1]
        yo, so = oracle.wkv7(*ops, s0)
        assert rel_err(y[b:b + 1, :, h:h + 1], yo) <= TOL_BF16, (b, h)
        assert rel_err(s_out[b:b + 1, h:h + 1], so) <= TOL_BF16, (b, h)
        for c in range(1, states.shape[2]):
            _, ref = oracle.wkv7(*[x[:, :64 * c] for x in ops], s0)
            assert rel_err(states[b:b + 1, h:h + 1, c], ref) <= TOL_BF16, (b, h, c)


@pytest.mark.parametrize("H", [2, 60])  # 6 and 180 pairs: the task-parallel and the one-CTA-per-pair schedule
def test_fast_decay_ragged_batch(H):
    # packed rows of 70, 1, 200 and 130 tokens with a stretch of fast decay: the token-by-token path
    # indexes the packed layout through each row's offsets
    lengths = torch.tensor([70, 1, 200, 130])
    cu = wi.cu_seqlens(lengths)
    total = int(lengths.sum())

    def wfun(g, shape):
        w = 0.5452 + 0.4548 * torch.rand(shape, generator=g)
        w[:, 60:180] = 0.02 + 0.25 * torch.rand(w[:, 60:180].shape, generator=g)
        return w

    d = _draw(1, total, H, 970 + H, wfun)
    Bn = lengths.numel()
    g = torch.Generator().manual_seed(971 + H)
    s_in = (torch.randn((Bn, H, 64, 64), generator=g) * 0.1).contiguous()
    ops = {n: d[n][0].cuda() for n in OPS}
    y = torch.empty(total, H, 64, dtype=torch.bfloat16, device="cuda")
    s_out = torch.empty(Bn, H, 64, 64, device="cuda")
    rk.rwkv7_wkv_prefill_varlen_bf16(rk.RWKV7_PATH_CHUNK, cu.cuda(), int(lengths.max()), *[ops[n] for n in OPS],
                                     s_in.cuda(), y, s_out)
    torch.cuda.synchronize()
    assert rk.rwkv7_get_last_error() == 0
    heads = range(H) if H <= 2 else (0, H // 2, H - 1)
    for b in range(Bn):
        lo, hi = int(cu[b]), int(cu[b + 1])
        for h in heads:
            sl = [d[n + "_f32"][:, lo:hi, h:h + 1] for n in OPS]
            yo, so = oracle.wkv7(*sl, s_in[b:b + 1, h:h + 1])
            assert rel_err(y[lo:hi, h:h + 1][None], yo) <= TOL_BF16, (b, h)
            assert rel_err(s_out[b:b + 1, h:h + 1], so) <= TOL_BF16, (b, h)
