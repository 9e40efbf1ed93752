"""GPU parity of the training backward (``rwkv7_wkv_backward_bf16``, with the checkpoints of
``rwkv7_wkv_prefill_save_bf16``) against the float64 backward oracle, through the C ABI.

The gradients are float32 outputs computed in float32 from exact (bf16) inputs, so the bar is the
float32 accumulation error over the sequence rather than an output rounding: max|gpu - oracle| over
max|oracle|, per output, <= TOL_BWD.  It is stated here from the arithmetic: every gradient is a
sum over later tokens of float32 products (relative rounding 2^-24 per operation), with the
recomputed states carrying the same float32 error as the forward scan, which meets 1e-4 on fp32
operands; 1e-3 leaves an order of magnitude for the longer sums.  That bar holds for checkpoints
saved by the sequential scan; checkpoints saved by the chunked (tensor-core) forward carry its
state error (tf32 products, within the 5e-3 bf16 bar of the forward), which the gradients inherit,
so those are held to 5e-3.
"""

import numpy as np
import pytest
import torch

import oracle
import rwkv_delta_rule_b200 as rk
import wkv7_inputs as wi
from helpers import OPS, need_cuda, oracle_ops, rel_err, to_dev

pytestmark = pytest.mark.gpu

TOL_BWD = 1e-3
GRADS = ("dr", "dw", "dk", "dv", "da", "db")


@pytest.fixture(autouse=True)
def _cuda():
    need_cuda()
    rk.load_library()
    yield
    assert rk.rwkv7_get_last_error() == 0


def _check(d, gr, with_s0=True, with_ds=True, tol=TOL_BWD, path=rk.RWKV7_PATH_SCAN):
    s0 = d["s0"] if with_s0 else None
    ds = gr["ds_out"] if with_ds else None
    go = oracle.wkv7_backward(*oracle_ops(d), s0, gr["dy_f32"], ds)
    dv = to_dev(d)
    y, s_out, states = rk.prefill_save(*[dv[n] for n in OPS], dv["s0"] if with_s0 else None, path=path)
    g = rk.backward(*[dv[n] for n in OPS], states, gr["dy"].cuda(), ds.cuda() if ds is not None else None)
    torch.cuda.synchronize()
    errs = {n: rel_err(g[i], go[i]) for i, n in enumerate(GRADS + ("ds_in",))}
    for n, e in errs.items():
        assert e <= tol, (n, e, errs)
    return errs


@pytest.mark.parametrize("T", [1, 7, 8, 63, 64, 65, 130, 300])
def test_backward_matches_oracle(T):
    d = wi.draw(2, T, 3, seed=800 + T, s0_std=0.1)
    gr = wi.draw_grads(2, T, 3, seed=801 + T)
    _check(d, gr)


def test_backward_without_initial_state_or_state_gradient():
    d = wi.draw(2, 200, 2, seed=820)
    gr = wi.draw_grads(2, 200, 2, seed=821, ds_std=None)
    _check(d, gr, with_s0=False, with_ds=False)


@pytest.mark.parametrize("z_mean", [-3.0, 1.0])
def test_backward_decay_regimes(z_mean):
    d = wi.draw(1, 500, 2, seed=830, z_mean=z_mean, s0_std=0.1)
    gr = wi.draw_grads(1, 500, 2, seed=831)
    _check(d, gr)


# the chunked forward picks its schedule from the shape: 6 pairs run task-parallel, 120 pairs one
# CTA per pair (fewer than 3/4 of the SMs would be left idle)
@pytest.mark.parametrize("path,B,H,tol", [(rk.RWKV7_PATH_SCAN, 2, 3, 1e-4), (rk.RWKV7_PATH_CHUNK, 2, 3, 5e-3),
                                          (rk.RWKV7_PATH_CHUNK, 2, 60, 5e-3)], ids=["scan", "chunk-tasks", "chunk-pair"])
def test_saved_states_match_the_oracle_states(path, B, H, tol):
    # states[b, h, c] is the state before token 64 c: the oracle's end state after 64 c tokens; the
    # forward's own outputs are unchanged by saving
    T = 200
    d = wi.draw(B, T, H, seed=840, s0_std=0.1)
    dv = to_dev(d)
    y, s_out, states = rk.prefill_save(*[dv[n] for n in OPS], dv["s0"], path=path)
    y2, s2 = rk.prefill(*[dv[n] for n in OPS], dv["s0"], path=path)
    torch.cuda.synchronize()
    assert torch.equal(y, y2) and torch.equal(s_out, s2)
    assert torch.equal(states[:, :, 0].cpu(), d["s0"])
    for c in range(1, rk.n_checkpoints(T)):
        sub = [x[:, :64 * c] for x in oracle_ops(d)]
        _, so = oracle.wkv7(*sub, d["s0"])
        assert rel_err(states[:, :, c], so) <= tol


def test_backward_from_chunked_checkpoints():
    d = wi.draw(2, 300, 3, seed=845, s0_std=0.1)
    gr = wi.draw_grads(2, 300, 3, seed=846)
    _check(d, gr, tol=5e-3, path=rk.RWKV7_PATH_CHUNK)


def test_empty_sequence_passes_the_state_gradient():
    B, H = 2, 3
    d = wi.draw(B, 1, H, seed=850)
    ds = torch.randn((B, H, 64, 64), generator=torch.Generator().manual_seed(851)).cuda()
    empty = torch.empty((B, 0, H, 64), dtype=torch.bfloat16, device="cuda")
    g = rk.backward(*[empty] * 6, torch.empty((B, H, 0, 64, 64), device="cuda"), empty, ds)
    torch.cuda.synchronize()
    assert torch.equal(g[6], ds)
    assert all(x.numel() == 0 for x in g[:6])


def test_sampled_pairs_at_the_d768_shape():
    # B8 T1024 H12 on the GPU; two (b, h) pairs recomputed by the oracle
    B, T, H = 8, 1024, 12
    d = wi.draw(B, T, H, seed=860, s0_std=0.1)
    gr = wi.draw_grads(B, T, H, seed=861)
    dv = to_dev(d)
    _, _, states = rk.prefill_save(*[dv[n] for n in OPS], dv["s0"], path=rk.RWKV7_PATH_SCAN)
    g = rk.backward(*[dv[n] for n in OPS], states, gr["dy"].cuda(), gr["ds_out"].cuda())
    torch.cuda.synchronize()
    for (b, h) in ((0, 0), (5, 11)):
        sub = [x[b:b + 1, :, h:h + 1] for x in oracle_ops(d)]
        go = oracle.wkv7_backward(*sub, d["s0"][b:b + 1, h:h + 1], gr["dy_f32"][b:b + 1, :, h:h + 1],
                                  gr["ds_out"][b:b + 1, h:h + 1])
        for i, n in enumerate(GRADS):
            assert rel_err(g[i][b:b + 1, :, h:h + 1], go[i]) <= TOL_BWD, (n, b, h)
        assert rel_err(g[6][b:b + 1, h:h + 1], go[6]) <= TOL_BWD


def test_backward_rejects_missing_checkpoints():
    d = wi.draw(1, 100, 2, seed=870)
    dv = to_dev(d)
    gr = wi.draw_grads(1, 100, 2, seed=871)
    with pytest.raises(ValueError):
        rk.backward(*[dv[n] for n in OPS], torch.zeros((1, 2, 1, 64, 64), device="cuda"), gr["dy"].cuda())
