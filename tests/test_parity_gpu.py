"""GPU parity: every CUDA kernel against the float64 oracle on the same seeded
inputs, through the C ABI.

Bars (max|gpu - oracle| / max|oracle| over the compared output): 1e-4 for
float32 operands, 5e-3 for bfloat16 operands (float32 state in both).  Small
cases compare every element and span several token tiles plus a ragged tail;
the full-size workloads compare sampled (batch, head) pairs, which the oracle
computes on their own (pairs are independent of each other).
"""

import numpy as np
import pytest
import torch

import oracle
import rwkv_delta_rule_b200 as rk
import wkv7_inputs as wi
from helpers import OPS, TOL_BF16, TOL_BF16_PAIR, TOL_F32, need_cuda, oracle_ops, rel_err, to_dev

pytestmark = pytest.mark.gpu


@pytest.fixture(autouse=True)
def _cuda():
    need_cuda()
    rk.load_library()
    yield
    assert rk.rwkv7_get_last_error() == 0


def gpu_prefill(dd, s0, path=rk.RWKV7_PATH_AUTO):
    y, s = rk.prefill(*[dd[n] for n in OPS], s0, path=path)
    torch.cuda.synchronize()
    return y, s


# ---- small cases: whole outputs ----------------------------------------------------------------------

def test_scan_f32_prefill_b1_t64_h2():
    d = wi.draw_case(wi.CASES["prefill_f32_b1_t64_h2"])
    yo, so = oracle.wkv7(*oracle_ops(d), None)
    y, s = gpu_prefill(to_dev(d), None)
    assert rel_err(y, yo) <= TOL_F32
    assert rel_err(s, so) <= TOL_F32


PATHS = [pytest.param(rk.RWKV7_PATH_SCAN, id="scan"), pytest.param(rk.RWKV7_PATH_CHUNK, id="chunk")]


@pytest.mark.parametrize("path", PATHS)
@pytest.mark.parametrize("T", [1, 2, 31, 32, 33, 63, 64, 65, 100, 127, 128, 129, 257])
def test_bf16_ragged_tails(T, path):
    d = wi.draw(2, T, 3, seed=100 + T, dtype="bf16", s0_std=0.1)
    yo, so = oracle.wkv7(*oracle_ops(d), d["s0"])
    dd = to_dev(d)
    y, s = gpu_prefill(dd, dd["s0"], path)
    assert rel_err(y, yo) <= TOL_BF16
    assert rel_err(s, so) <= TOL_BF16


@pytest.mark.parametrize("path", PATHS)
@pytest.mark.parametrize("z_mean", [-3.0, 1.0, 3.0])
def test_bf16_decay_regimes(z_mean, path):
    """Slow (w ~ 0.97), fast (w ~ 0.65) and fastest (w ~ 0.56) decay."""
    d = wi.draw(2, 700, 2, seed=int(20 + z_mean), dtype="bf16", z_mean=z_mean, s0_std=0.1)
    yo, so = oracle.wkv7(*oracle_ops(d), d["s0"])
    dd = to_dev(d)
    y, s = gpu_prefill(dd, dd["s0"], path)
    assert rel_err(y, yo) <= TOL_BF16
    assert rel_err(s, so) <= TOL_BF16


def test_chunk_matches_scan_elementwise():
    """The two kernels agree with each other on every element (both fp32-state)."""
    d = wi.draw(3, 640, 4, seed=33, dtype="bf16", s0_std=0.1)
    dd = to_dev(d)
    yc, sc = gpu_prefill(dd, dd["s0"], rk.RWKV7_PATH_CHUNK)
    ys, ss = gpu_prefill(dd, dd["s0"], rk.RWKV7_PATH_SCAN)
    assert rel_err(yc, ys.float().cpu().numpy()) <= TOL_BF16_PAIR
    assert rel_err(sc, ss.cpu().numpy()) <= 1e-3


def test_scan_f32_longer_with_state():
    d = wi.draw(2, 300, 2, seed=7, dtype="f32", s0_std=0.1)
    yo, so = oracle.wkv7(*oracle_ops(d), d["s0"])
    dd = to_dev(d)
    y, s = gpu_prefill(dd, dd["s0"])
    assert rel_err(y, yo) <= TOL_F32
    assert rel_err(s, so) <= TOL_F32


@pytest.mark.parametrize("path", PATHS)
def test_t_zero_copies_state(path):
    d = wi.draw(2, 0, 3, seed=9, dtype="bf16", s0_std=0.1)
    dd = to_dev(d)
    y, s = gpu_prefill(dd, dd["s0"], path)
    assert torch.equal(s, dd["s0"])
    y, s = gpu_prefill(dd, None, path)
    assert torch.count_nonzero(s) == 0


@pytest.mark.parametrize("path", PATHS)
def test_in_place_state(path):
    d = wi.draw(1, 145, 2, seed=10, dtype="bf16", s0_std=0.1)
    yo, so = oracle.wkv7(*oracle_ops(d), d["s0"])
    dd = to_dev(d)
    st = dd["s0"].clone()
    y = torch.empty_like(dd["r"])
    rk.rwkv7_wkv_prefill_bf16_path(path, *[dd[n] for n in OPS], st, y, st)
    torch.cuda.synchronize()
    assert rel_err(y, yo) <= TOL_BF16
    assert rel_err(st, so) <= TOL_BF16


@pytest.mark.parametrize("path", PATHS)
def test_chained_calls_equal_one_call(path):
    d = wi.draw(2, 230, 2, seed=11, dtype="bf16", s0_std=0.1)
    yo, so = oracle.wkv7(*oracle_ops(d), d["s0"])
    dd = to_dev(d)
    s = dd["s0"]
    ys = []
    for lo, hi in ((0, 1), (1, 64), (64, 65), (65, 130), (130, 230)):
        part = {n: dd[n][:, lo:hi].contiguous() for n in OPS}
        yp, s = gpu_prefill(part, s, path)
        ys.append(yp)
    assert rel_err(torch.cat(ys, 1), yo) <= TOL_BF16
    assert rel_err(s, so) <= TOL_BF16


@pytest.mark.parametrize("dtype", ["f32", "bf16"])
def test_decode_steps_equal_oracle(dtype):
    T = 40
    d = wi.draw(3, T, 5, seed=12, dtype=dtype, s0_std=0.1)
    yo, so = oracle.wkv7(*oracle_ops(d), d["s0"])
    dd = to_dev(d)
    st = dd["s0"].clone()
    ys = []
    for t in range(T):
        ys.append(rk.decode_(*[dd[n][:, t].contiguous() for n in OPS], st))
    torch.cuda.synchronize()
    tol = TOL_F32 if dtype == "f32" else TOL_BF16
    assert rel_err(torch.stack(ys, 1), yo) <= tol
    assert rel_err(st, so) <= tol


@pytest.mark.parametrize("bf16_state", [False, True])
def test_decode_steps_in_a_cuda_graph(bf16_state):
    # back-to-back steps on ONE state, captured in a CUDA graph and replayed: each step's launch may
    # overlap the previous step's last wave (programmatic dependent launch) and must still read the
    # state that step wrote
    B, H, T = 4, 6, 24
    d = wi.draw(B, T, H, seed=14, s0_std=0.1)
    ops = [n + "_f32" for n in OPS]
    steps = {n: torch.stack([d[n][:, t].contiguous() for t in range(T)]).cuda() for n in OPS}  # [T, B, H, 64]
    ys = torch.empty((T, B, H, 64), dtype=torch.bfloat16, device="cuda")
    st = (d["s0"].to(torch.bfloat16) if bf16_state else d["s0"]).cuda()
    st0 = st.clone()
    step = rk.rwkv7_wkv_decode_bf16_bf16state if bf16_state else rk.rwkv7_wkv_decode_bf16

    def run():
        for t in range(T):
            step(*[steps[n][t] for n in OPS], st, ys[t])

    side = torch.cuda.Stream()
    side.wait_stream(torch.cuda.current_stream())
    with torch.cuda.stream(side):
        run()  # warm-up outside the capture
    torch.cuda.current_stream().wait_stream(side)
    g = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g):
        run()
    st.copy_(st0)
    g.replay()
    torch.cuda.synchronize()
    if bf16_state:
        s_or = oracle.round_bf16(d["s0"].numpy())
        yo = []
        for t in range(T):
            y1, s_or = oracle.decode_step_bf16_state(*[d[n][:, t] for n in ops], s_or)
            yo.append(y1)
        assert rel_err(ys.transpose(0, 1), np.stack(yo, 1)) <= TOL_BF16
        assert rel_err(st.float(), s_or) <= 2.0 ** -7
    else:
        yo, so = oracle.wkv7(*oracle_ops(d), d["s0"])
        assert rel_err(ys.transpose(0, 1), yo) <= TOL_BF16
        assert rel_err(st, so) <= TOL_BF16


@pytest.mark.parametrize("path", PATHS)
def test_varlen_small(path):
    lens = torch.tensor([1, 0, 33, 64, 65, 7, 200])
    d = wi.draw_packed(lens, 3, seed=13, s0_std=0.1)
    cu = d["cu_seqlens"]
    yo, so = oracle.wkv7_varlen(*oracle_ops(d), cu, d["s0"])
    dd = to_dev(d)
    y = torch.empty_like(dd["r"])
    s = torch.empty_like(dd["s0"])
    rk.rwkv7_wkv_prefill_varlen_bf16(path, cu.cuda(), int(lens.max()), *[dd[n] for n in OPS],
                                     dd["s0"], y, s)
    torch.cuda.synchronize()
    assert rel_err(y, yo) <= TOL_BF16
    assert rel_err(s, so) <= TOL_BF16


# ---- full-size workloads: sampled (b, h) pairs -------------------------------------------------------

def sampled_pairs(B, H, n, seed):
    rng = np.random.default_rng(seed)
    pairs = {(0, 0), (B - 1, H - 1)}
    while len(pairs) < min(n, B * H):
        pairs.add((int(rng.integers(B)), int(rng.integers(H))))
    return sorted(pairs)


def check_pairs(d, s0, y, s, pairs, tol, t_lo=0, t_hi=None):
    for (b, h) in pairs:
        ops = [d[n + "_f32"][b:b + 1, t_lo:t_hi, h:h + 1] for n in OPS]
        si = None if s0 is None else s0[b:b + 1, h:h + 1]
        yo, so = oracle.wkv7(*ops, si)
        assert rel_err(y[b:b + 1, t_lo:t_hi, h:h + 1], yo) <= tol, (b, h)
        assert rel_err(s[b:b + 1, h:h + 1], so) <= tol, (b, h)


@pytest.mark.slow
def test_full_prefill_d768_b8_t4096():
    case = wi.CASES["prefill_d768_b8_t4096"]
    d = wi.draw_case(case)
    dd = to_dev(d)
    y, s = gpu_prefill(dd, dd["s0"], rk.RWKV7_PATH_CHUNK)
    check_pairs(d, d["s0"], y.cpu(), s.cpu(), sampled_pairs(case.B, case.H, 6, 1), TOL_BF16)
    ys, ss = gpu_prefill(dd, dd["s0"], rk.RWKV7_PATH_SCAN)
    assert rel_err(y, ys.float().cpu().numpy()) <= TOL_BF16_PAIR
    assert rel_err(s, ss.cpu().numpy()) <= TOL_BF16


@pytest.mark.slow
@pytest.mark.parametrize("path", [rk.RWKV7_PATH_CHUNK, rk.RWKV7_PATH_SCAN])
def test_full_size_pure_accumulation_every_pair(path):
    # w = 1, a = b = 0 at the D768 B8 T4096 H12 shape and launch configuration: the recurrence reduces to
    # S_t = S0 + sum_{tau <= t} v_tau k_tau^T, a closed form checked on EVERY (b, h): the end state in
    # full, y at sampled tokens (float64 matmuls of the same bf16 values)
    case = wi.CASES["prefill_d768_b8_t4096"]
    d = wi.draw_case(case)
    dd = to_dev(d)
    dd["w"] = torch.ones_like(dd["w"])
    dd["a"] = torch.zeros_like(dd["a"])
    dd["b"] = torch.zeros_like(dd["b"])
    y, s = gpu_prefill(dd, dd["s0"], path)
    v = d["v"].double().numpy().transpose(0, 2, 3, 1)  # [B, H, 64 (i), T]
    k = d["k"].double().numpy().transpose(0, 2, 1, 3)  # [B, H, T, 64 (j)]
    r = d["r"].double().numpy()                          # [B, T, H, 64]
    s0 = d["s0"].double().numpy()
    assert rel_err(s, s0 + np.matmul(v, k)) <= TOL_F32
    yc = y.float().cpu().numpy()
    for t in (0, 63, 64, 1000, case.T - 1):
        st = s0 + np.matmul(v[..., :t + 1], k[:, :, :t + 1])
        yo = np.einsum("bhij,bhj->bhi", st, r[:, t])
        assert rel_err(yc[:, t], yo) <= TOL_BF16, t


@pytest.mark.slow
def test_full_prefill_d2048_chained():
    case = wi.CASES["prefill_d2048_b16_t8192_chained"]
    d = wi.draw_case(case)
    dd = to_dev(d)
    half = case.T // 2
    p1 = {n: dd[n][:, :half].contiguous() for n in OPS}
    p2 = {n: dd[n][:, half:].contiguous() for n in OPS}
    y1, s1 = gpu_prefill(p1, None)
    y2, s2 = gpu_prefill(p2, s1)
    del p1, p2
    y = torch.cat([y1, y2], 1).cpu()
    check_pairs(d, None, y, s2.cpu(), sampled_pairs(case.B, case.H, 4, 2), TOL_BF16)


@pytest.mark.slow
def test_full_decode_l24_d1024_equals_prefill():
    case = wi.CASES["decode_l24_d1024_b256_1024steps"]
    d = wi.draw_case(case)
    dd = to_dev(d)
    steps = {n: dd[n].transpose(0, 1).contiguous() for n in OPS}  # [T, B, H, N]
    st = torch.zeros(case.B, case.H, 64, 64, device="cuda")
    y = torch.empty_like(steps["r"])
    for t in range(case.T):
        rk.rwkv7_wkv_decode_bf16(*[steps[n][t] for n in OPS], st, y[t])
    torch.cuda.synchronize()
    y = y.transpose(0, 1)
    pairs = sampled_pairs(case.B, case.H, 4, 3)
    check_pairs(d, None, y.cpu(), st.cpu(), pairs, TOL_BF16)
    # decode == prefill on every element, for both prefill kernels; each
    # prefill also against the oracle on the sampled pairs
    for path, tol_s in ((rk.RWKV7_PATH_SCAN, 1e-4), (rk.RWKV7_PATH_CHUNK, 2e-3)):
        yp, sp = gpu_prefill(dd, None, path)
        assert rel_err(y, yp.float().cpu().numpy()) <= TOL_BF16_PAIR
        assert rel_err(st, sp.cpu().numpy()) <= tol_s
        check_pairs(d, None, yp.cpu(), sp.cpu(), pairs, TOL_BF16)
        del yp, sp


@pytest.mark.slow
def test_full_prefill_d4096_b4_t16384_and_ragged():
    # the headline workload in the launch configuration the bench times (AUTO: one CTA per pair at 256
    # pairs): 12 sampled pairs against the oracle, and every element against the sequential scan, an
    # independent kernel (the chunked form's inverse and decay algebra on every pair)
    case = wi.CASES["prefill_d4096_b4_t16384"]
    d = wi.draw_case(case)
    dd = to_dev(d)
    y, s = gpu_prefill(dd, None)
    check_pairs(d, None, y.cpu(), s.cpu(), sampled_pairs(case.B, case.H, 12, 4), TOL_BF16)
    ys, ss = gpu_prefill(dd, None, rk.RWKV7_PATH_SCAN)
    assert rel_err(y, ys.float().cpu().numpy()) <= TOL_BF16_PAIR
    assert rel_err(s, ss.cpu().numpy()) <= TOL_BF16
    del dd, y, s, d, ys, ss
    lens = wi.ragged_lengths(case.B, 1024, 16384, seed=case.seed + 1)
    d = wi.draw_packed(lens, case.H, seed=case.seed + 2, z_mean=case.z_mean)
    dd = to_dev(d)
    cu = d["cu_seqlens"]
    y = torch.empty_like(dd["r"])
    s = torch.empty(case.B, case.H, 64, 64, device="cuda")
    rk.rwkv7_wkv_prefill_varlen_bf16(rk.RWKV7_PATH_AUTO, cu.cuda(), int(lens.max()), *[dd[n] for n in OPS], None,
                                     y, s)
    torch.cuda.synchronize()
    y = y.cpu()
    s = s.cpu()
    for b in range(case.B):
        lo, hi = int(cu[b]), int(cu[b + 1])
        for h in (0, case.H - 1):
            ops = [d[n + "_f32"][lo:hi, h:h + 1][None] for n in OPS]
            yo, so = oracle.wkv7(*ops, None)
            assert rel_err(y[lo:hi, h:h + 1][None], yo) <= TOL_BF16, (b, h)
            assert rel_err(s[b:b + 1, h:h + 1], so) <= TOL_BF16, (b, h)


@pytest.mark.slow
def test_full_size_headline_pure_accumulation_every_pair():
    # w = 1, a = b = 0 at the headline shape (B4 T16384 H64) and launch configuration: the end state of
    # EVERY (b, h) equals sum_t v_t k_t^T (zero initial state), and y at sampled tokens equals the
    # closed form (float64 matmuls of the same bf16 values)
    case = wi.CASES["prefill_d4096_b4_t16384"]
    d = wi.draw_case(case)
    dd = to_dev(d)
    dd["w"] = torch.ones_like(dd["w"])
    dd["a"] = torch.zeros_like(dd["a"])
    dd["b"] = torch.zeros_like(dd["b"])
    y, s = gpu_prefill(dd, None)
    del dd
    v = d["v"].double().numpy().transpose(0, 2, 3, 1)  # [B, H, 64 (i), T]
    k = d["k"].double().numpy().transpose(0, 2, 1, 3)  # [B, H, T, 64 (j)]
    r = d["r"].double().numpy()                          # [B, T, H, 64]
    assert rel_err(s, np.matmul(v, k)) <= TOL_F32
    yc = y.float().cpu().numpy()
    for t in (0, 63, 64, 8191, case.T - 1):
        st = np.matmul(v[..., :t + 1], k[:, :, :t + 1])
        yo = np.einsum("bhij,bhj->bhi", st, r[:, t])
        assert rel_err(yc[:, t], yo) <= TOL_BF16, t
