"""Pins for the float64 oracle: each check fixes the oracle to something other
than itself -- a hand-worked example, closed forms, the transition-matrix
product evaluated with numpy, invariances of the definition, and a long-double
build of the same source.  CPU only.

The recurrence (RWKV-7 G0 7.2B walkthrough, lshu.cn/news/198401, section 7.1):
S <- S diag(w) + (S a) b^T + v k^T, y = S r, per (batch row, head).
"""

import os

import numpy as np
import pytest

import oracle
import wkv7_inputs

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")


def rand_ops(rng, B, T, H, N, *, w_lo=0.5, w_hi=1.0):
    r = rng.standard_normal((B, T, H, N))
    k = rng.standard_normal((B, T, H, N))
    v = rng.standard_normal((B, T, H, N))
    a = rng.standard_normal((B, T, H, N)) / np.sqrt(N)
    b = rng.standard_normal((B, T, H, N)) / np.sqrt(N)
    w = rng.uniform(w_lo, w_hi, (B, T, H, N))
    s0 = rng.standard_normal((B, H, N, N))
    return r, w, k, v, a, b, s0


def read_golden(name):
    vals = {}
    with open(os.path.join(GOLDEN, name)) as f:
        for line in f:
            line = line.split("#", 1)[0].strip()
            if not line:
                continue
            key, rest = line.split(":", 1)
            vals[key.strip()] = np.array([float(x) for x in rest.split()], dtype=np.float64)
    return vals


def test_hand_worked_example():
    """Hand-derived N=2, T=2 example (tests/golden/x070_worked_n2_t2.txt).

    Its operands are asymmetric, so a transposed state, decay applied to rows,
    sa taken after the decay, or y read before the update all change the values."""
    g = read_golden("x070_worked_n2_t2.txt")
    shp = (1, 2, 1, 2)
    ops = [g[n].reshape(shp) for n in ("r", "w", "k", "v", "a", "b")]
    y, s = oracle.wkv7(*ops, g["s0"].reshape(1, 1, 2, 2))
    np.testing.assert_array_equal(y.reshape(-1), g["y"])
    np.testing.assert_array_equal(s.reshape(-1), g["s_out"])


def test_pure_accumulation_closed_form():
    """w = 1, a = b = 0: S_t = S0 + sum_{m<=t} v_m k_m^T and y_t = S_t r_t
    (the causal sum of outer products), computed with a numpy cumulative sum."""
    rng = np.random.default_rng(1)
    B, T, H, N = 2, 37, 3, 8
    r, w, k, v, a, b, s0 = rand_ops(rng, B, T, H, N)
    w[:] = 1.0
    a[:] = 0.0
    b[:] = 0.0
    y, s = oracle.wkv7(r, w, k, v, a, b, s0)
    outer = np.einsum("bthi,bthj->bthij", v, k)
    St = s0[:, None] + np.cumsum(outer, axis=1)  # [B,T,H,N,N]
    y_ref = np.einsum("bthij,bthj->bthi", St, r)
    np.testing.assert_allclose(y, y_ref, rtol=0, atol=1e-12 * np.abs(y_ref).max())
    np.testing.assert_allclose(s, St[:, -1], rtol=0, atol=1e-12 * np.abs(St).max())


def test_delta_rule_exact_write():
    """w = 1, a = -kh, b = kh, k = kh with |kh| = 1: one step writes v along kh
    exactly (S_new kh = v) and leaves every direction orthogonal to kh alone
    (Swarma wiki RWKV entry, "Delta Rule"; RWKV-LM README copy, the meta
    in-context learner / in-context gradient descent reading)."""
    rng = np.random.default_rng(2)
    N = 16
    for T in (1, 5):
        r, w, k, v, a, b, s0 = rand_ops(rng, 1, T, 1, N)
        kh = rng.standard_normal((1, T, 1, N))
        kh /= np.linalg.norm(kh, axis=-1, keepdims=True)
        w[:] = 1.0
        a[:] = -kh
        b[:] = kh
        k[:] = kh
        S = s0[0, 0]
        for t in range(T):
            _, s_new = oracle.wkv7(*[x[:, t:t + 1] for x in (r, w, k, v, a, b)], S[None, None])
            Sn = s_new[0, 0]
            u = kh[0, t, 0]
            np.testing.assert_allclose(Sn @ u, v[0, t, 0], atol=1e-12)
            # random direction orthogonal to u
            x = rng.standard_normal(N)
            x -= u * (u @ x)
            np.testing.assert_allclose(Sn @ x, S @ x, atol=1e-12)
            S = Sn


def test_diagonal_decay_closed_form():
    """a = b = 0: S_T[i,j] = S0[i,j] prod_l w_lj + sum_m v_mi k_mj prod_{l>m} w_lj,
    and y_t from S_t, by O(T^2) brute force."""
    rng = np.random.default_rng(3)
    B, T, H, N = 1, 23, 2, 6
    r, w, k, v, a, b, s0 = rand_ops(rng, B, T, H, N)
    a[:] = 0.0
    b[:] = 0.0
    y, s = oracle.wkv7(r, w, k, v, a, b, s0)
    for h in range(H):
        for t in range(T):
            St = s0[0, h] * np.prod(w[0, :t + 1, h], axis=0)[None, :]
            for m in range(t + 1):
                St = St + np.outer(v[0, m, h], k[0, m, h]) * np.prod(w[0, m + 1:t + 1, h], axis=0)[None, :]
            np.testing.assert_allclose(y[0, t, h], St @ r[0, t, h], rtol=1e-12, atol=1e-12)
            if t == T - 1:
                np.testing.assert_allclose(s[0, h], St, rtol=1e-12, atol=1e-12)


@pytest.mark.parametrize("N", [1, 3, 8])
def test_transition_matrix_product(N):
    """General case: with A_t = diag(w_t) + a_t b_t^T the step is
    S_t = S_{t-1} A_t + v_t k_t^T, so S_T = S0 A_1...A_T + sum_t v_t k_t^T A_{t+1}...A_T.
    Evaluated with numpy matrix products (forward products of the A_t)."""
    rng = np.random.default_rng(4 + N)
    B, T, H = 2, 19, 2
    r, w, k, v, a, b, s0 = rand_ops(rng, B, T, H, N)
    y, s = oracle.wkv7(r, w, k, v, a, b, s0)
    for bi in range(B):
        for h in range(H):
            A = [np.diag(w[bi, t, h]) + np.outer(a[bi, t, h], b[bi, t, h]) for t in range(T)]
            for t in range(T):
                P = np.eye(N)
                for l in range(t + 1):
                    P = P @ A[l]
                St = s0[bi, h] @ P
                for m in range(t + 1):
                    Q = np.eye(N)
                    for l in range(m + 1, t + 1):
                        Q = Q @ A[l]
                    St = St + np.outer(v[bi, m, h], k[bi, m, h]) @ Q
                np.testing.assert_allclose(y[bi, t, h], St @ r[bi, t, h], rtol=1e-10, atol=1e-10)
            np.testing.assert_allclose(s[bi, h], St, rtol=1e-10, atol=1e-10)


def test_split_invariance():
    """Carrying the state across calls gives the result of one call, for any
    split points (RWKV-LM README copy: forward on the whole token list equals
    forward on pieces with the state passed along)."""
    rng = np.random.default_rng(5)
    B, T, H, N = 2, 70, 2, 8
    ops = rand_ops(rng, B, T, H, N)
    y, s = oracle.wkv7(*ops[:6], ops[6])
    for cuts in ([1], [63, 64, 65], [7, 30, 31, 69]):
        edges = [0] + cuts + [T]
        S = ops[6]
        ys = []
        for lo, hi in zip(edges[:-1], edges[1:]):
            yy, S = oracle.wkv7(*[x[:, lo:hi] for x in ops[:6]], S)
            ys.append(yy)
        np.testing.assert_array_equal(np.concatenate(ys, axis=1), y)
        np.testing.assert_array_equal(S, s)


def test_t_zero_and_zero_state():
    rng = np.random.default_rng(6)
    r, w, k, v, a, b, s0 = rand_ops(rng, 1, 0, 2, 4)
    y, s = oracle.wkv7(r, w, k, v, a, b, s0)
    assert y.shape == (1, 0, 2, 4)
    np.testing.assert_array_equal(s, s0)
    r, w, k, v, a, b, s0 = rand_ops(rng, 1, 5, 2, 4)
    y0, s_0 = oracle.wkv7(r, w, k, v, a, b, None)
    y1, s_1 = oracle.wkv7(r, w, k, v, a, b, np.zeros_like(s0))
    np.testing.assert_array_equal(y0, y1)
    np.testing.assert_array_equal(s_0, s_1)


def test_linearity_in_state_and_values():
    """For fixed (w, a, b, k, r), y and S_T are jointly linear in (S0, V)."""
    rng = np.random.default_rng(7)
    B, T, H, N = 1, 29, 2, 8
    r, w, k, v1, a, b, s1 = rand_ops(rng, B, T, H, N)
    _, _, _, v2, _, _, s2 = rand_ops(rng, B, T, H, N)
    al, be = 0.7, -1.9
    ya, sa_ = oracle.wkv7(r, w, k, v1, a, b, s1)
    yb, sb_ = oracle.wkv7(r, w, k, v2, a, b, s2)
    yc, sc_ = oracle.wkv7(r, w, k, al * v1 + be * v2, a, b, al * s1 + be * s2)
    np.testing.assert_allclose(yc, al * ya + be * yb, atol=1e-11 * np.abs(yc).max())
    np.testing.assert_allclose(sc_, al * sa_ + be * sb_, atol=1e-11 * np.abs(sc_).max())


def test_key_channel_permutation():
    """Relabelling key channels j consistently in w, k, a, b, r and the state's
    columns leaves y unchanged and permutes the columns of S_T."""
    rng = np.random.default_rng(8)
    B, T, H, N = 1, 31, 2, 8
    r, w, k, v, a, b, s0 = rand_ops(rng, B, T, H, N)
    p = rng.permutation(N)
    y, s = oracle.wkv7(r, w, k, v, a, b, s0)
    yp, sp = oracle.wkv7(r[..., p], w[..., p], k[..., p], v, a[..., p], b[..., p], s0[..., p])
    np.testing.assert_allclose(yp, y, rtol=1e-12, atol=1e-12)
    np.testing.assert_allclose(sp, s[..., p], rtol=1e-12, atol=1e-12)


def test_value_channel_permutation():
    """Relabelling value channels i (rows of S, channels of v and y) permutes y
    and the rows of S_T the same way."""
    rng = np.random.default_rng(9)
    B, T, H, N = 1, 17, 1, 8
    r, w, k, v, a, b, s0 = rand_ops(rng, B, T, H, N)
    p = rng.permutation(N)
    y, s = oracle.wkv7(r, w, k, v, a, b, s0)
    yp, sp = oracle.wkv7(r, w, k, v[..., p], a, b, s0[:, :, p, :])
    np.testing.assert_allclose(yp, y[..., p], rtol=1e-12, atol=1e-12)
    np.testing.assert_allclose(sp, s[:, :, p, :], rtol=1e-12, atol=1e-12)


def test_batch_and_head_independence():
    """Each (b, h) pair evolves alone: permuting batch rows and heads permutes
    the outputs, and a pair computed on its own matches."""
    rng = np.random.default_rng(10)
    B, T, H, N = 3, 11, 4, 4
    r, w, k, v, a, b, s0 = rand_ops(rng, B, T, H, N)
    y, s = oracle.wkv7(r, w, k, v, a, b, s0)
    pb, ph = rng.permutation(B), rng.permutation(H)
    perm = lambda x: x[pb][:, :, ph]
    yp, sp = oracle.wkv7(*[perm(x) for x in (r, w, k, v, a, b)], s0[pb][:, ph])
    np.testing.assert_array_equal(yp, perm(y))
    np.testing.assert_array_equal(sp, s[pb][:, ph])
    y1, s1 = oracle.wkv7(*[x[1:2, :, 2:3] for x in (r, w, k, v, a, b)], s0[1:2, 2:3])
    np.testing.assert_array_equal(y1, y[1:2, :, 2:3])
    np.testing.assert_array_equal(s1, s[1:2, 2:3])


def test_thread_count_does_not_change_results():
    rng = np.random.default_rng(11)
    ops = rand_ops(rng, 2, 9, 3, 8)
    y1, s1 = oracle.wkv7(*ops[:6], ops[6], nthreads=1)
    y4, s4 = oracle.wkv7(*ops[:6], ops[6], nthreads=4)
    np.testing.assert_array_equal(y1, y4)
    np.testing.assert_array_equal(s1, s4)


def test_float32_operands_match_float64_path():
    """Passing exactly representable float32 operands gives the float64 result."""
    rng = np.random.default_rng(12)
    ops = [x.astype(np.float32).astype(np.float64) for x in rand_ops(rng, 1, 13, 2, 8)]
    y64, s64 = oracle.wkv7(*ops[:6], ops[6], precision="f64")
    y32, s32 = oracle.wkv7(*[x.astype(np.float32) for x in ops[:6]], ops[6], precision="f32in")
    np.testing.assert_array_equal(y64, y32)
    np.testing.assert_array_equal(s64, s32)


def test_rounding_bound_against_long_double():
    """The same source built with long double bounds the oracle's own rounding
    on the fp32 prefill workload (B1 T64 H2): relative gap ~1e-15."""
    if oracle.real_bytes("long double") <= 8:
        pytest.skip("long double is not wider than double here")
    d = wkv7_inputs.draw_case(wkv7_inputs.CASES["prefill_f32_b1_t64_h2"])
    ops = [d[n + "_f32"] for n in "rwkvab"]
    y, s = oracle.wkv7(*ops, None)
    yl, sl = oracle.wkv7(*ops, None, real="long double")
    assert np.abs(y - yl).max() <= 1e-13 * np.abs(yl).max()
    assert np.abs(s - sl).max() <= 1e-13 * np.abs(sl).max()


def test_varlen_matches_per_row_calls():
    rng = np.random.default_rng(13)
    lens = [3, 1, 7]
    cu = np.concatenate([[0], np.cumsum(lens)])
    H, N = 2, 4
    tot = int(cu[-1])
    ops = [rng.standard_normal((tot, H, N)) for _ in range(6)]
    ops[1] = rng.uniform(0.5, 1.0, (tot, H, N))
    s0 = rng.standard_normal((len(lens), H, N, N))
    y, s = oracle.wkv7_varlen(*ops, cu, s0)
    for bi in range(len(lens)):
        lo, hi = cu[bi], cu[bi + 1]
        yb, sb = oracle.wkv7(*[x[lo:hi][None] for x in ops], s0[bi:bi + 1])
        np.testing.assert_array_equal(y[lo:hi], yb[0])
        np.testing.assert_array_equal(s[bi], sb[0])


def test_input_generator_recipe():
    """The generator's structural facts: unit key directions, a = -kh,
    |b| <= |kh| componentwise, w in (0.5452, 1), bf16-rounded storage."""
    d = wkv7_inputs.draw(2, 8, 3, seed=1234, dtype="f32", s0_std=0.1)
    kh = -d["a"]
    np.testing.assert_allclose(kh.norm(dim=-1).numpy(), 1.0, rtol=1e-6)
    assert float(d["w"].min()) > 0.5452 and float(d["w"].max()) < 1.0
    assert bool(((d["b"].abs() <= kh.abs() + 1e-7)).all())
    ratio = (d["k"] / kh).numpy()
    assert ratio.min() >= 0.5 - 1e-6 and ratio.max() <= 1.5 + 1e-6
    db = wkv7_inputs.draw(2, 8, 3, seed=1234, dtype="bf16", s0_std=0.1)
    import torch

    assert db["r"].dtype == torch.bfloat16
    np.testing.assert_array_equal(db["r_f32"].numpy(), db["r"].float().numpy())
    assert abs(float(d["s0"].std()) - 0.1) < 0.02
