"""Pins of the float64 backward oracle (``oracle.wkv7_backward``) against things it does not share:
central finite differences of the forward oracle, torch autograd of an independent token loop,
closed forms of the special case w = 1, a = 0 (where the state is a plain prefix sum), and the
forward oracle run on the reversed sequence with a and b swapped (the adjoint state's recurrence),
which gives dv and ds_in.

The scalar differentiated everywhere is L = sum <dy, y> + <ds_out, s_out>.
"""

import numpy as np
import pytest
import torch

import oracle

NAMES = ("r", "w", "k", "v", "a", "b")


def _draw(B, T, H, N, seed, *, w_one=False, a_zero=False):
    rng = np.random.default_rng(seed)
    x = {n: rng.standard_normal((B, T, H, N)) for n in NAMES}
    x["w"] = np.ones((B, T, H, N)) if w_one else np.exp(-0.6 * rng.random((B, T, H, N)))
    kh = rng.standard_normal((B, T, H, N))
    kh /= np.linalg.norm(kh, axis=-1, keepdims=True)
    x["a"] = np.zeros((B, T, H, N)) if a_zero else -kh
    x["b"] = kh * rng.random((B, T, H, N))
    s0 = 0.3 * rng.standard_normal((B, H, N, N))
    dy = rng.standard_normal((B, T, H, N))
    ds = rng.standard_normal((B, H, N, N))
    return x, s0, dy, ds


def _loss(x, s0, dy, ds):
    y, s = oracle.wkv7(*[x[n] for n in NAMES], s0, precision="f64")
    return float((dy * y).sum() + (ds * s).sum())


def test_every_element_matches_central_differences():
    x, s0, dy, ds = _draw(1, 4, 1, 3, seed=1)
    g = oracle.wkv7_backward(*[x[n] for n in NAMES], s0, dy, ds)
    eps = 1e-6
    for idx, name in enumerate(NAMES + ("s0",)):
        base = s0 if name == "s0" else x[name]
        for pos in np.ndindex(base.shape):
            xp = {n: x[n].copy() for n in NAMES}
            sp, sm = s0.copy(), s0.copy()
            xm = {n: x[n].copy() for n in NAMES}
            if name == "s0":
                sp[pos] += eps
                sm[pos] -= eps
            else:
                xp[name][pos] += eps
                xm[name][pos] -= eps
            fd = (_loss(xp, sp, dy, ds) - _loss(xm, sm, dy, ds)) / (2 * eps)
            assert abs(fd - g[idx][pos]) <= 1e-7 * max(1.0, abs(fd)), (name, pos, fd, g[idx][pos])


@pytest.mark.parametrize("T", [1, 63, 64, 65, 130])
def test_directional_derivatives_across_blocks(T):
    # the oracle recomputes states per 64-token block; lengths around the block size
    x, s0, dy, ds = _draw(2, T, 2, 4, seed=10 + T)
    g = oracle.wkv7_backward(*[x[n] for n in NAMES], s0, dy, ds)
    rng = np.random.default_rng(20 + T)
    eps = 1e-6
    for idx, name in enumerate(NAMES + ("s0",)):
        d = rng.standard_normal(s0.shape if name == "s0" else x[name].shape)
        xp = {n: x[n] + (eps * d if n == name else 0) for n in NAMES}
        xm = {n: x[n] - (eps * d if n == name else 0) for n in NAMES}
        sp = s0 + eps * d if name == "s0" else s0
        sm = s0 - eps * d if name == "s0" else s0
        fd = (_loss(xp, sp, dy, ds) - _loss(xm, sm, dy, ds)) / (2 * eps)
        an = float((g[idx] * d).sum())
        assert abs(fd - an) <= 1e-7 * max(1.0, abs(an)), (name, fd, an)


def test_matches_torch_autograd_of_an_independent_loop():
    B, T, H, N = 2, 9, 2, 5
    x, s0, dy, ds = _draw(B, T, H, N, seed=30)
    tx = {n: torch.tensor(x[n], dtype=torch.float64, requires_grad=True) for n in NAMES}
    ts0 = torch.tensor(s0, dtype=torch.float64, requires_grad=True)
    S = ts0
    ys = []
    for t in range(T):
        r, w, k, v, a, b = [tx[n][:, t] for n in NAMES]  # [B, H, N]
        sa = torch.einsum("bhij,bhj->bhi", S, a)
        S = S * w[:, :, None, :] + sa[..., :, None] * b[:, :, None, :] + v[..., :, None] * k[:, :, None, :]
        ys.append(torch.einsum("bhij,bhj->bhi", S, r))
    y = torch.stack(ys, dim=1)
    L = (torch.tensor(dy) * y).sum() + (torch.tensor(ds) * S).sum()
    L.backward()
    g = oracle.wkv7_backward(*[x[n] for n in NAMES], s0, dy, ds)
    for idx, name in enumerate(NAMES):
        ref = tx[name].grad.numpy()
        assert np.abs(g[idx] - ref).max() <= 1e-12 * max(1.0, np.abs(ref).max()), name
    ref = ts0.grad.numpy()
    assert np.abs(g[6] - ref).max() <= 1e-12 * max(1.0, np.abs(ref).max())


def test_closed_form_when_the_state_is_a_prefix_sum():
    # w = 1 and a = 0: S_t = S0 + sum_{m<=t} v_m k_m^T for any b, and the gradient seen by the state
    # after token t is G_t = ds_out + sum_{u>=t} dy_u r_u^T
    B, T, H, N = 1, 11, 2, 4
    x, s0, dy, ds = _draw(B, T, H, N, seed=40, w_one=True, a_zero=True)
    r, k, v, b = x["r"][0], x["k"][0], x["v"][0], x["b"][0]  # [T, H, N]
    vk = np.einsum("thi,thj->thij", v, k)
    S_after = s0[0][None] + np.cumsum(vk, axis=0)                      # [T, H, N, N]
    S_before = S_after - vk
    dyr = np.einsum("thi,thj->thij", dy[0], r)
    G = ds[0][None] + np.cumsum(dyr[::-1], axis=0)[::-1]                 # [T, H, N, N]
    g = oracle.wkv7_backward(*[x[n] for n in NAMES], s0, dy, ds)
    expect = {
        "r": np.einsum("thij,thi->thj", S_after, dy[0]),
        "k": np.einsum("thij,thi->thj", G, v),
        "v": np.einsum("thij,thj->thi", G, k),
        "w": np.einsum("thij,thij->thj", G, S_before),
        "a": np.einsum("thij,thi->thj", S_before, np.einsum("thij,thj->thi", G, b)),
        "b": np.zeros_like(b),
    }
    for idx, name in enumerate(NAMES):
        assert np.abs(g[idx][0] - expect[name]).max() <= 1e-11 * max(1.0, np.abs(expect[name]).max()), name
    assert np.abs(g[6][0] - G[0]).max() <= 1e-11 * np.abs(G[0]).max()


def test_empty_sequence_passes_the_state_gradient_through():
    x, s0, dy, ds = _draw(1, 0, 2, 4, seed=50)
    g = oracle.wkv7_backward(*[x[n] for n in NAMES], s0, dy, ds)
    assert all(a.size == 0 for a in g[:6])
    assert np.array_equal(g[6], ds)


@pytest.mark.parametrize("T", [1, 5, 70])
def test_adjoint_state_is_the_forward_recurrence_reversed(T):
    # G_t = dL/dS_t obeys G_{t-1} = G_t (diag(w_t) + a_t b_t^T)^T + dy_{t-1} r_{t-1}^T from
    # G_{T-1} = ds_out + dy_{T-1} r_{T-1}^T: the forward recurrence in reverse time with a and b
    # swapped, v := dy and k := r.  Run by the FORWARD oracle with r := k, its outputs are G_t k_t =
    # dv_t and its end state (after one more step with token 0's transition and no injection) is
    # ds_in: two backward outputs from the forward oracle alone.
    x, s0, dy, ds = _draw(2, T, 3, 8, seed=40 + T)
    g = oracle.wkv7_backward(*[x[n] for n in NAMES], s0, dy, ds)
    B, _, H, N = dy.shape
    rev = {n: np.zeros((B, T + 1, H, N)) for n in NAMES}
    rev["w"][:, 0] = 1.0                           # step 0: only the injection dy_{T-1} r_{T-1}^T
    rev["w"][:, 1:] = x["w"][:, ::-1]              # step tau >= 1: transition of token T - tau
    rev["a"][:, 1:] = x["b"][:, ::-1]
    rev["b"][:, 1:] = x["a"][:, ::-1]
    rev["v"][:, :T] = dy[:, ::-1]                  # step tau < T: injection of token T - 1 - tau
    rev["k"][:, :T] = x["r"][:, ::-1]
    rev["r"][:, :T] = x["k"][:, ::-1]              # read-out G_t k_t
    y, s = oracle.wkv7(*[rev[n] for n in NAMES], ds, precision="f64")
    scale = np.abs(g[3]).max()
    np.testing.assert_allclose(y[:, :T][:, ::-1], g[3], atol=1e-12 * scale)   # dv
    np.testing.assert_allclose(s, g[6], atol=1e-12 * np.abs(g[6]).max())      # ds_in
