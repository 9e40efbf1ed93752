"""CPU check of the chunked (WY/UT-form) prefill algebra that the tensor-core
kernel implements, step for step, in float64, against the oracle.

Per chunk of C tokens, with Gamma_t = prod_{u<=t} w_u (within the chunk):

  A~ = a * Gamma_{t-1}, R~ = r * Gamma_t, B^ = b / Gamma_t, K^ = k / Gamma_t
  products   [Mrb Mrk; Lab Lak] = [R~; A~] [B^; K^]^T, causally masked
             (Lab, Lak strictly lower; Mrb, Mrk lower incl. the diagonal)
  inverse    Tinv = (I - Lab)^-1, by 16x16 diagonal blocks then block rows
  WY form    [W~ U~] = Tinv [A~ Lak]
  transition [Q P; E F] = [R~ Mrk; 0 K-^T] + [Mrb; B-^T] [W~ U~]
             with B- = b * Gamma_C / Gamma_t, K- = k * Gamma_C / Gamma_t
  chain      [Y; S_C^T - D S_0^T] = [Q P; E F] [S_0^T; V],  D = diag(Gamma_C)

Tokens past the end of a ragged last chunk are padded with w = 1 and zero
r, k, a, b, v, so they change nothing.
"""

import numpy as np
import pytest

import oracle

C = 64
BLK = 16


def blocked_unit_lower_inverse(L):
    """(I - L)^-1 for strictly lower L (C x C), by diagonal BLK blocks and block rows."""
    n = L.shape[0]
    nb = n // BLK
    T = np.zeros_like(L)
    for s in range(nb):
        sl = slice(BLK * s, BLK * (s + 1))
        Ls = L[sl, sl]
        Ds = np.zeros((BLK, BLK))
        for c in range(BLK):  # column-wise forward substitution
            x = np.zeros(BLK)
            x[c] = 1.0
            for r in range(c + 1, BLK):
                x[r] = Ls[r, c:r] @ x[c:r]
            Ds[:, c] = x
        T[sl, sl] = Ds
    for s in range(1, nb):
        rs = slice(BLK * s, BLK * (s + 1))
        Ds = T[rs, rs]
        for m in range(s):
            cs = slice(BLK * m, BLK * (m + 1))
            Z = L[rs, BLK * m:BLK * s] @ T[BLK * m:BLK * s, cs]
            T[rs, cs] = Ds @ Z
    return T


def chunked_head(r, w, k, v, a, b, s0):
    """r..b: [T, N]; s0: [N, N] (row = value).  Returns y [T, N], s_out [N, N]."""
    T, N = r.shape
    ST = s0.T.copy()
    y = np.zeros((T, N))
    for c0 in range(0, T, C):
        Lc = min(C, T - c0)
        pad = lambda x, fill=0.0: np.concatenate([x[c0:c0 + Lc], np.full((C - Lc, N), fill)], 0)
        rr, kk, vv, aa, bb = (pad(x) for x in (r, k, v, a, b))
        ww = pad(w, 1.0)
        G = np.cumprod(ww, axis=0)
        Gx = np.vstack([np.ones((1, N)), G[:-1]])
        GC = G[-1]
        At, Rt, Bh, Kh = aa * Gx, rr * G, bb / G, kk / G
        D1 = np.vstack([Rt, At]) @ np.vstack([Bh, Kh]).T
        strict = np.tril(np.ones((C, C)), -1)
        incl = np.tril(np.ones((C, C)), 0)
        Mrb, Mrk = D1[:C, :C] * incl, D1[:C, C:] * incl
        Lab, Lak = D1[C:, :C] * strict, D1[C:, C:] * strict
        Tinv = blocked_unit_lower_inverse(Lab)
        WU = Tinv @ np.hstack([At, Lak])
        Bbar, Kbar = bb * (GC / G), kk * (GC / G)
        init = np.vstack([np.hstack([Rt, Mrk]), np.hstack([np.zeros((N, N)), Kbar.T])])
        D2 = init + np.vstack([Mrb, Bbar.T]) @ WU
        D4 = D2 @ np.vstack([ST, vv])
        y[c0:c0 + Lc] = D4[:Lc]
        ST = GC[:, None] * ST + D4[C:]
    return y, ST.T


def test_blocked_inverse_matches_dense_inverse():
    rng = np.random.default_rng(0)
    L = np.tril(rng.standard_normal((C, C)) * 0.2, -1)
    np.testing.assert_allclose(blocked_unit_lower_inverse(L), np.linalg.inv(np.eye(C) - L), atol=1e-10)


@pytest.mark.parametrize("T", [1, 17, 64, 65, 150, 256])
def test_chunk_algebra_matches_oracle(T):
    rng = np.random.default_rng(T)
    N = 64
    r, k, v = (rng.standard_normal((T, N)) for _ in range(3))
    kh = rng.standard_normal((T, N))
    kh /= np.linalg.norm(kh, axis=1, keepdims=True)
    a = -kh
    b = kh * rng.uniform(0, 1, (T, N))
    w = np.exp(-0.606531 / (1 + np.exp(-rng.standard_normal((T, N)) - 1.0)))
    s0 = rng.standard_normal((N, N)) * 0.1
    y, s = chunked_head(r, w, k, v, a, b, s0)
    yo, so = oracle.wkv7(*[x[None, :, None] for x in (r, w, k, v, a, b)], s0[None, None])
    np.testing.assert_allclose(y, yo[0, :, 0], atol=1e-9 * np.abs(yo).max())
    np.testing.assert_allclose(s, so[0, 0], atol=1e-9 * np.abs(so).max())
