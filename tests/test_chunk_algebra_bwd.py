"""CPU check, in float64 against the backward oracle, of a chunked (WY-form) backward: the
reverse-mode derivative of the chunked prefill algebra that the tensor-core forward kernel runs
(the step sequence of ``test_chunk_algebra.chunked_head``), chunk by chunk from the last, so that
a backward kernel can be built from the same dense products.  Per chunk, with X = [S0^T; V],
P = [Mrb; B-^T], Z = [A~ Lak] and the adjoints dY (of y) and dS_C^T (of the end state, transposed):

  chain       dD4 = [dY; dS_C^T];  dS0^T = diag(Gamma_C) dS_C^T + (D2^T dD4)[:N];  dV = (D2^T dD4)[N:]
              dGamma_C += rowsum(dS_C^T .* S0^T);  dD2 = dD4 X^T
  transition  dP = dD2 WU^T;  dWU = P^T dD2;  dinit = dD2 (blocks R~, Mrk, K-^T)
  WY form     dTinv = dWU Z^T;  dZ = Tinv^T dWU;  dLab = Tinv^T dTinv Tinv^T (strictly lower)
  products    dD1 = the masked adjoints of [Mrb Mrk; Lab Lak];  d[R~; A~] = dD1 [B^; K^];
              d[B^; K^] = dD1^T [R~; A~]
  operands    back through A~ = a Gamma_{t-1}, R~ = r Gamma_t, B^ = b / Gamma_t, K^ = k / Gamma_t,
              B-, K- = (b, k) Gamma_C / Gamma_t, and Gamma_t = prod_{u<=t} w_u
              (dw_u = sum_{t>=u} dGamma_t Gamma_t / w_u)

The start state of every chunk comes from a forward pass that keeps the chunk-boundary states (as
the checkpointing forward does).  Eleven dense products per chunk, each of the shapes the forward
kernel already runs on the tensor cores.  Not built as a kernel yet: the training backward runs the
sequential form.
"""

import numpy as np
import pytest

import oracle
from test_chunk_algebra import C, blocked_unit_lower_inverse


def chunk_forward_parts(rr, ww, kk, vv, aa, bb, ST):
    """The forward chunk of ``chunked_head`` (padded C x N operands, ST = S0^T), keeping every
    intermediate the backward needs."""
    N = rr.shape[1]
    G = np.cumprod(ww, axis=0)
    Gx = np.vstack([np.ones((1, N)), G[:-1]])
    GC = G[-1]
    At, Rt, Bh, Kh = aa * Gx, rr * G, bb / G, kk / G
    Lm, Rm = np.vstack([Rt, At]), np.vstack([Bh, Kh])
    D1 = Lm @ Rm.T
    strict = np.tril(np.ones((C, C)), -1)
    incl = np.tril(np.ones((C, C)), 0)
    Mrb, Mrk = D1[:C, :C] * incl, D1[:C, C:] * incl
    Lab, Lak = D1[C:, :C] * strict, D1[C:, C:] * strict
    Tinv = blocked_unit_lower_inverse(Lab)
    Z = np.hstack([At, Lak])
    WU = Tinv @ Z
    Bbar, Kbar = bb * (GC / G), kk * (GC / G)
    init = np.vstack([np.hstack([Rt, Mrk]), np.hstack([np.zeros((N, N)), Kbar.T])])
    P = np.vstack([Mrb, Bbar.T])
    D2 = init + P @ WU
    X = np.vstack([ST, vv])
    D4 = D2 @ X
    return dict(G=G, Gx=Gx, GC=GC, At=At, Rt=Rt, Bh=Bh, Kh=Kh, Lm=Lm, Rm=Rm, Tinv=Tinv, Z=Z, WU=WU, P=P,
                D2=D2, X=X, D4=D4, strict=strict, incl=incl)


def chunk_backward(f, rr, ww, kk, vv, aa, bb, ST, dY, dSTn):
    """Adjoints of one chunk: given dY (C x N) and dSTn (adjoint of S_C^T), returns
    (dr, dw, dk, dv, da, db) (C x N each) and the adjoint of S0^T."""
    N = rr.shape[1]
    G, Gx, GC = f["G"], f["Gx"], f["GC"]
    # chain: D4 = D2 X, S_C^T = diag(GC) S0^T + D4[C:], Y = D4[:C]
    dD4 = np.vstack([dY, dSTn])
    dX = f["D2"].T @ dD4
    dD2 = dD4 @ f["X"].T
    dST = GC[:, None] * dSTn + dX[:N]
    dvv = dX[N:]
    dGC = np.sum(dSTn * ST, axis=1)
    # transition: D2 = init + P WU
    dP = dD2 @ f["WU"].T
    dWU = f["P"].T @ dD2
    dRt = dD2[:C, :N].copy()
    dMrk = dD2[:C, N:].copy()
    dKbar = dD2[C:, N:].T.copy()
    dMrb = dP[:C]
    dBbar = dP[C:].T
    # WY form: WU = Tinv Z, Tinv = (I - Lab)^-1
    Tinv = f["Tinv"]
    dTinv = dWU @ f["Z"].T
    dZ = Tinv.T @ dWU
    dAt = dZ[:, :N].copy()
    dLak = dZ[:, N:]
    dLab = Tinv.T @ dTinv @ Tinv.T
    # products: D1 = Lm Rm^T, masked
    dD1 = np.block([[dMrb * f["incl"], dMrk * f["incl"]], [dLab * f["strict"], dLak * f["strict"]]])
    dLm = dD1 @ f["Rm"]
    dRm = dD1.T @ f["Lm"]
    dRt += dLm[:C]
    dAt += dLm[C:]
    dBh, dKh = dRm[:C], dRm[C:]
    # operands
    drr = dRt * G
    daa = dAt * Gx
    dbb = dBh / G + dBbar * (GC / G)
    dkk = dKh / G + dKbar * (GC / G)
    dG = dRt * rr - (dBh * bb + dKh * kk) / G**2 - (dBbar * bb + dKbar * kk) * GC / G**2
    dGC = dGC + np.sum((dBbar * bb + dKbar * kk) / G, axis=0)
    dG[:-1] += (dAt * aa)[1:]  # Gx[t] = G[t - 1]
    dG[-1] += dGC
    dww = np.cumsum((dG * G)[::-1], axis=0)[::-1] / ww
    return (drr, dww, dkk, dvv, daa, dbb), dST


def chunked_backward_head(r, w, k, v, a, b, s0, dy, ds_out):
    """r..b, dy: [T, N]; s0, ds_out: [N, N].  Returns (dr, dw, dk, dv, da, db, ds_in)."""
    T, N = r.shape
    pad = lambda x, c0, Lc, fill=0.0: np.concatenate([x[c0:c0 + Lc], np.full((C - Lc, N), fill)], 0)
    # forward: the start state of every chunk
    starts, ST = [], s0.T.copy()
    chunks = list(range(0, T, C))
    for c0 in chunks:
        Lc = min(C, T - c0)
        ops = [pad(x, c0, Lc) for x in (r, w, k, v, a, b)]
        ops[1] = pad(w, c0, Lc, 1.0)
        starts.append(ST)
        f = chunk_forward_parts(ops[0], ops[1], ops[2], ops[3], ops[4], ops[5], ST)
        ST = f["GC"][:, None] * ST + f["D4"][C:]
    grads = [np.zeros((T, N)) for _ in range(6)]
    dSTn = ds_out.T.copy()
    for c0, ST0 in zip(reversed(chunks), reversed(starts)):
        Lc = min(C, T - c0)
        rr, kk, vv, aa, bb = (pad(x, c0, Lc) for x in (r, k, v, a, b))
        ww = pad(w, c0, Lc, 1.0)
        f = chunk_forward_parts(rr, ww, kk, vv, aa, bb, ST0)
        g, dSTn = chunk_backward(f, rr, ww, kk, vv, aa, bb, ST0, pad(dy, c0, Lc), dSTn)
        for i in range(6):
            grads[i][c0:c0 + Lc] = g[i][:Lc]
    return tuple(grads) + (dSTn.T,)


def _inputs(T, seed, N=64):
    rng = np.random.default_rng(seed)
    r, k, v = (rng.standard_normal((T, N)) for _ in range(3))
    kh = rng.standard_normal((T, N))
    kh /= np.linalg.norm(kh, axis=1, keepdims=True)
    a = -kh
    b = kh * rng.uniform(0, 1, (T, N))
    w = np.exp(-0.606531 / (1 + np.exp(-rng.standard_normal((T, N)) - 1.0)))
    s0 = rng.standard_normal((N, N)) * 0.1
    dy = rng.standard_normal((T, N))
    ds_out = rng.standard_normal((N, N)) * 0.1
    return r, w, k, v, a, b, s0, dy, ds_out


@pytest.mark.parametrize("T", [1, 30, 64, 65, 150])
def test_chunked_backward_matches_the_backward_oracle(T):
    r, w, k, v, a, b, s0, dy, ds_out = _inputs(T, seed=200 + T)
    got = chunked_backward_head(r, w, k, v, a, b, s0, dy, ds_out)
    ref = oracle.wkv7_backward(*[x[None, :, None] for x in (r, w, k, v, a, b)], s0[None, None], dy[None, :, None],
                               ds_out[None, None])
    names = ("dr", "dw", "dk", "dv", "da", "db")
    for i, n in enumerate(names):
        scale = np.abs(ref[i]).max()
        np.testing.assert_allclose(got[i], ref[i][0, :, 0], atol=1e-9 * scale, err_msg=n)
    np.testing.assert_allclose(got[6], ref[6][0, 0], atol=1e-9 * np.abs(ref[6]).max(), err_msg="ds_in")
