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

The second part fixes the operand precision of those products for such a kernel, by emulating the
rounding of each product's operands (tf32 or bf16) on bf16 inputs: every product in bf16 misses the
5e-3 bar; the inverse's adjoint (dTinv, both dLab products) and dD2 in bf16 with the rest, and the
recomputed forward products, in tf32 stay within 2.5e-3.
"""

import numpy as np
import pytest

import oracle
from test_chunk_algebra import C, blocked_unit_lower_inverse


def exact(name, a, b):
    return a @ b


def chunk_forward_parts(rr, ww, kk, vv, aa, bb, ST, mm=exact):
    """The forward chunk of ``chunked_head`` (padded C x N operands, ST = S0^T), keeping every
    intermediate the backward needs.  ``mm(name, a, b)`` forms each matrix product."""
    N = rr.shape[1]
    G = np.cumprod(ww, axis=0)
    Gx = np.vstack([np.ones((1, N)), G[:-1]])
    GC = G[-1]
    At, Rt, Bh, Kh = aa * Gx, rr * G, bb / G, kk / G
    Lm, Rm = np.vstack([Rt, At]), np.vstack([Bh, Kh])
    D1 = mm("MMA1", Lm, Rm.T)
    strict = np.tril(np.ones((C, C)), -1)
    incl = np.tril(np.ones((C, C)), 0)
    Mrb, Mrk = D1[:C, :C] * incl, D1[:C, C:] * incl
    Lab, Lak = D1[C:, :C] * strict, D1[C:, C:] * strict
    Tinv = blocked_unit_lower_inverse(Lab)
    Z = np.hstack([At, Lak])
    WU = mm("MMA3", Tinv, Z)
    Bbar, Kbar = bb * (GC / G), kk * (GC / G)
    init = np.vstack([np.hstack([Rt, Mrk]), np.hstack([np.zeros((N, N)), Kbar.T])])
    P = np.vstack([Mrb, Bbar.T])
    D2 = init + mm("MMA2", P, WU)
    X = np.vstack([ST, vv])
    D4 = mm("MMA4", D2, X)
    return dict(G=G, Gx=Gx, GC=GC, At=At, Rt=Rt, Bh=Bh, Kh=Kh, Lm=Lm, Rm=Rm, Tinv=Tinv, Z=Z, WU=WU, P=P,
                D2=D2, X=X, D4=D4, strict=strict, incl=incl)


def chunk_backward(f, rr, ww, kk, vv, aa, bb, ST, dY, dSTn, mm=exact):
    """Adjoints of one chunk: given dY (C x N) and dSTn (adjoint of S_C^T), returns
    (dr, dw, dk, dv, da, db) (C x N each) and the adjoint of S0^T."""
    N = rr.shape[1]
    G, Gx, GC = f["G"], f["Gx"], f["GC"]
    # chain: D4 = D2 X, S_C^T = diag(GC) S0^T + D4[C:], Y = D4[:C]
    dD4 = np.vstack([dY, dSTn])
    dX = mm("dX", f["D2"].T, dD4)
    dD2 = mm("dD2", dD4, f["X"].T)
    dST = GC[:, None] * dSTn + dX[:N]
    dvv = dX[N:]
    dGC = np.sum(dSTn * ST, axis=1)
    # transition: D2 = init + P WU
    dP = mm("dP", dD2, f["WU"].T)
    dWU = mm("dWU", f["P"].T, dD2)
    dRt = dD2[:C, :N].copy()
    dMrk = dD2[:C, N:].copy()
    dKbar = dD2[C:, N:].T.copy()
    dMrb = dP[:C]
    dBbar = dP[C:].T
    # WY form: WU = Tinv Z, Tinv = (I - Lab)^-1
    Tinv = f["Tinv"]
    dTinv = mm("dTinv", dWU, f["Z"].T)
    dZ = mm("dZ", Tinv.T, dWU)
    dAt = dZ[:, :N].copy()
    dLak = dZ[:, N:]
    dLab = mm("dLab2", mm("dLab1", Tinv.T, dTinv), Tinv.T)
    # products: D1 = Lm Rm^T, masked
    dD1 = np.block([[dMrb * f["incl"], dMrk * f["incl"]], [dLab * f["strict"], dLak * f["strict"]]])
    dLm = mm("dLm", dD1, f["Rm"])
    dRm = mm("dRm", dD1.T, f["Lm"])
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


def chunked_backward_head(r, w, k, v, a, b, s0, dy, ds_out, mm=exact):
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
        f = chunk_forward_parts(ops[0], ops[1], ops[2], ops[3], ops[4], ops[5], ST, mm)
        ST = f["GC"][:, None] * ST + f["D4"][C:]
    grads = [np.zeros((T, N)) for _ in range(6)]
    dSTn = ds_out.T.copy()
    for c0, ST0 in zip(reversed(chunks), reversed(starts)):
        Lc = min(C, T - c0)
        rr, kk, vv, aa, bb = (pad(x, c0, Lc) for x in (r, k, v, a, b))
        ww = pad(w, c0, Lc, 1.0)
        f = chunk_forward_parts(rr, ww, kk, vv, aa, bb, ST0, mm)
        g, dSTn = chunk_backward(f, rr, ww, kk, vv, aa, bb, ST0, pad(dy, c0, Lc), dSTn, mm)
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


# ---- operand precision of the products (plan for a tensor-core backward) ----------------------------

def round_operand(x, fmt):
    """Round to tf32 (10 explicit mantissa bits) or bf16 (7), to nearest even, via float32."""
    if fmt == "f64":
        return x
    u = np.asarray(x, dtype=np.float32).view(np.uint32).astype(np.uint64)
    drop = 13 if fmt == "tf32" else 16
    u = (u + ((1 << (drop - 1)) - 1) + ((u >> drop) & 1)) >> drop << drop
    return u.astype(np.uint32).view(np.float32).astype(np.float64)


def rounding_mm(plan):
    return lambda name, a, b: round_operand(a, plan[name]) @ round_operand(b, plan[name])


BWD = ("dX", "dD2", "dP", "dWU", "dTinv", "dZ", "dLab1", "dLab2", "dLm", "dRm")


def _worst_rel_err(plan, T=256, seeds=(1, 2)):
    worst = 0.0
    for seed in seeds:
        r, w, k, v, a, b, s0, dy, ds_out = _inputs(T, seed)
        r, w, k, v, a, b, dy = (round_operand(x, "bf16") for x in (r, w, k, v, a, b, dy))  # bf16 operands
        ref = oracle.wkv7_backward(*[x[None, :, None] for x in (r, w, k, v, a, b)], s0[None, None],
                                   dy[None, :, None], ds_out[None, None])
        got = chunked_backward_head(r, w, k, v, a, b, s0, dy, ds_out, rounding_mm(plan))
        for i in range(7):
            rr = ref[i][0, :, 0] if i < 6 else ref[6][0, 0]
            worst = max(worst, float(np.abs(got[i] - rr).max() / np.abs(rr).max()))
    return worst


def test_product_precision_plan():
    # the forward products recomputed at tf32; of the backward's, the inverse's adjoint (dTinv and
    # both dLab products) and dD2 in bf16, the rest in tf32: within the 5e-3 bar of bf16 operands with
    # margin, while every product in bf16 is not (the column-sum products dLm, dRm need tf32)
    fwd = {"MMA1": "tf32", "MMA3": "tf32", "MMA2": "tf32", "MMA4": "tf32"}
    plan = dict(fwd, **{n: "tf32" for n in BWD})
    plan.update({n: "bf16" for n in ("dTinv", "dLab1", "dLab2", "dD2")})
    assert _worst_rel_err(plan) <= 2.5e-3
    assert _worst_rel_err(dict(fwd, **{n: "bf16" for n in BWD})) > 5e-3
