"""Float64 CPU oracle for the RWKV-7 (x070) state recurrence -- TEST INFRASTRUCTURE.

Only ``tests/``, ``__graft_entry__.smoke()`` and the CPU-baseline leg of
``bench.py`` may import this package.  The CUDA library never calls it, and it
imports nothing from the CUDA library: the two share only the seeded input
generator ``wkv7_inputs``.

The arithmetic lives in ``wkv7_oracle.c`` (token-by-token definition, see its
header for the passages it follows) and ``wkv7_oracle_bwd.c`` (its gradients by the chain rule:
the pages give no backward, so that file is pinned by finite differences and by torch autograd of
an independent loop, ``tests/test_oracle_backward.py``).  This module compiles it with gcc
(``-O2 -ffp-contract=off``, no fast-math) and wraps it with ctypes.

Pins: every function here is checked by ``tests/test_oracle_pins.py`` against
closed forms, a matrix-product restatement evaluated with numpy, a hand-worked
example, invariances and a long-double build of the same source.
"""

from __future__ import annotations

import ctypes
import os
import subprocess
import threading
from typing import Optional, Tuple

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "wkv7_oracle.c")
_SRC_BWD = os.path.join(_HERE, "wkv7_oracle_bwd.c")
_BUILD = os.path.join(_HERE, "_build")
_LIBS = {"double": "liboracle_wkv7.so", "long double": "liboracle_wkv7_ld.so"}
_lock = threading.Lock()
_loaded = {}


def build(force: bool = False) -> None:
    """Compile both precisions of the oracle library (idempotent)."""
    os.makedirs(_BUILD, exist_ok=True)
    for real, name in _LIBS.items():
        out = os.path.join(_BUILD, name)
        if not force and os.path.exists(out) and os.path.getmtime(out) >= os.path.getmtime(_SRC):
            continue
        tmp = out + ".tmp%d" % os.getpid()
        cmd = ["gcc", "-O2", "-std=c11", "-fPIC", "-shared", "-pthread", "-ffp-contract=off",
               "-fno-fast-math", f"-DORACLE_REAL={real}", _SRC, "-o", tmp]
        subprocess.run(cmd, check=True)
        os.replace(tmp, out)
    out = os.path.join(_BUILD, "liboracle_wkv7_bwd.so")
    if force or not os.path.exists(out) or os.path.getmtime(out) < os.path.getmtime(_SRC_BWD):
        tmp = out + ".tmp%d" % os.getpid()
        subprocess.run(["gcc", "-O2", "-std=c11", "-fPIC", "-shared", "-pthread", "-ffp-contract=off",
                        "-fno-fast-math", _SRC_BWD, "-o", tmp], check=True)
        os.replace(tmp, out)


def _lib(real: str = "double") -> ctypes.CDLL:
    with _lock:
        if real not in _loaded:
            build()
            lib = ctypes.CDLL(os.path.join(_BUILD, _LIBS[real]))
            dp = ctypes.POINTER(ctypes.c_double)
            fp = ctypes.POINTER(ctypes.c_float)
            ci = ctypes.c_int
            lib.wkv7_oracle_f64.argtypes = [ci, ci, ci, ci] + [dp] * 6 + [dp, dp, dp, ci]
            lib.wkv7_oracle_f64.restype = ci
            lib.wkv7_oracle_f32in.argtypes = [ci, ci, ci, ci] + [fp] * 6 + [dp, dp, dp, ci]
            lib.wkv7_oracle_f32in.restype = ci
            lib.wkv7_oracle_real_bytes.restype = ci
            _loaded[real] = lib
        return _loaded[real]


def _lib_bwd() -> ctypes.CDLL:
    with _lock:
        if "bwd" not in _loaded:
            build()
            lib = ctypes.CDLL(os.path.join(_BUILD, "liboracle_wkv7_bwd.so"))
            dp = ctypes.POINTER(ctypes.c_double)
            ci = ctypes.c_int
            lib.wkv7_oracle_bwd_f64.argtypes = [ci, ci, ci, ci] + [dp] * 9 + [dp] * 7 + [ci]
            lib.wkv7_oracle_bwd_f64.restype = ci
            _loaded["bwd"] = lib
        return _loaded["bwd"]


def _as_np(x, dt) -> np.ndarray:
    if hasattr(x, "detach"):  # torch tensor on the CPU
        x = x.detach()
        import torch

        x = x.to(torch.float64 if dt == np.float64 else torch.float32).contiguous().numpy()
    return np.ascontiguousarray(np.asarray(x, dtype=dt))


def default_threads() -> int:
    return max(1, len(os.sched_getaffinity(0)) if hasattr(os, "sched_getaffinity") else os.cpu_count() or 1)


def wkv7(r, w, k, v, a, b, s_in=None, *, nthreads: Optional[int] = None, precision: str = "auto",
         real: str = "double") -> Tuple[np.ndarray, np.ndarray]:
    """Run the recurrence over ``[B, T, H, N]`` operands.

    ``precision``: ``"f32in"`` passes the operands as float32 (exact for fp32 and
    bf16 data), ``"f64"`` as float64; ``"auto"`` keeps float64 arrays as float64
    and everything else as float32.  ``s_in`` is ``[B, H, N, N]`` or None (zero).
    Returns ``(y [B, T, H, N], s_out [B, H, N, N])`` as float64 numpy arrays.
    """
    shp = tuple(r.shape)
    if len(shp) != 4:
        raise ValueError("operands must be [B, T, H, N]")
    B, T, H, N = shp
    for x in (w, k, v, a, b):
        if tuple(x.shape) != shp:
            raise ValueError("operand shapes differ")
    if precision == "auto":
        is64 = getattr(r, "dtype", None) in (np.float64,) or str(getattr(r, "dtype", "")) == "torch.float64"
        precision = "f64" if is64 else "f32in"
    dt = np.float64 if precision == "f64" else np.float32
    ops = [_as_np(x, dt) for x in (r, w, k, v, a, b)]
    sin = None if s_in is None else _as_np(s_in, np.float64)
    if sin is not None and sin.shape != (B, H, N, N):
        raise ValueError("s_in must be [B, H, N, N]")
    y = np.zeros((B, T, H, N), dtype=np.float64)
    s_out = np.zeros((B, H, N, N), dtype=np.float64)
    lib = _lib(real)
    cptr = ctypes.POINTER(ctypes.c_double if dt == np.float64 else ctypes.c_float)
    dp = ctypes.POINTER(ctypes.c_double)
    fn = lib.wkv7_oracle_f64 if dt == np.float64 else lib.wkv7_oracle_f32in
    rc = fn(B, T, H, N, *[o.ctypes.data_as(cptr) for o in ops],
            None if sin is None else sin.ctypes.data_as(dp), y.ctypes.data_as(dp),
            s_out.ctypes.data_as(dp), int(nthreads or default_threads()))
    if rc != 0:
        raise RuntimeError(f"oracle failed with code {rc}")
    return y, s_out


def wkv7_varlen(r, w, k, v, a, b, cu_seqlens, s_in=None, *, nthreads: Optional[int] = None):
    """Ragged batch in packed layout: operands ``[total_T, H, N]``, rows split by
    ``cu_seqlens`` (``B + 1`` offsets).  Each row is an independent sequence.
    Returns ``(y [total_T, H, N], s_out [B, H, N, N])``."""
    cu = [int(x) for x in (cu_seqlens.tolist() if hasattr(cu_seqlens, "tolist") else cu_seqlens)]
    Bn = len(cu) - 1
    total, H, N = tuple(r.shape)
    y = np.zeros((total, H, N), dtype=np.float64)
    s_out = np.zeros((Bn, H, N, N), dtype=np.float64)
    for bi in range(Bn):
        lo, hi = cu[bi], cu[bi + 1]
        sl = [x[lo:hi][None] for x in (r, w, k, v, a, b)]
        si = None if s_in is None else s_in[bi:bi + 1]
        yb, sb = wkv7(*sl, si, nthreads=nthreads)
        y[lo:hi] = yb[0]
        s_out[bi] = sb[0]
    return y, s_out


def x070_prologue(xw, k, xa, k_k) -> Tuple[np.ndarray, np.ndarray, np.ndarray]:
    """The x070 operand prologue in float64 (RWKV-7 G0 7.2B walkthrough, lshu.cn/news/198401,
    section 7.1): the decay comes from its pre-activation as ``exp(-exp(w'))`` with
    ``w' = -softplus(-xw) - 0.5``; the in-context learning rate is ``sigmoid(xa)``; the key is
    scaled by ``k_k`` and L2-normalised over the head (``x / max(||x||, 1e-12)``) into ``kk``; the
    kernel operands are ``a = -kk`` and ``b = kk * sigmoid(xa)``.

    ``xw, k, xa``: ``[..., N]``; ``k_k``: ``[H, N]`` broadcast over the leading dims, or None for
    ones.  Returns float64 ``(w, a, b)`` of the same shape."""
    xw = _as_np(xw, np.float64)
    k = _as_np(k, np.float64)
    xa = _as_np(xa, np.float64)
    softplus_neg = np.log1p(np.exp(-np.abs(-xw))) + np.maximum(-xw, 0.0)  # softplus(-xw), stable form
    w = np.exp(-np.exp(-softplus_neg - 0.5))
    rate = 1.0 / (1.0 + np.exp(-xa))
    kx = k if k_k is None else k * _as_np(k_k, np.float64)
    norm = np.sqrt(np.sum(kx * kx, axis=-1, keepdims=True))
    kk = kx / np.maximum(norm, 1e-12)
    return w, -kk, kk * rate


def wkv7_model_native(r, xw, k, v, xa, k_k, s_in=None, *, nthreads: Optional[int] = None):
    """The recurrence on model-native inputs: the prologue above, then ``wkv7`` in float64
    (``k`` itself enters the recurrence unchanged)."""
    w, a, b = x070_prologue(xw, k, xa, k_k)
    return wkv7(_as_np(r, np.float64), w, _as_np(k, np.float64), _as_np(v, np.float64), a, b, s_in,
                nthreads=nthreads, precision="f64")


LN_EPS = 64e-5  # the GroupNorm eps of the x070 ln_x (the page marks it as not to be changed)


def group_norm_heads(y, ln_w=None, ln_b=None, eps: float = LN_EPS) -> np.ndarray:
    """The x070 ``ln_x`` epilogue in float64 (RWKV-7 G0 7.2B walkthrough, lshu.cn/news/198401, section
    7.1: GroupNorm with eps 64e-5, one group per head): for every token and head, the 64 channels of
    ``y`` minus their mean, divided by ``sqrt(var + eps)`` (variance over the 64 channels, divisor
    64), times ``ln_w`` plus ``ln_b`` (``[H, N]``; None means ones / zeros).  ``y``: ``[..., H, N]``."""
    y = _as_np(y, np.float64)
    mu = y.mean(axis=-1, keepdims=True)
    var = ((y - mu) ** 2).mean(axis=-1, keepdims=True)
    out = (y - mu) / np.sqrt(var + eps)
    if ln_w is not None:
        out = out * _as_np(ln_w, np.float64)
    if ln_b is not None:
        out = out + _as_np(ln_b, np.float64)
    return out


def real_bytes(real: str = "double") -> int:
    return int(_lib(real).wkv7_oracle_real_bytes())


def wkv7_backward(r, w, k, v, a, b, s_in, dy, ds_out=None, *, nthreads: Optional[int] = None):
    """Gradients of ``L = sum <dy, y> + <ds_out, s_out>`` for the recurrence of ``wkv7`` (float64,
    token-by-token chain rule; see ``wkv7_oracle_bwd.c``).  Token tensors ``[B, T, H, N]``, states
    ``[B, H, N, N]``; ``s_in`` / ``ds_out`` None mean zero.  Returns float64 arrays
    ``(dr, dw, dk, dv, da, db, ds_in)``."""
    ops = [_as_np(x, np.float64) for x in (r, w, k, v, a, b)]
    B, T, H, N = ops[0].shape
    dyn = _as_np(dy, np.float64)
    assert dyn.shape == (B, T, H, N)
    s0 = None if s_in is None else _as_np(s_in, np.float64)
    dso = None if ds_out is None else _as_np(ds_out, np.float64)
    outs = [np.zeros((B, T, H, N)) for _ in range(6)]
    ds_in = np.zeros((B, H, N, N))
    dp = ctypes.POINTER(ctypes.c_double)

    def ptr(x):
        return None if x is None else x.ctypes.data_as(dp)

    st = _lib_bwd().wkv7_oracle_bwd_f64(B, T, H, N, *[ptr(x) for x in ops], ptr(s0), ptr(dyn), ptr(dso),
                                        *[ptr(x) for x in outs], ptr(ds_in), int(nthreads or default_threads()))
    if st != 0:
        raise RuntimeError(f"oracle backward failed ({st})")
    return tuple(outs) + (ds_in,)


def round_bf16(x) -> np.ndarray:
    """Round float64 values to the nearest bfloat16 value, ties to even (8 significant bits), as float64.
    For values in bfloat16's normal range (the reduced-precision decode state); zero stays zero."""
    x = np.asarray(x, dtype=np.float64)
    m, e = np.frexp(x)  # x = m * 2^e with 0.5 <= |m| < 1
    return np.ldexp(np.rint(m * 256.0), e - 8)  # np.rint: round half to even


def decode_step_bf16_state(r, w, k, v, a, b, s):
    """One decode step with a bfloat16 state: the recurrence in float64 (``wkv7`` with T = 1) from the
    state values ``s`` ``[B, H, N, N]``, then the new state rounded to bfloat16.  Token operands
    ``[B, H, N]``.  Returns ``(y, s_new)`` as float64."""
    ops = [_as_np(x, np.float64)[:, None] for x in (r, w, k, v, a, b)]
    y, s_new = wkv7(*ops, _as_np(s, np.float64), precision="f64")
    return y[:, 0], round_bf16(s_new)
