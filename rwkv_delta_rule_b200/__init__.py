"""Python binding of the RWKV-7 (x070) state-recurrence library ``librwkv7.so``.

Argument marshalling only: every function here checks tensor shapes, dtypes
and devices, passes raw device pointers and the current CUDA stream to the
``extern "C"`` entry point of the same name (declared in ``include/rwkv7.h``)
and raises on a non-OK status.  All computation happens in the CUDA kernels.
There is no CPU fallback: if the library is missing, importing the entry
points raises.

The recurrence (RWKV-7 G0 7.2B walkthrough, lshu.cn/news/198401, section 7.1),
per batch row b and head h, with a float32 64 x 64 state S:

    sa = S a_t;   S = S diag(w_t) + sa b_t^T + v_t k_t^T;   y_t = S r_t
"""

from __future__ import annotations

import ctypes
import os
from typing import Optional

import torch

__all__ = [
    "RWKV7_PATH_AUTO", "RWKV7_PATH_SCAN", "RWKV7_PATH_CHUNK", "RWKV7_SCHED_AUTO", "RWKV7_SCHED_PAIR",
    "RWKV7_SCHED_TASKS", "RWKV7_SCHED_PIPE", "Rwkv7Error", "library_path", "load_library",
    "rwkv7_wkv_prefill", "rwkv7_wkv_prefill_bf16", "rwkv7_wkv_prefill_bf16_path", "rwkv7_wkv_prefill_varlen_bf16",
    "rwkv7_wkv_decode", "rwkv7_wkv_decode_bf16", "rwkv7_wkv_prefill_fused_bf16", "rwkv7_wkv_decode_fused_bf16",
    "rwkv7_wkv_prefill_ext_bf16", "rwkv7_wkv_decode_ext_bf16", "Options",
    "rwkv7_status_string", "rwkv7_get_last_error", "rwkv7_version", "rwkv7_test_set_wait_hooks",
    "rwkv7_wkv_prefill_save_bf16", "rwkv7_wkv_backward_bf16", "rwkv7_wkv_decode_bf16_bf16state",
    "rwkv7_wkv_decode_ext_bf16state",
    "rwkv7_wkv_prefill_host_bf16", "rwkv7_wkv_prefill_host_noalloc_bf16", "NOALLOC_STAGING_BYTES", "prefill", "decode_", "prefill_model_native", "decode_model_native_", "prefill_ext", "decode_ext_",
    "prefill_save", "backward", "EXPORTED_SYMBOLS",
]

RWKV7_PATH_AUTO, RWKV7_PATH_SCAN, RWKV7_PATH_CHUNK = 0, 1, 2
# chunk-path schedules (rwkv7_options.chunk_schedule)
RWKV7_SCHED_AUTO, RWKV7_SCHED_PAIR, RWKV7_SCHED_TASKS, RWKV7_SCHED_PIPE = 0, 1, 2, 3
N_HEAD = 64

EXPORTED_SYMBOLS = (
    "rwkv7_wkv_prefill", "rwkv7_wkv_prefill_bf16", "rwkv7_wkv_prefill_bf16_path", "rwkv7_wkv_prefill_varlen_bf16",
    "rwkv7_wkv_decode", "rwkv7_wkv_decode_bf16", "rwkv7_wkv_prefill_fused_bf16", "rwkv7_wkv_decode_fused_bf16",
    "rwkv7_wkv_prefill_ext_bf16", "rwkv7_wkv_decode_ext_bf16",
    "rwkv7_wkv_prefill_save_bf16", "rwkv7_wkv_backward_bf16", "rwkv7_wkv_decode_bf16_bf16state",
    "rwkv7_wkv_prefill_host_bf16", "rwkv7_status_string", "rwkv7_get_last_error", "rwkv7_version",
    "rwkv7_wkv_prefill_host_noalloc_bf16", "rwkv7_test_set_wait_hooks", "rwkv7_wkv_decode_ext_bf16state",
)
# RWKV7_NOALLOC_STAGING_BYTES of include/rwkv7.h: the staging limit of rwkv7_wkv_prefill_host_noalloc_bf16
NOALLOC_STAGING_BYTES = 32 * 1024 * 1024

_HERE = os.path.dirname(os.path.abspath(__file__))
_lib: Optional[ctypes.CDLL] = None


class Options(ctypes.Structure):
    """``rwkv7_options`` of include/rwkv7.h (host struct; the pointers are device addresses)."""

    _fields_ = [("model_native", ctypes.c_int), ("k_k", ctypes.c_void_p), ("group_norm", ctypes.c_int),
                ("ln_w", ctypes.c_void_p), ("ln_b", ctypes.c_void_p), ("chunk_schedule", ctypes.c_int),
                ("independent_state", ctypes.c_int)]


class Rwkv7Error(RuntimeError):
    def __init__(self, fn: str, status: int):
        super().__init__(f"{fn}: {rwkv7_status_string(status)} (status {status})")
        self.status = status


def library_path() -> str:
    return os.path.join(_HERE, "librwkv7.so")


def load_library() -> ctypes.CDLL:
    """Load ``librwkv7.so`` (built in-tree by ``rwkv_delta_rule_b200.build``)."""
    global _lib
    if _lib is not None:
        return _lib
    path = library_path()
    if not os.path.exists(path):
        raise RuntimeError(f"librwkv7.so not built ({path}); run `python -m rwkv_delta_rule_b200.build`")
    lib = ctypes.CDLL(path)
    vp, ci = ctypes.c_void_p, ctypes.c_int
    pre = [ci, ci, ci, ci] + [vp] * 6 + [vp, vp, vp, vp]
    for name, args in (
        ("rwkv7_wkv_prefill", pre),
        ("rwkv7_wkv_prefill_bf16", pre),
        ("rwkv7_wkv_prefill_bf16_path", [ci] + pre),
        ("rwkv7_wkv_prefill_varlen_bf16", [ci, ci, ci, ci, ci, ci, vp] + [vp] * 6 + [vp, vp, vp, vp]),
        ("rwkv7_wkv_decode", [ci, ci, ci] + [vp] * 6 + [vp, vp, vp]),
        ("rwkv7_wkv_decode_bf16", [ci, ci, ci] + [vp] * 6 + [vp, vp, vp]),
        ("rwkv7_wkv_prefill_fused_bf16", [ci, ci, ci, ci, ci] + [vp] * 6 + [vp, vp, vp, vp]),
        ("rwkv7_wkv_decode_fused_bf16", [ci, ci, ci] + [vp] * 6 + [vp, vp, vp]),
        ("rwkv7_wkv_prefill_ext_bf16", [ci, ci, ci, ci, ci] + [vp] * 6 + [ctypes.POINTER(Options), vp, vp, vp, vp]),
        ("rwkv7_wkv_decode_ext_bf16", [ci, ci, ci] + [vp] * 6 + [ctypes.POINTER(Options), vp, vp, vp]),
        ("rwkv7_wkv_prefill_save_bf16", [ci, ci, ci, ci, ci] + [vp] * 6 + [vp, vp, vp, vp, vp]),
        ("rwkv7_wkv_backward_bf16", [ci, ci, ci, ci] + [vp] * 6 + [vp, vp, vp] + [vp] * 7 + [vp]),
        ("rwkv7_wkv_decode_bf16_bf16state", [ci, ci, ci] + [vp] * 6 + [vp, vp, vp]),
        ("rwkv7_wkv_decode_ext_bf16state", [ci, ci, ci] + [vp] * 6 + [ctypes.POINTER(Options), vp, vp, vp]),
        ("rwkv7_wkv_prefill_host_bf16", [ci, ci, ci, ci, ci] + [vp] * 6 + [vp, vp, vp] + [vp] * 6 + [vp, vp, vp]
         + [ci, vp]),
        ("rwkv7_wkv_prefill_host_noalloc_bf16", [ci] + pre),
    ):
        fn = getattr(lib, name)
        fn.argtypes = args
        fn.restype = ci
    lib.rwkv7_status_string.argtypes = [ci]
    lib.rwkv7_status_string.restype = ctypes.c_char_p
    lib.rwkv7_get_last_error.argtypes = []
    lib.rwkv7_get_last_error.restype = ci
    lib.rwkv7_version.argtypes = []
    lib.rwkv7_version.restype = ci
    lib.rwkv7_test_set_wait_hooks.argtypes = [ctypes.c_uint, ctypes.c_longlong]
    lib.rwkv7_test_set_wait_hooks.restype = ci
    _lib = lib
    return lib


# ---- marshalling helpers ------------------------------------------------------------------------

def _ptr(t: Optional[torch.Tensor]) -> Optional[int]:
    return None if t is None else t.data_ptr()


def _stream(stream) -> Optional[int]:
    if stream is None:
        return torch.cuda.current_stream().cuda_stream
    if isinstance(stream, torch.cuda.Stream):
        return stream.cuda_stream
    return int(stream)


def _check_host(t: torch.Tensor, name: str, dtype: torch.dtype, shape):
    if t is None:
        raise ValueError(f"{name} is required")
    if t.is_cuda:
        raise ValueError(f"{name} must be a host (CPU) tensor")
    if t.dtype != dtype or not t.is_contiguous() or tuple(t.shape) != tuple(shape):
        raise ValueError(f"{name} must be a contiguous {dtype} tensor of shape {tuple(shape)}")


def _check(t: Optional[torch.Tensor], name: str, dtype: torch.dtype, shape=None, allow_none=False):
    if t is None:
        if allow_none:
            return
        raise ValueError(f"{name} is required")
    if not t.is_cuda:
        raise ValueError(f"{name} must be a CUDA tensor")
    if t.dtype != dtype:
        raise ValueError(f"{name} must be {dtype}, got {t.dtype}")
    if not t.is_contiguous():
        raise ValueError(f"{name} must be contiguous")
    if shape is not None and tuple(t.shape) != tuple(shape):
        raise ValueError(f"{name} must have shape {tuple(shape)}, got {tuple(t.shape)}")


def _call(name: str, *args) -> None:
    st = getattr(load_library(), name)(*args)
    if st != 0:
        raise Rwkv7Error(name, st)


def _prefill_common(name, dtype, r, w, k, v, a, b, s_in, y, s_out, stream, path=None):
    B, T, H, N = r.shape
    for nm, t in (("r", r), ("w", w), ("k", k), ("v", v), ("a", a), ("b", b), ("y", y)):
        _check(t, nm, dtype, (B, T, H, N))
    _check(s_in, "s_in", torch.float32, (B, H, N, N), allow_none=True)
    _check(s_out, "s_out", torch.float32, (B, H, N, N))
    args = [B, T, H, N] + [_ptr(t) for t in (r, w, k, v, a, b, s_in, y, s_out)] + [_stream(stream)]
    if path is not None:
        args = [int(path)] + args
    _call(name, *args)


# ---- entry points (same names as the C ABI) --------------------------------------------------------

def rwkv7_wkv_prefill(r, w, k, v, a, b, s_in, y, s_out, stream=None) -> None:
    """float32 prefill: operands / y ``[B,T,H,64]``, states ``[B,H,64,64]`` (s_in may be None)."""
    _prefill_common("rwkv7_wkv_prefill", torch.float32, r, w, k, v, a, b, s_in, y, s_out, stream)


def rwkv7_wkv_prefill_bf16(r, w, k, v, a, b, s_in, y, s_out, stream=None) -> None:
    """bfloat16 prefill (kernel chosen by the library), float32 states."""
    _prefill_common("rwkv7_wkv_prefill_bf16", torch.bfloat16, r, w, k, v, a, b, s_in, y, s_out, stream)


def rwkv7_wkv_prefill_bf16_path(path, r, w, k, v, a, b, s_in, y, s_out, stream=None) -> None:
    """bfloat16 prefill with an explicit kernel (RWKV7_PATH_SCAN or RWKV7_PATH_CHUNK)."""
    _prefill_common("rwkv7_wkv_prefill_bf16_path", torch.bfloat16, r, w, k, v, a, b, s_in, y, s_out, stream,
                    path=path)


def rwkv7_wkv_prefill_host_bf16(path, r, w, k, v, a, b, s_in, y, s_out, dev, slices=0, stream=None) -> None:
    """bfloat16 prefill from and to host memory: r .. b, s_in (or None), y and s_out are CPU tensors
    (page-locked for the copies to overlap); ``dev`` maps "r", "w", "k", "v", "a", "b", "s_in" (when
    s_in is given), "y", "s_out" to CUDA staging tensors of the same shapes.  The call queues the
    sliced copies and launches on ``stream``; synchronise it before reading y / s_out."""
    B, T, H, N = r.shape
    for nm, t in (("r", r), ("w", w), ("k", k), ("v", v), ("a", a), ("b", b), ("y", y)):
        _check_host(t, nm, torch.bfloat16, (B, T, H, N))
        _check(dev[nm], "dev " + nm, torch.bfloat16, (B, T, H, N))
    _check_host(s_out, "s_out", torch.float32, (B, H, N, N))
    _check(dev["s_out"], "dev s_out", torch.float32, (B, H, N, N))
    if s_in is not None:
        _check_host(s_in, "s_in", torch.float32, (B, H, N, N))
        _check(dev["s_in"], "dev s_in", torch.float32, (B, H, N, N))
    dsi = dev["s_in"] if s_in is not None else None
    _call("rwkv7_wkv_prefill_host_bf16", int(path), B, T, H, N, *[_ptr(t) for t in (r, w, k, v, a, b, s_in, y, s_out)],
          *[_ptr(dev[n]) for n in ("r", "w", "k", "v", "a", "b")], _ptr(dsi), _ptr(dev["y"]), _ptr(dev["s_out"]),
          int(slices), _stream(stream))


def rwkv7_wkv_prefill_host_noalloc_bf16(path, r, w, k, v, a, b, s_in, y, s_out, stream=None) -> None:
    """bfloat16 prefill from and to host memory that allocates nothing: r .. b, s_in (or None), y and
    s_out are CPU tensors, staged through the library's static device array (at most
    ``NOALLOC_STAGING_BYTES`` per call).  For callers that cannot allocate device memory.  Queued on
    ``stream``; synchronise it before reading y / s_out."""
    B, T, H, N = r.shape
    for nm, t in (("r", r), ("w", w), ("k", k), ("v", v), ("a", a), ("b", b), ("y", y)):
        _check_host(t, nm, torch.bfloat16, (B, T, H, N))
    _check_host(s_out, "s_out", torch.float32, (B, H, N, N))
    if s_in is not None:
        _check_host(s_in, "s_in", torch.float32, (B, H, N, N))
    _call("rwkv7_wkv_prefill_host_noalloc_bf16", int(path), B, T, H, N,
          *[_ptr(t) for t in (r, w, k, v, a, b, s_in, y, s_out)], _stream(stream))


def rwkv7_wkv_prefill_varlen_bf16(path, cu_seqlens, max_T, r, w, k, v, a, b, s_in, y, s_out, stream=None) -> None:
    """Ragged bfloat16 prefill: operands / y ``[total_T,H,64]`` packed, ``cu_seqlens`` int32 ``[B+1]`` on the
    device, states ``[B,H,64,64]``."""
    total, H, N = r.shape
    Bn = cu_seqlens.numel() - 1
    _check(cu_seqlens, "cu_seqlens", torch.int32, (Bn + 1,))
    for nm, t in (("r", r), ("w", w), ("k", k), ("v", v), ("a", a), ("b", b), ("y", y)):
        _check(t, nm, torch.bfloat16, (total, H, N))
    _check(s_in, "s_in", torch.float32, (Bn, H, N, N), allow_none=True)
    _check(s_out, "s_out", torch.float32, (Bn, H, N, N))
    _call("rwkv7_wkv_prefill_varlen_bf16", int(path), Bn, total, int(max_T), H, N, _ptr(cu_seqlens),
          *[_ptr(t) for t in (r, w, k, v, a, b, s_in, y, s_out)], _stream(stream))


def _decode_common(name, dtype, r, w, k, v, a, b, s_inout, y, stream):
    B, H, N = r.shape
    for nm, t in (("r", r), ("w", w), ("k", k), ("v", v), ("a", a), ("b", b), ("y", y)):
        _check(t, nm, dtype, (B, H, N))
    _check(s_inout, "s_inout", torch.float32, (B, H, N, N))
    _call(name, B, H, N, *[_ptr(t) for t in (r, w, k, v, a, b, s_inout, y)], _stream(stream))


def rwkv7_wkv_decode(r, w, k, v, a, b, s_inout, y, stream=None) -> None:
    """float32 one-token step: operands / y ``[B,H,64]``, state ``[B,H,64,64]`` updated in place."""
    _decode_common("rwkv7_wkv_decode", torch.float32, r, w, k, v, a, b, s_inout, y, stream)


def rwkv7_wkv_decode_bf16(r, w, k, v, a, b, s_inout, y, stream=None) -> None:
    """bfloat16 one-token step, float32 state updated in place."""
    _decode_common("rwkv7_wkv_decode_bf16", torch.bfloat16, r, w, k, v, a, b, s_inout, y, stream)


def rwkv7_wkv_prefill_fused_bf16(path, r, xw, k, v, xa, k_k, s_in, y, s_out, stream=None) -> None:
    """Prefill on model-native inputs: bf16 ``r, xw, k, v, xa`` / y ``[B,T,H,64]``, float32 ``k_k``
    ``[H,64]`` or None (ones); w, a and b are formed in the kernels."""
    B, T, H, N = r.shape
    for nm, t in (("r", r), ("xw", xw), ("k", k), ("v", v), ("xa", xa), ("y", y)):
        _check(t, nm, torch.bfloat16, (B, T, H, N))
    _check(k_k, "k_k", torch.float32, (H, N), allow_none=True)
    _check(s_in, "s_in", torch.float32, (B, H, N, N), allow_none=True)
    _check(s_out, "s_out", torch.float32, (B, H, N, N))
    _call("rwkv7_wkv_prefill_fused_bf16", int(path), B, T, H, N,
          *[_ptr(t) for t in (r, xw, k, v, xa, k_k, s_in, y, s_out)], _stream(stream))


def rwkv7_wkv_decode_fused_bf16(r, xw, k, v, xa, k_k, s_inout, y, stream=None) -> None:
    """One decode step on model-native inputs ``[B,H,64]`` (bf16), ``k_k`` ``[H,64]`` float32 or None."""
    B, H, N = r.shape
    for nm, t in (("r", r), ("xw", xw), ("k", k), ("v", v), ("xa", xa), ("y", y)):
        _check(t, nm, torch.bfloat16, (B, H, N))
    _check(k_k, "k_k", torch.float32, (H, N), allow_none=True)
    _check(s_inout, "s_inout", torch.float32, (B, H, N, N))
    _call("rwkv7_wkv_decode_fused_bf16", B, H, N, *[_ptr(t) for t in (r, xw, k, v, xa, k_k, s_inout, y)],
          _stream(stream))


def _options(model_native: bool, k_k, group_norm: bool, ln_w, ln_b, H: int, N: int, schedule: int = 0,
             independent_state: bool = False) -> Options:
    if model_native:
        _check(k_k, "k_k", torch.float32, (H, N), allow_none=True)
    if group_norm:
        _check(ln_w, "ln_w", torch.float32, (H, N), allow_none=True)
        _check(ln_b, "ln_b", torch.float32, (H, N), allow_none=True)
    return Options(int(bool(model_native)), _ptr(k_k) if model_native else None, int(bool(group_norm)),
                   _ptr(ln_w) if group_norm else None, _ptr(ln_b) if group_norm else None, int(schedule),
                   int(bool(independent_state)))


def rwkv7_wkv_prefill_ext_bf16(path, r, w, k, v, a, b, s_in, y, s_out, *, model_native=False, k_k=None,
                               group_norm=False, ln_w=None, ln_b=None, schedule=0, stream=None) -> None:
    """bf16 prefill with options: model-native inputs (``w``, ``a`` hold x_w, x_a; ``b`` None), the
    ln_x GroupNorm epilogue on ``y`` (``ln_w`` / ``ln_b`` ``[H,64]`` float32 or None), and the chunk
    path's schedule (``RWKV7_SCHED_*``)."""
    B, T, H, N = r.shape
    names = (("r", r), ("w", w), ("k", k), ("v", v), ("a", a), ("y", y)) + (() if model_native else (("b", b),))
    for nm, t in names:
        _check(t, nm, torch.bfloat16, (B, T, H, N))
    _check(s_in, "s_in", torch.float32, (B, H, N, N), allow_none=True)
    _check(s_out, "s_out", torch.float32, (B, H, N, N))
    opt = _options(model_native, k_k, group_norm, ln_w, ln_b, H, N, schedule)
    _call("rwkv7_wkv_prefill_ext_bf16", int(path), B, T, H, N,
          *[_ptr(t) for t in (r, w, k, v, a, None if model_native else b)], ctypes.byref(opt),
          _ptr(s_in), _ptr(y), _ptr(s_out), _stream(stream))


def rwkv7_wkv_decode_ext_bf16(r, w, k, v, a, b, s_inout, y, *, model_native=False, k_k=None, group_norm=False,
                              ln_w=None, ln_b=None, independent_state=False, stream=None) -> None:
    """bf16 decode step with options (see ``rwkv7_wkv_prefill_ext_bf16``); ``independent_state``: no step
    still running before this one on the stream writes this step's state (``rwkv7_options``), so the
    state loads may start before the previous step has finished."""
    B, H, N = r.shape
    names = (("r", r), ("w", w), ("k", k), ("v", v), ("a", a), ("y", y)) + (() if model_native else (("b", b),))
    for nm, t in names:
        _check(t, nm, torch.bfloat16, (B, H, N))
    _check(s_inout, "s_inout", torch.float32, (B, H, N, N))
    opt = _options(model_native, k_k, group_norm, ln_w, ln_b, H, N, independent_state=independent_state)
    _call("rwkv7_wkv_decode_ext_bf16", B, H, N, *[_ptr(t) for t in (r, w, k, v, a, None if model_native else b)],
          ctypes.byref(opt), _ptr(s_inout), _ptr(y), _stream(stream))


def rwkv7_wkv_decode_bf16_bf16state(r, w, k, v, a, b, s_inout, y, stream=None) -> None:
    """One decode step with the state stored as bfloat16 ``[B, H, 64, 64]`` (updated in place)."""
    B, H, N = r.shape
    for nm, t in (("r", r), ("w", w), ("k", k), ("v", v), ("a", a), ("b", b), ("y", y)):
        _check(t, nm, torch.bfloat16, (B, H, N))
    _check(s_inout, "s_inout", torch.bfloat16, (B, H, N, N))
    _call("rwkv7_wkv_decode_bf16_bf16state", B, H, N, *[_ptr(t) for t in (r, w, k, v, a, b, s_inout, y)],
          _stream(stream))


def rwkv7_wkv_decode_ext_bf16state(r, w, k, v, a, b, s_inout, y, *, independent_state=False, stream=None) -> None:
    """``rwkv7_wkv_decode_bf16_bf16state`` with options: ``independent_state`` as for
    ``rwkv7_wkv_decode_ext_bf16``."""
    B, H, N = r.shape
    for nm, t in (("r", r), ("w", w), ("k", k), ("v", v), ("a", a), ("b", b), ("y", y)):
        _check(t, nm, torch.bfloat16, (B, H, N))
    _check(s_inout, "s_inout", torch.bfloat16, (B, H, N, N))
    opt = Options(0, None, 0, None, None, 0, int(bool(independent_state)))
    _call("rwkv7_wkv_decode_ext_bf16state", B, H, N, *[_ptr(t) for t in (r, w, k, v, a, b)], ctypes.byref(opt),
          _ptr(s_inout), _ptr(y), _stream(stream))


def n_checkpoints(T: int) -> int:
    """Saved states per (b, h) of ``rwkv7_wkv_prefill_save_bf16``: one before every 64th token."""
    return (int(T) + 63) // 64


def rwkv7_wkv_prefill_save_bf16(r, w, k, v, a, b, s_in, y, s_out, states, stream=None, *,
                                path: int = RWKV7_PATH_AUTO) -> None:
    """bf16 prefill that also writes ``states`` float32 ``[B, H, ceil(T/64), 64, 64]``, the state before
    every 64th token, for ``rwkv7_wkv_backward_bf16``."""
    B, T, H, N = r.shape
    for nm, t in (("r", r), ("w", w), ("k", k), ("v", v), ("a", a), ("b", b), ("y", y)):
        _check(t, nm, torch.bfloat16, (B, T, H, N))
    _check(s_in, "s_in", torch.float32, (B, H, N, N), allow_none=True)
    _check(s_out, "s_out", torch.float32, (B, H, N, N))
    _check(states, "states", torch.float32, (B, H, n_checkpoints(T), N, N))
    _call("rwkv7_wkv_prefill_save_bf16", int(path), B, T, H, N,
          *[_ptr(t) for t in (r, w, k, v, a, b, s_in, y, s_out, states)], _stream(stream))


def rwkv7_wkv_backward_bf16(r, w, k, v, a, b, states, dy, ds_out, dr, dw, dk, dv, da, db, ds_in,
                            stream=None) -> None:
    """Gradients (float32) of a loss with dL/dy = ``dy`` (bf16) and dL/ds_out = ``ds_out`` (float32 or
    None) with respect to r, w, k, v, a, b (``[B, T, H, 64]``) and s_in (``ds_in`` or None)."""
    B, T, H, N = r.shape
    for nm, t in (("r", r), ("w", w), ("k", k), ("v", v), ("a", a), ("b", b), ("dy", dy)):
        _check(t, nm, torch.bfloat16, (B, T, H, N))
    for nm, t in (("dr", dr), ("dw", dw), ("dk", dk), ("dv", dv), ("da", da), ("db", db)):
        _check(t, nm, torch.float32, (B, T, H, N))
    _check(states, "states", torch.float32, (B, H, n_checkpoints(T), N, N))
    _check(ds_out, "ds_out", torch.float32, (B, H, N, N), allow_none=True)
    _check(ds_in, "ds_in", torch.float32, (B, H, N, N), allow_none=True)
    _call("rwkv7_wkv_backward_bf16", B, T, H, N, *[_ptr(t) for t in (r, w, k, v, a, b, states, dy, ds_out)],
          *[_ptr(t) for t in (dr, dw, dk, dv, da, db, ds_in)], _stream(stream))


def rwkv7_status_string(status: int) -> str:
    return load_library().rwkv7_status_string(int(status)).decode()


def rwkv7_get_last_error() -> int:
    return int(load_library().rwkv7_get_last_error())


def rwkv7_version() -> int:
    return int(load_library().rwkv7_version())


def rwkv7_test_set_wait_hooks(max_polls: int = 0, skip_publish_pair: int = -1) -> None:
    """Test hook of the failure path: bound every device wait of later chunked launches to
    ``max_polls`` polls (0 = production bound) and keep the chain flag of pair ``skip_publish_pair``'s
    first chunk down in the task-parallel schedule (-1 = none).  ``(0, -1)`` restores the defaults."""
    _call("rwkv7_test_set_wait_hooks", int(max_polls), int(skip_publish_pair))


# ---- conveniences: allocate outputs with torch, then call the entry points ------------------------

def prefill(r, w, k, v, a, b, s_in=None, *, path: int = RWKV7_PATH_AUTO, stream=None):
    """Allocate ``y`` and ``s_out`` and run prefill; returns ``(y, s_out)``."""
    B, T, H, N = r.shape
    y = torch.empty_like(r)
    s_out = torch.empty((B, H, N, N), dtype=torch.float32, device=r.device)
    if r.dtype == torch.float32:
        if path not in (RWKV7_PATH_AUTO, RWKV7_PATH_SCAN):
            raise ValueError("float32 prefill runs on the scan kernel only")
        rwkv7_wkv_prefill(r, w, k, v, a, b, s_in, y, s_out, stream)
    else:
        rwkv7_wkv_prefill_bf16_path(path, r, w, k, v, a, b, s_in, y, s_out, stream)
    return y, s_out


def decode_(r, w, k, v, a, b, state, y=None, *, stream=None):
    """One decode step updating ``state`` in place; returns ``y``."""
    if y is None:
        y = torch.empty_like(r)
    if r.dtype == torch.float32:
        rwkv7_wkv_decode(r, w, k, v, a, b, state, y, stream)
    else:
        rwkv7_wkv_decode_bf16(r, w, k, v, a, b, state, y, stream)
    return y


def prefill_model_native(r, xw, k, v, xa, k_k=None, s_in=None, *, path: int = RWKV7_PATH_AUTO, stream=None):
    """Allocate ``y`` and ``s_out`` and run the prefill on model-native inputs; returns ``(y, s_out)``."""
    B, T, H, N = r.shape
    y = torch.empty_like(r)
    s_out = torch.empty((B, H, N, N), dtype=torch.float32, device=r.device)
    rwkv7_wkv_prefill_fused_bf16(path, r, xw, k, v, xa, k_k, s_in, y, s_out, stream)
    return y, s_out


def decode_model_native_(r, xw, k, v, xa, k_k, state, y=None, *, stream=None):
    """One decode step on model-native inputs, updating ``state`` in place; returns ``y``."""
    if y is None:
        y = torch.empty_like(r)
    rwkv7_wkv_decode_fused_bf16(r, xw, k, v, xa, k_k, state, y, stream)
    return y


def prefill_ext(r, w, k, v, a, b=None, s_in=None, *, path: int = RWKV7_PATH_AUTO, model_native=False, k_k=None,
                group_norm=False, ln_w=None, ln_b=None, schedule=0, stream=None):
    """Allocate ``y`` and ``s_out`` and run the prefill with options; returns ``(y, s_out)``."""
    B, T, H, N = r.shape
    y = torch.empty_like(r)
    s_out = torch.empty((B, H, N, N), dtype=torch.float32, device=r.device)
    rwkv7_wkv_prefill_ext_bf16(path, r, w, k, v, a, b, s_in, y, s_out, model_native=model_native, k_k=k_k,
                               group_norm=group_norm, ln_w=ln_w, ln_b=ln_b, schedule=schedule, stream=stream)
    return y, s_out


def decode_ext_(r, w, k, v, a, b, state, y=None, *, model_native=False, k_k=None, group_norm=False, ln_w=None,
                ln_b=None, stream=None):
    """One decode step with options, updating ``state`` in place; returns ``y``."""
    if y is None:
        y = torch.empty_like(r)
    rwkv7_wkv_decode_ext_bf16(r, w, k, v, a, b, state, y, model_native=model_native, k_k=k_k,
                              group_norm=group_norm, ln_w=ln_w, ln_b=ln_b, stream=stream)
    return y


def prefill_save(r, w, k, v, a, b, s_in=None, *, path: int = RWKV7_PATH_AUTO, stream=None):
    """Allocate and run the checkpointing prefill; returns ``(y, s_out, states)``."""
    B, T, H, N = r.shape
    y = torch.empty_like(r)
    s_out = torch.empty((B, H, N, N), dtype=torch.float32, device=r.device)
    states = torch.empty((B, H, n_checkpoints(T), N, N), dtype=torch.float32, device=r.device)
    rwkv7_wkv_prefill_save_bf16(r, w, k, v, a, b, s_in, y, s_out, states, stream=stream, path=path)
    return y, s_out, states


def backward(r, w, k, v, a, b, states, dy, ds_out=None, *, stream=None):
    """Allocate and run the backward; returns float32 ``(dr, dw, dk, dv, da, db, ds_in)``."""
    B, T, H, N = r.shape
    g = [torch.empty((B, T, H, N), dtype=torch.float32, device=r.device) for _ in range(6)]
    ds_in = torch.empty((B, H, N, N), dtype=torch.float32, device=r.device)
    rwkv7_wkv_backward_bf16(r, w, k, v, a, b, states, dy, ds_out, *g, ds_in, stream=stream)
    return tuple(g) + (ds_in,)
