"""Seeded synthetic inputs for the x070 state recurrence.

This module only draws random operands. It holds none of the recurrence's
arithmetic, so both the float64 oracle and the CUDA library can be fed from it
without sharing any code with each other.

Recipe (one torch CPU ``Generator`` per case, seeded, drawn in this order):

* ``r, z, kh_raw, s, v, alpha`` of shape ``[B, T, H, N]`` and, if requested,
  the initial state ``S0`` of shape ``[B, H, N, N]``;
* ``r, v ~ N(0, 1)``; ``z ~ N(z_mean, 1)``; ``s ~ U(0.5, 1.5)``;
  ``alpha ~ U(0, 1)``; ``S0 ~ N(0, s0_std)`` (std, not variance);
* ``kh = kh_raw / ||kh_raw||`` over the N channels of each (b, t, h), so every
  token gets a fresh unit key direction per head;
* ``k = kh * s``, ``a = -kh``, ``b = kh * alpha``;
* ``w = exp(-0.606531 * sigmoid(z))``.  This is the model's decay
  parametrisation: the pages build the decay as ``exp(-exp(x))`` with
  ``x = -softplus(-u) - 0.5``, and ``exp(-softplus(-u)) = sigmoid(u)``, so the
  decay is ``exp(-e^-0.5 * sigmoid(u))`` with ``e^-0.5 = 0.606531``
  (RWKV-7 G0 7.2B walkthrough, lshu.cn/news/198401, section 7.1).  Every w lies
  in ``(0.5452, 1)``.

All arithmetic above is float32; the operands are then rounded to the storage
dtype (round-to-nearest-even for bf16).  The returned float32 copies hold the
*rounded* values, so the oracle sees exactly the bytes the GPU sees.

``device``: the draws above can also run on a CUDA device (a generator of that
device, same seed, same order).  The distributions are the same but the random
stream is the device's, so the values differ from a CPU draw of the same seed;
the benchmark draws its full-size workloads this way (seconds instead of
minutes), every parity test draws on the CPU.

The configurations are the pages' model widths with head size 64:
0.1B D768 (H=12), 1.5B D2048 (H=32), L24-D1024 (H=16), 7.2B-scale D4096 (H=64).
"""

from __future__ import annotations

import dataclasses
from typing import Dict, Optional

import torch

N_HEAD = 64
DECAY_SCALE = 0.606531  # e^-0.5 rounded as in the model's decay clamp


@dataclasses.dataclass(frozen=True)
class Case:
    """One synthetic workload: shape, storage dtype and generator settings."""

    name: str
    B: int
    T: int
    H: int
    dtype: str  # "f32" or "bf16"
    seed: int
    z_mean: float = 0.0
    s0_std: Optional[float] = None  # None: zero initial state
    N: int = N_HEAD


# The five workloads.  Decode (``decode_l24_d1024``) draws T = 1024 tokens and
# feeds them one step at a time; the chained case feeds two halves.
CASES: Dict[str, Case] = {
    "prefill_f32_b1_t64_h2": Case("prefill_f32_b1_t64_h2", 1, 64, 2, "f32", 1000),
    "prefill_d768_b8_t4096": Case("prefill_d768_b8_t4096", 8, 4096, 12, "bf16", 1001, s0_std=0.1),
    "prefill_d2048_b16_t8192_chained": Case("prefill_d2048_b16_t8192_chained", 16, 8192, 32, "bf16", 1002),
    "decode_l24_d1024_b256_1024steps": Case("decode_l24_d1024_b256_1024steps", 256, 1024, 16, "bf16", 1003),
    "prefill_d4096_b4_t16384": Case("prefill_d4096_b4_t16384", 4, 16384, 64, "bf16", 1004, z_mean=1.0),
}


def storage_dtype(name: str) -> torch.dtype:
    if name == "f32":
        return torch.float32
    if name == "bf16":
        return torch.bfloat16
    raise ValueError(f"unknown storage dtype {name!r}")


def draw(B: int, T: int, H: int, N: int = N_HEAD, *, seed: int, dtype: str = "bf16",
         z_mean: float = 0.0, s0_std: Optional[float] = None, device=None,
         f32_copies: bool = True) -> Dict[str, torch.Tensor]:
    """Draw one workload.

    Returns a dict with
      ``r, w, k, v, a, b``: storage-dtype tensors ``[B, T, H, N]`` (contiguous, on ``device``,
      the CPU by default);
      ``<name>_f32``: the same values as float32 (omitted when ``f32_copies`` is False);
      ``s0``: float32 ``[B, H, N, N]`` or ``None`` for a zero state.
    """
    dev = torch.device("cpu" if device is None else device)
    g = torch.Generator(device=dev)
    g.manual_seed(int(seed))
    shp = (B, T, H, N)
    f32 = torch.float32
    r = torch.randn(shp, generator=g, dtype=f32, device=dev)
    z = torch.randn(shp, generator=g, dtype=f32, device=dev) + float(z_mean)
    kh = torch.randn(shp, generator=g, dtype=f32, device=dev)
    s = torch.rand(shp, generator=g, dtype=f32, device=dev) + 0.5
    v = torch.randn(shp, generator=g, dtype=f32, device=dev)
    alpha = torch.rand(shp, generator=g, dtype=f32, device=dev)
    s0 = None
    if s0_std is not None:
        s0 = torch.randn((B, H, N, N), generator=g, dtype=f32, device=dev) * float(s0_std)

    kh = kh / kh.norm(dim=-1, keepdim=True)
    k = kh * s
    a = -kh
    b = kh * alpha
    w = torch.exp(-DECAY_SCALE * torch.sigmoid(z))
    del z, s, alpha

    sd = storage_dtype(dtype)
    out: Dict[str, torch.Tensor] = {}
    for nm, x in (("r", r), ("w", w), ("k", k), ("v", v), ("a", a), ("b", b)):
        xs = x.to(sd).contiguous()
        out[nm] = xs
        if f32_copies:
            out[nm + "_f32"] = xs.to(f32) if sd != f32 else xs
    out["s0"] = s0
    return out


def draw_model_native(B: int, T: int, H: int, N: int = N_HEAD, *, seed: int, z_mean: float = 0.0,
                      s0_std: Optional[float] = None, device=None) -> Dict[str, torch.Tensor]:
    """Draw model-native inputs for the fused operand prologue (no prologue arithmetic here).

    Returns bf16 ``[B, T, H, N]`` tensors ``r`` ~ N(0,1), ``xw`` (decay pre-activation) ~
    N(z_mean, 1), ``k`` = unit vector per (b, t, h) times U(0.5, 1.5) per channel, ``v`` ~ N(0,1)
    and ``xa`` (in-context learning-rate pre-activation) ~ N(0,1); ``<name>_f32`` copies; ``k_k``:
    float32 ``[H, N]`` ~ U(0.5, 1.5); ``s0``: float32 ``[B, H, N, N]`` or None.  ``device`` as in
    :func:`draw`.
    """
    dev = torch.device("cpu" if device is None else device)
    g = torch.Generator(device=dev)
    g.manual_seed(int(seed))
    shp = (B, T, H, N)
    f32 = torch.float32
    r = torch.randn(shp, generator=g, dtype=f32, device=dev)
    xw = torch.randn(shp, generator=g, dtype=f32, device=dev) + float(z_mean)
    kh = torch.randn(shp, generator=g, dtype=f32, device=dev)
    s = torch.rand(shp, generator=g, dtype=f32, device=dev) + 0.5
    v = torch.randn(shp, generator=g, dtype=f32, device=dev)
    xa = torch.randn(shp, generator=g, dtype=f32, device=dev)
    k_k = torch.rand((H, N), generator=g, dtype=f32, device=dev) + 0.5
    s0 = None
    if s0_std is not None:
        s0 = torch.randn((B, H, N, N), generator=g, dtype=f32, device=dev) * float(s0_std)
    k = kh / kh.norm(dim=-1, keepdim=True) * s
    out: Dict[str, torch.Tensor] = {}
    for nm, x in (("r", r), ("xw", xw), ("k", k), ("v", v), ("xa", xa)):
        xs = x.to(torch.bfloat16).contiguous()
        out[nm] = xs
        out[nm + "_f32"] = xs.to(f32)
    out["k_k"] = k_k.contiguous()
    out["s0"] = s0
    return out


def draw_group_norm(H: int, N: int = N_HEAD, *, seed: int) -> Dict[str, torch.Tensor]:
    """Draw the per-head GroupNorm affine parameters: ``ln_w`` float32 ``[H, N]`` ~ U(0.5, 1.5) and
    ``ln_b`` float32 ``[H, N]`` ~ N(0, 0.1^2)."""
    g = torch.Generator(device="cpu")
    g.manual_seed(int(seed))
    ln_w = torch.rand((H, N), generator=g, dtype=torch.float32) + 0.5
    ln_b = torch.randn((H, N), generator=g, dtype=torch.float32) * 0.1
    return {"ln_w": ln_w.contiguous(), "ln_b": ln_b.contiguous()}


def draw_grads(B: int, T: int, H: int, N: int = N_HEAD, *, seed: int, ds_std: Optional[float] = 1.0
               ) -> Dict[str, torch.Tensor]:
    """Draw the incoming gradients of a backward call: ``dy`` bf16 ``[B, T, H, N]`` ~ N(0, 1) (with a
    ``dy_f32`` copy) and ``ds_out`` float32 ``[B, H, N, N]`` ~ N(0, ds_std^2), or None."""
    g = torch.Generator(device="cpu")
    g.manual_seed(int(seed))
    dy = torch.randn((B, T, H, N), generator=g, dtype=torch.float32).to(torch.bfloat16).contiguous()
    ds = None
    if ds_std is not None:
        ds = (torch.randn((B, H, N, N), generator=g, dtype=torch.float32) * float(ds_std)).contiguous()
    return {"dy": dy, "dy_f32": dy.to(torch.float32), "ds_out": ds}


def draw_case(case: Case, *, T: Optional[int] = None, B: Optional[int] = None) -> Dict[str, torch.Tensor]:
    """Draw a named workload, optionally at a reduced B or T (same recipe, same seed)."""
    return draw(case.B if B is None else B, case.T if T is None else T, case.H, case.N,
                seed=case.seed, dtype=case.dtype, z_mean=case.z_mean, s0_std=case.s0_std)


def ragged_lengths(B: int, lo: int, hi: int, *, seed: int) -> torch.Tensor:
    """Per-row lengths ``T_b ~ U{lo..hi}`` (inclusive), int64, seeded."""
    g = torch.Generator(device="cpu")
    g.manual_seed(int(seed))
    return torch.randint(lo, hi + 1, (B,), generator=g, dtype=torch.int64)


def cu_seqlens(lengths: torch.Tensor) -> torch.Tensor:
    """Prefix offsets ``[0, T_0, T_0+T_1, ...]`` as int32 (packed-token layout)."""
    out = torch.zeros(lengths.numel() + 1, dtype=torch.int64)
    out[1:] = torch.cumsum(lengths.to(torch.int64), 0)
    return out.to(torch.int32)


def draw_packed(lengths: torch.Tensor, H: int, N: int = N_HEAD, *, seed: int, dtype: str = "bf16",
                z_mean: float = 0.0, s0_std: Optional[float] = None, device=None,
                f32_copies: bool = True) -> Dict[str, torch.Tensor]:
    """Draw a ragged batch in packed layout ``[sum(T_b), H, N]``.

    Same recipe as :func:`draw` with B = 1 and T = sum(T_b); row b owns tokens
    ``cu_seqlens[b] .. cu_seqlens[b+1]-1``.  ``s0`` is ``[len(lengths), H, N, N]``.
    """
    total = int(lengths.sum())
    d = draw(1, total, H, N, seed=seed, dtype=dtype, z_mean=z_mean, s0_std=None, device=device,
             f32_copies=f32_copies)
    out = {key: (val[0] if val is not None else None) for key, val in d.items()}
    if s0_std is not None:
        dev = torch.device("cpu" if device is None else device)
        g = torch.Generator(device=dev)
        g.manual_seed(int(seed) + 7919)
        out["s0"] = torch.randn((lengths.numel(), H, N, N), generator=g, dtype=torch.float32,
                                device=dev) * float(s0_std)
    else:
        out["s0"] = None
    out["cu_seqlens"] = cu_seqlens(lengths)
    return out
