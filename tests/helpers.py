"""Shared test helpers: error metrics and device transfer (no recurrence arithmetic)."""

import numpy as np
import torch

# Parity bars: max|gpu - oracle| / max|oracle| over a whole output.
TOL_F32 = 1e-4
TOL_BF16 = 5e-3
# Two GPU outputs that were each rounded to bf16: each rounding moves an
# element by up to half an ulp (2^-9 of its binade's top, i.e. up to 2^-8 of
# the element), so two of them can differ by one bf16 ulp near max|y|:
# 2^-7 = 7.8e-3 of max|y|, plus each kernel's own float32 error.
TOL_BF16_PAIR = 1e-2

OPS = ("r", "w", "k", "v", "a", "b")


def rel_err(got, ref) -> float:
    got = np.asarray(got.detach().float().cpu().numpy() if hasattr(got, "detach") else got, dtype=np.float64)
    ref = np.asarray(ref, dtype=np.float64)
    assert got.shape == ref.shape, (got.shape, ref.shape)
    scale = np.abs(ref).max()
    if scale == 0:
        return float(np.abs(got).max())
    return float(np.abs(got - ref).max() / scale)


def to_dev(d, dev="cuda"):
    """Storage-dtype operands and the initial state moved to the device."""
    out = {n: d[n].to(dev) for n in OPS}
    out["s0"] = None if d["s0"] is None else d["s0"].to(dev)
    return out


def oracle_ops(d):
    return [d[n + "_f32"] for n in OPS]


def need_cuda():
    import pytest

    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
