"""Host-side checks of the C ABI that need no GPU: the library loads, exports
every entry point that include/rwkv7.h declares, and rejects bad arguments
before launching anything (these calls return before any CUDA call)."""

import ctypes
import os
import re
import subprocess

import pytest

import rwkv_delta_rule_b200 as lib7

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
HEADER = os.path.join(ROOT, "include", "rwkv7.h")


@pytest.fixture(scope="module")
def cdll():
    from rwkv_delta_rule_b200 import build

    build.build()
    return lib7.load_library()


def declared_symbols():
    text = open(HEADER).read()
    return sorted(set(re.findall(r"RWKV7_API\s+[\w\s\*]+?\b(rwkv7_\w+)\s*\(", text)))


def test_header_declares_binding_names():
    assert declared_symbols() == sorted(lib7.EXPORTED_SYMBOLS)


def test_binding_declares_a_signature_for_every_entry_point():
    """ctypes passes Python ints as 32-bit C ints to a function without argtypes, which truncates
    pointers: every exported entry point must have its argument types set by load_library."""
    lib = lib7.load_library()
    for name in lib7.EXPORTED_SYMBOLS:
        fn = getattr(lib, name)
        assert fn.argtypes is not None, name
        assert fn.restype is not None, name


def test_library_exports_every_declared_symbol(cdll):
    out = subprocess.run(["nm", "-D", "--defined-only", lib7.library_path()], capture_output=True, text=True,
                         check=True).stdout
    exported = set(re.findall(r" T (rwkv7_\w+)", out))
    for sym in declared_symbols():
        assert sym in exported, sym
        assert hasattr(cdll, sym)
    # nothing else leaks out (the CUDA runtime is linked statically and hidden)
    assert all(s.startswith("rwkv7_") for s in re.findall(r" T (\w+)", out))


def test_library_needs_no_shared_cuda_runtime():
    out = subprocess.run(["ldd", lib7.library_path()], capture_output=True, text=True).stdout
    assert "libcudart" not in out


def test_status_strings(cdll):
    assert lib7.rwkv7_status_string(0) == "ok"
    assert "64" in lib7.rwkv7_status_string(5)
    assert "range" in lib7.rwkv7_status_string(6)
    assert lib7.rwkv7_status_string(99) == "unknown status"
    assert lib7.rwkv7_version() >= 100


FAKE = 0x10000  # 16-byte aligned, never dereferenced: every call below fails validation first
MIS = 0x10008   # 8-byte aligned only


def prefill_bf16(cdll, B=1, T=4, H=1, N=64, ptr=FAKE, s_out=FAKE, path=None):
    args = [B, T, H, N] + [ptr] * 6 + [None, ptr, s_out, None]
    if path is None:
        return cdll.rwkv7_wkv_prefill_bf16(*args)
    return cdll.rwkv7_wkv_prefill_bf16_path(path, *args)


def test_rejects_head_size(cdll):
    assert prefill_bf16(cdll, N=32) == 5
    assert cdll.rwkv7_wkv_prefill(1, 4, 1, 128, *([FAKE] * 6), None, FAKE, FAKE, None) == 5
    assert cdll.rwkv7_wkv_decode_bf16(1, 1, 63, *([FAKE] * 6), FAKE, FAKE, None) == 5


def test_rejects_bad_sizes_and_nulls(cdll):
    assert prefill_bf16(cdll, B=0) == 1
    assert prefill_bf16(cdll, H=-1) == 1
    assert prefill_bf16(cdll, T=-1) == 1
    assert prefill_bf16(cdll, ptr=None) == 1
    assert prefill_bf16(cdll, s_out=None) == 1
    assert prefill_bf16(cdll, path=7) == 1
    assert cdll.rwkv7_wkv_decode(0, 1, 64, *([FAKE] * 6), FAKE, FAKE, None) == 1
    assert cdll.rwkv7_wkv_decode(1, 1, 64, *([FAKE] * 5), None, FAKE, FAKE, None) == 1


def test_rejects_misaligned(cdll):
    assert prefill_bf16(cdll, ptr=MIS) == 2
    assert prefill_bf16(cdll, s_out=MIS) == 2
    assert cdll.rwkv7_wkv_decode_bf16(1, 1, 64, *([FAKE] * 5), MIS, FAKE, FAKE, None) == 2


def test_varlen_rejects(cdll):
    base = [FAKE] * 6 + [None, FAKE, FAKE, None]
    assert cdll.rwkv7_wkv_prefill_varlen_bf16(0, 2, 10, 8, 1, 64, None, *base) == 1  # no offsets
    assert cdll.rwkv7_wkv_prefill_varlen_bf16(0, 2, 10, 8, 1, 64, MIS, *base) == 2
    assert cdll.rwkv7_wkv_prefill_varlen_bf16(0, 2, 10, -1, 1, 64, FAKE, *base) == 1
    assert cdll.rwkv7_wkv_prefill_varlen_bf16(9, 2, 10, 8, 1, 64, FAKE, *base) == 1
    assert cdll.rwkv7_wkv_prefill_varlen_bf16(0, 2, 10, 8, 1, 32, FAKE, *base) == 5


def test_training_and_bf16_state_entry_points_reject(cdll):
    ops = [FAKE] * 6
    # rwkv7_wkv_prefill_save_bf16(path, B, T, H, N, ops, s_in, y, s_out, states, stream)
    assert cdll.rwkv7_wkv_prefill_save_bf16(0, 1, 4, 1, 32, *ops, None, FAKE, FAKE, FAKE, None) == 5
    assert cdll.rwkv7_wkv_prefill_save_bf16(0, 1, 4, 1, 64, *ops, None, FAKE, FAKE, None, None) == 1
    assert cdll.rwkv7_wkv_prefill_save_bf16(0, 1, 4, 1, 64, *ops, None, FAKE, FAKE, MIS, None) == 2
    assert cdll.rwkv7_wkv_prefill_save_bf16(5, 1, 4, 1, 64, *ops, None, FAKE, FAKE, FAKE, None) == 1
    # rwkv7_wkv_backward_bf16(B, T, H, N, ops, states, dy, ds_out, dr dw dk dv da db, ds_in, stream)
    grads = [FAKE] * 6
    assert cdll.rwkv7_wkv_backward_bf16(1, 4, 1, 16, *ops, FAKE, FAKE, None, *grads, None, None) == 5
    assert cdll.rwkv7_wkv_backward_bf16(0, 4, 1, 64, *ops, FAKE, FAKE, None, *grads, None, None) == 1
    assert cdll.rwkv7_wkv_backward_bf16(1, 4, 1, 64, *ops, None, FAKE, None, *grads, None, None) == 1
    assert cdll.rwkv7_wkv_backward_bf16(1, 4, 1, 64, *ops, FAKE, FAKE, None, *grads[:5], None, None, None) == 1
    assert cdll.rwkv7_wkv_backward_bf16(1, 4, 1, 64, *ops, FAKE, FAKE, MIS, *grads, None, None) == 2
    # rwkv7_wkv_decode_bf16_bf16state(B, H, N, ops, s_inout, y, stream)
    assert cdll.rwkv7_wkv_decode_bf16_bf16state(1, 1, 64, *ops, None, FAKE, None) == 1
    assert cdll.rwkv7_wkv_decode_bf16_bf16state(1, 1, 64, *ops, MIS, FAKE, None) == 2
    assert cdll.rwkv7_wkv_decode_bf16_bf16state(1, 1, 48, *ops, FAKE, FAKE, None) == 5
    # rwkv7_wkv_decode_ext_bf16state(B, H, N, ops, opt, s_inout, y, stream): only independent_state applies
    opt = ctypes.byref(lib7.Options(0, None, 0, None, None, 0, 1))
    assert cdll.rwkv7_wkv_decode_ext_bf16state(1, 1, 64, *ops, ctypes.byref(lib7.Options(1, None, 0, None, None, 0, 0)),
                                               FAKE, FAKE, None) == 1  # model-native inputs
    assert cdll.rwkv7_wkv_decode_ext_bf16state(1, 1, 64, *ops, ctypes.byref(lib7.Options(0, None, 1, None, None, 0, 0)),
                                               FAKE, FAKE, None) == 1  # group norm
    assert cdll.rwkv7_wkv_decode_ext_bf16state(1, 1, 64, *ops, opt, None, FAKE, None) == 1
    assert cdll.rwkv7_wkv_decode_ext_bf16state(1, 1, 64, *ops, opt, MIS, FAKE, None) == 2
    assert cdll.rwkv7_wkv_decode_ext_bf16state(1, 1, 32, *ops, opt, FAKE, FAKE, None) == 5


def test_host_prefill_rejects(cdll):
    ops = [FAKE] * 6
    # rwkv7_wkv_prefill_host_bf16(path, B, T, H, N, host ops, s_in, y, s_out, dev ops, dev s_in, dev y,
    #                             dev s_out, slices, stream)
    def call(path=0, N=64, host=FAKE, dev=FAKE, s_in=None, dev_s_in=None, slices=0):
        return cdll.rwkv7_wkv_prefill_host_bf16(path, 2, 4, 1, N, *([host] * 6), s_in, host, host, *([dev] * 6),
                                                dev_s_in, dev, dev, slices, None)
    assert call(path=9) == 1
    assert call(N=32) == 5
    assert call(host=None) == 1
    assert call(dev=None) == 1
    assert call(host=MIS) == 2
    assert call(dev=MIS) == 2
    assert call(s_in=FAKE, dev_s_in=None) == 1  # an initial state needs its staging buffer
    assert call(slices=-1) == 1


def test_binding_rejects_cpu_tensors():
    import torch

    x = torch.zeros(1, 2, 1, 64, dtype=torch.bfloat16)
    s = torch.zeros(1, 1, 64, 64)
    with pytest.raises(ValueError):
        lib7.rwkv7_wkv_prefill_bf16(x, x, x, x, x, x, None, x, s)
