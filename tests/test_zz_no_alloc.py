"""GPU test of rwkv7_wkv_prefill_host_noalloc_bf16, the host-buffer prefill that allocates nothing.

That entry point serves callers who hold their data in host memory and cannot allocate device
memory (a program that reaches the GPU only through this library, or one that must not call
cudaMalloc / cudaFree): it stages through one static device array of the library instead of
caller-given device buffers.  Here it is called through the C ABI (ctypes) twice in a row, with
different shapes, paths and inputs, and each result is compared with the device-buffer entry point
rwkv7_wkv_prefill_bf16_path on the same inputs.  The second call finds the first call's data still in
the shared array, so it also shows that nothing stale leaks into a result.

This file is named to be collected last, so a run that stops at the first failure has run every
other test before it; it also passes on its own in a fresh process.
"""

import pytest
import torch

import rwkv_delta_rule_b200 as lib7
import wkv7_inputs as wi
from helpers import OPS, TOL_BF16, TOL_BF16_PAIR, need_cuda, rel_err

pytestmark = pytest.mark.gpu


def _noalloc(cdll, path, host, s_in, y, s_out):
    """Calls the C entry point with host pointers on the current stream; returns its status."""
    B, T, H, N = host["r"].shape
    ptrs = [host[n].data_ptr() for n in OPS]
    return cdll.rwkv7_wkv_prefill_host_noalloc_bf16(
        int(path), B, T, H, N, *ptrs, None if s_in is None else s_in.data_ptr(), y.data_ptr(), s_out.data_ptr(),
        torch.cuda.current_stream().cuda_stream)


def _device_reference(path, d, s0):
    """The same prefill through the device-buffer entry point."""
    dev = {n: d[n].cuda() for n in OPS}
    B, T, H, N = d["r"].shape
    y = torch.empty((B, T, H, N), dtype=torch.bfloat16, device="cuda")
    s = torch.empty((B, H, N, N), dtype=torch.float32, device="cuda")
    lib7.rwkv7_wkv_prefill_bf16_path(path, *[dev[n] for n in OPS], None if s0 is None else s0.cuda(), y, s)
    torch.cuda.synchronize()
    return y.cpu(), s.cpu()


@pytest.mark.parametrize("pinned", [True, False])
def test_noalloc_host_prefill_matches_device_entry_point(pinned):
    need_cuda()
    cdll = lib7.load_library()
    calls = [
        # chunked kernel (AUTO at T >= 48), initial state given, ragged last chunk
        dict(B=2, T=200, H=3, seed=71, s0_std=0.1, path=lib7.RWKV7_PATH_AUTO),
        # sequential kernel, zero initial state, a different layout of the shared array
        dict(B=3, T=70, H=2, seed=72, s0_std=None, path=lib7.RWKV7_PATH_SCAN),
    ]
    for c in calls:
        d = wi.draw(c["B"], c["T"], c["H"], seed=c["seed"], dtype="bf16", s0_std=c["s0_std"])
        host = {n: (d[n].pin_memory() if pinned else d[n].clone()) for n in OPS}
        s0 = d["s0"]
        s_in = None if s0 is None else (s0.pin_memory() if pinned else s0.clone())
        B, T, H, N = d["r"].shape
        y = torch.full((B, T, H, N), float("nan"), dtype=torch.bfloat16)
        s_out = torch.full((B, H, N, N), float("nan"), dtype=torch.float32)
        if pinned:
            y, s_out = y.pin_memory(), s_out.pin_memory()
        assert _noalloc(cdll, c["path"], host, s_in, y, s_out) == 0
        torch.cuda.current_stream().synchronize()
        assert lib7.rwkv7_get_last_error() == 0
        y_ref, s_ref = _device_reference(c["path"], d, s0)
        assert rel_err(y, y_ref.double()) <= TOL_BF16_PAIR, c
        assert rel_err(s_out, s_ref.double()) <= TOL_BF16, c


def test_noalloc_rejects_calls_beyond_the_staging_limit():
    need_cuda()
    cdll = lib7.load_library()
    # B=1, T=8192, H=4: 7 operand-sized regions of 4 MiB each + one state = 28.06 MiB fits; T=9400 does not
    H, N = 4, 64
    fits = 7 * (8192 * H * N * 2) + H * N * N * 4
    assert fits <= lib7.NOALLOC_STAGING_BYTES
    T = 9400
    need = 7 * (T * H * N * 2) + H * N * N * 4
    assert need > lib7.NOALLOC_STAGING_BYTES
    ops = [torch.zeros((1, T, H, N), dtype=torch.bfloat16) for _ in OPS]
    y = torch.full((1, T, H, N), 7.0, dtype=torch.bfloat16)
    s_out = torch.full((1, H, N, N), 7.0)
    st = cdll.rwkv7_wkv_prefill_host_noalloc_bf16(0, 1, T, H, N, *[t.data_ptr() for t in ops], None, y.data_ptr(),
                                                  s_out.data_ptr(), None)
    assert st == 1  # RWKV7_ERR_INVALID, nothing enqueued
    torch.cuda.synchronize()
    assert bool((y == 7.0).all()) and bool((s_out == 7.0).all())
    with pytest.raises(lib7.Rwkv7Error):
        lib7.rwkv7_wkv_prefill_host_noalloc_bf16(0, *ops, None, y, s_out)
