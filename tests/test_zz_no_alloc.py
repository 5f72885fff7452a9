"""tsenor_mask_noalloc: the plan + round kernels with the plan between them
in a fixed array inside the library, for callers that cannot allocate device
memory at call time (their memory is held by another allocator, or they run
under a fixed device-memory budget).  Its masks must equal tsenor_mask's bit
for bit (masks are integer results), call after call, even though every call
reuses the same array.

Collected last on purpose: if it fails, a run that stops at the first failure
has already run every other test.
"""
import ctypes as C

import numpy as np
import pytest

import synth

torch = pytest.importorskip("torch")
pytestmark = pytest.mark.gpu

import sparse_mask_search_b200 as tsl  # noqa: E402


def _device(storage, dtype):
    if dtype == "bf16":
        return torch.from_numpy(np.ascontiguousarray(storage).view(np.int16)).view(torch.bfloat16).cuda()
    return torch.from_numpy(np.ascontiguousarray(storage)).cuda()


def _noalloc_raw(Wd, N, M, tau, iters, sweeps, out):
    """Call the C entry point directly through the C ABI."""
    L = tsl.lib()
    dtype = tsl.TSENOR_BF16 if Wd.dtype == torch.bfloat16 else tsl.TSENOR_F32
    rows, cols = Wd.shape
    return L.tsenor_mask_noalloc(C.c_void_p(Wd.data_ptr()), dtype, rows, cols, N, M, float(tau), iters, sweeps,
                                 C.c_void_p(out.data_ptr()), C.c_void_p(torch.cuda.current_stream().cuda_stream))


def test_noalloc_matches_tsenor_mask_on_consecutive_calls():
    # two calls in a row on different shapes, patterns and dtypes: the second
    # call reuses the array the first one filled
    cases = [
        ("bf16", "t3_outlier_cols", 0.02, 512, 1024, 16, 32, 20.0, 300, 8),
        ("f32", "normal", 1.0, 256, 320, 3, 8, 20.0, 200, 4),
    ]
    for k, (dtype, dist, scale, rows, cols, N, M, tau, iters, sweeps) in enumerate(cases):
        storage, _ = synth.make_matrix(rows, cols, dtype, dist, scale, seed=50 + k)
        Wd = _device(storage, dtype)
        ref = tsl.tsenor_mask(Wd, N, M, tau, iters, sweeps)
        out = torch.full_like(ref, -1)
        assert _noalloc_raw(Wd, N, M, tau, iters, sweeps, out) == 0
        torch.cuda.synchronize()
        assert torch.equal(out, ref), f"call {k}"


def test_noalloc_rejects_sizes_above_its_array():
    Wd = torch.zeros((64, 64), dtype=torch.bfloat16, device="cuda")
    out = torch.zeros((64, 2), dtype=torch.int32, device="cuda")
    L = tsl.lib()
    rows, cols = 8192, 4096          # 2 * 16 Mi params: rejected on the host before any launch
    status = L.tsenor_mask_noalloc(C.c_void_p(Wd.data_ptr()), tsl.TSENOR_BF16, rows, cols, 2, 4, 10.0, 5, 1,
                                   C.c_void_p(out.data_ptr()), None)
    assert status == -6
    assert b"TSENOR_NOALLOC_MAX_PARAMS" in L.tsenor_status_string(status)
    assert rows * cols > tsl.NOALLOC_MAX_PARAMS
