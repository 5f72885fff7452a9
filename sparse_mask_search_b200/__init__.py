"""Python binding of the B200 transposable N:M mask library (include/tsenor.h).

Argument marshalling only: every step of the solver runs in the CUDA kernels
of libtsenor_b200.so.  PyTorch provides device memory and streams.  There is
no CPU fallback: if the library is missing, importing a function raises.
"""
from __future__ import annotations

import ctypes as C
import os

HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(HERE, "libtsenor_b200.so")

TSENOR_F32, TSENOR_BF16 = 0, 1
STATUS = {0: "TSENOR_OK", -1: "TSENOR_ERR_ARG", -2: "TSENOR_ERR_SHAPE", -3: "TSENOR_ERR_UNSUPPORTED_M",
          -4: "TSENOR_ERR_CUDA", -5: "TSENOR_ERR_DEVICE", -6: "TSENOR_ERR_TOO_LARGE"}
NOALLOC_MAX_PARAMS = 16 * 1024 * 1024
MAX_TAU = 80.0            # TSENOR_MAX_TAU: larger tau is rejected (TSENOR_ERR_ARG)
EXPORTS = ("tsenor_mask", "tsenor_plan", "tsenor_round", "tsenor_objective", "tsenor_error_count",
           "tsenor_status_string", "tsenor_last_error", "tsenor_mask_noalloc", "tsenor_mask_safeguard",
           "tsenor_mask_padded", "tsenor_mask_warm", "tsenor_plan_warm", "tsenor_mask_scores", "tsenor_mask_host")

_lib = None


class TsenorError(RuntimeError):
    def __init__(self, status: int, msg: str):
        super().__init__(f"{STATUS.get(status, status)}: {msg}")
        self.status = status


def lib() -> C.CDLL:
    """Load the CUDA library (raises if it has not been built)."""
    global _lib
    if _lib is None:
        if not os.path.exists(LIB_PATH):
            raise ImportError(f"{LIB_PATH} is missing: build it with "
                              "`python -m sparse_mask_search_b200.build` (nvcc, sm_100a)")
        L = C.CDLL(LIB_PATH)
        p, i64, i32, f32 = C.c_void_p, C.c_int64, C.c_int, C.c_float
        L.tsenor_mask.argtypes = [p, i32, i64, i64, i32, i32, f32, i32, i32, p, p]
        L.tsenor_mask_noalloc.argtypes = [p, i32, i64, i64, i32, i32, f32, i32, i32, p, p]
        L.tsenor_plan.argtypes = [p, i32, i64, i64, i32, i32, f32, i32, p, p]
        L.tsenor_mask_padded.argtypes = [p, i32, i64, i64, i32, i32, f32, i32, i32, p, p]
        L.tsenor_mask_safeguard.argtypes = [p, i32, i64, i64, i32, i32, f32, i32, i32, p, p, p, p]
        L.tsenor_mask_scores.argtypes = [p, i64, i64, i32, i32, f32, i32, i32, p, p]
        L.tsenor_mask_host.argtypes = [p, i32, i64, i64, i32, i32, f32, i32, i32, p, p]
        L.tsenor_mask_warm.argtypes = [p, i32, i64, i64, i32, i32, f32, i32, i32, f32, i32, p, p, p, p]
        L.tsenor_plan_warm.argtypes = [p, i32, i64, i64, i32, i32, f32, i32, f32, i32, p, p, p, p]
        L.tsenor_round.argtypes = [p, p, i32, i64, i64, i32, i32, i32, p, p]
        L.tsenor_objective.argtypes = [p, i32, i64, i64, p, i32, i32, p, p]
        L.tsenor_error_count.argtypes = [p, C.POINTER(C.c_int64)]
        L.tsenor_status_string.argtypes = [i32]
        L.tsenor_status_string.restype = C.c_char_p
        L.tsenor_last_error.restype = C.c_char_p
        for name in EXPORTS:
            getattr(L, name).restype = getattr(L, name).restype or C.c_int
        _lib = L
    return _lib


def _check(status: int) -> None:
    if status != 0:
        L = lib()
        msg = L.tsenor_status_string(status).decode()
        if status == -4:
            msg += ": " + L.tsenor_last_error().decode()
        raise TsenorError(status, msg)


def _stream_handle(stream) -> int | None:
    import torch
    if stream is None:
        stream = torch.cuda.current_stream()
    return stream.cuda_stream if hasattr(stream, "cuda_stream") else int(stream)


def _dtype_code(W) -> int:
    import torch
    if W.dtype == torch.bfloat16:
        return TSENOR_BF16
    if W.dtype == torch.float32:
        return TSENOR_F32
    raise TypeError(f"W must be bfloat16 or float32, got {W.dtype}")


def words_per_row(cols: int) -> int:
    return (cols + 31) // 32


def _check_2d_cuda(t, name):
    if not t.is_cuda or t.dim() != 2 or not t.is_contiguous():
        raise ValueError(f"{name} must be a contiguous 2-D CUDA tensor")


def tsenor_mask(W, N: int, M: int, tau: float, iters: int, sweeps: int, out=None, stream=None):
    """Transposable N:M mask of W; returns (rows, ceil(cols/32)) int32 words (bit patterns)."""
    import torch
    _check_2d_cuda(W, "W")
    rows, cols = W.shape
    if out is None:
        out = torch.empty((rows, words_per_row(cols)), dtype=torch.int32, device=W.device)
    _check(lib().tsenor_mask(W.data_ptr(), _dtype_code(W), rows, cols, N, M, float(tau), iters, sweeps,
                             out.data_ptr(), _stream_handle(stream)))
    return out


def tsenor_mask_noalloc(W, N: int, M: int, tau: float, iters: int, sweeps: int, out=None, stream=None):
    """tsenor_mask without any device allocation by the library.

    For callers whose device memory is reserved by another allocator or who
    run under a fixed memory budget.  The plan between the two kernels lives
    in a 64 MiB array inside the library (rows*cols <= NOALLOC_MAX_PARAMS).
    All calls on a device share that array: calls that overlap on the GPU
    race.  The first call on a device looks up the array's address; make it
    before any stream capture.  Only ``out`` is allocated here (by torch)
    when it is not given.
    """
    import torch
    _check_2d_cuda(W, "W")
    rows, cols = W.shape
    if out is None:
        out = torch.empty((rows, words_per_row(cols)), dtype=torch.int32, device=W.device)
    _check(lib().tsenor_mask_noalloc(W.data_ptr(), _dtype_code(W), rows, cols, N, M, float(tau), iters,
                                     sweeps, out.data_ptr(), _stream_handle(stream)))
    return out


def tsenor_mask_safeguard(W, prev_mask, N: int, M: int, tau: float, iters: int, sweeps: int, out=None,
                          kept=None, stream=None):
    """tsenor_mask that keeps, per block, prev_mask where it is valid and keeps more |W|.

    ``kept`` (optional int64 CUDA tensor of one element) receives the count of
    blocks that kept prev_mask (added to its value).
    """
    import torch
    _check_2d_cuda(W, "W")
    rows, cols = W.shape
    if out is None:
        out = torch.empty((rows, words_per_row(cols)), dtype=torch.int32, device=W.device)
    _check(lib().tsenor_mask_safeguard(W.data_ptr(), _dtype_code(W), rows, cols, N, M, float(tau), iters, sweeps,
                                       prev_mask.data_ptr(), out.data_ptr(),
                                       kept.data_ptr() if kept is not None else None, _stream_handle(stream)))
    return out


def tsenor_mask_scores(scores, N: int, M: int, tau: float, iters: int, sweeps: int, out=None, stream=None):
    """Transposable N:M mask of an importance-score matrix (float32; magnitudes are used)."""
    import torch
    _check_2d_cuda(scores, "scores")
    if scores.dtype != torch.float32:
        raise TypeError("scores must be float32")
    rows, cols = scores.shape
    if out is None:
        out = torch.empty((rows, words_per_row(cols)), dtype=torch.int32, device=scores.device)
    _check(lib().tsenor_mask_scores(scores.data_ptr(), rows, cols, N, M, float(tau), iters, sweeps, out.data_ptr(),
                                    _stream_handle(stream)))
    return out


def tsenor_mask_host(W_host, N: int, M: int, tau: float, iters: int, sweeps: int, out=None, stream=None):
    """tsenor_mask of a HOST matrix into a HOST mask, the copies overlapped with the solve.

    W_host: contiguous 2-D CPU tensor (bfloat16 or float32), ideally pinned.
    Returns the (rows, ceil(cols/32)) int32 mask on the host (pinned when
    allocated here).  The result is complete once ``stream`` (default: the
    current CUDA stream) reaches this point, e.g. after its synchronize().
    """
    import torch
    if W_host.is_cuda or W_host.dim() != 2 or not W_host.is_contiguous():
        raise ValueError("W_host must be a contiguous 2-D CPU tensor")
    rows, cols = W_host.shape
    if out is None:
        out = torch.empty((rows, words_per_row(cols)), dtype=torch.int32, pin_memory=True)
    elif out.is_cuda or not out.is_contiguous() or out.numel() < rows * words_per_row(cols):
        raise ValueError("out must be a contiguous CPU int32 tensor of (rows, ceil(cols/32))")
    _check(lib().tsenor_mask_host(W_host.data_ptr(), _dtype_code(W_host), rows, cols, N, M, float(tau), iters,
                                  sweeps, out.data_ptr(), _stream_handle(stream)))
    return out


def tsenor_mask_padded(W, N: int, M: int, tau: float, iters: int, sweeps: int, out=None, stream=None):
    """tsenor_mask for any shape: W is zero-padded to multiples of M, the mask cropped back."""
    import torch
    _check_2d_cuda(W, "W")
    rows, cols = W.shape
    if out is None:
        out = torch.empty((rows, words_per_row(cols)), dtype=torch.int32, device=W.device)
    _check(lib().tsenor_mask_padded(W.data_ptr(), _dtype_code(W), rows, cols, N, M, float(tau), iters, sweeps,
                                    out.data_ptr(), _stream_handle(stream)))
    return out


def _warm_buffers(W, M, potentials, iters_used):
    import torch
    rows, cols = W.shape
    nb = (rows // M) * (cols // M) if M > 0 and rows % M == 0 and cols % M == 0 else 0
    if potentials is None:
        potentials = torch.empty((nb, 2 * M), dtype=torch.float32, device=W.device)
    elif (potentials.dtype != torch.float32 or not potentials.is_cuda or not potentials.is_contiguous()
          or potentials.numel() < nb * 2 * M):
        raise ValueError("potentials must be a contiguous float32 CUDA tensor of (n_blocks, 2M)")
    if iters_used is None:
        iters_used = torch.empty((nb,), dtype=torch.int32, device=W.device)
    elif (iters_used.dtype != torch.int32 or not iters_used.is_cuda or not iters_used.is_contiguous()
          or iters_used.numel() < nb):
        raise ValueError("iters_used must be a contiguous int32 CUDA tensor of n_blocks")
    return potentials, iters_used


def tsenor_mask_warm(W, N: int, M: int, tau: float, iters: int, sweeps: int, tol: float = 0.0, potentials=None,
                     warm: bool = False, iters_used=None, out=None, stream=None):
    """tsenor_mask with warm start and adaptive stopping.

    potentials: (n_blocks, 2M) float32 CUDA tensor, U then V per block
    (natural-log units), read when ``warm`` and overwritten with the final
    state (allocated when None; then ``warm`` must be False).  ``tol`` > 0
    stops a block after the first iteration whose row and column potentials
    are all within tol.  Returns (mask, potentials, iters_used).
    """
    import torch
    _check_2d_cuda(W, "W")
    rows, cols = W.shape
    if warm and potentials is None:
        raise ValueError("warm start needs potentials")
    potentials, iters_used = _warm_buffers(W, M, potentials, iters_used)
    if out is None:
        out = torch.empty((rows, words_per_row(cols)), dtype=torch.int32, device=W.device)
    _check(lib().tsenor_mask_warm(W.data_ptr(), _dtype_code(W), rows, cols, N, M, float(tau), iters, sweeps,
                                  float(tol), int(bool(warm)), potentials.data_ptr(), iters_used.data_ptr(),
                                  out.data_ptr(), _stream_handle(stream)))
    return out, potentials, iters_used


def tsenor_plan_warm(W, N: int, M: int, tau: float, iters: int, tol: float = 0.0, potentials=None,
                     warm: bool = False, iters_used=None, out=None, stream=None):
    """The plan of tsenor_mask_warm; returns (plan, potentials, iters_used)."""
    import torch
    _check_2d_cuda(W, "W")
    rows, cols = W.shape
    if warm and potentials is None:
        raise ValueError("warm start needs potentials")
    potentials, iters_used = _warm_buffers(W, M, potentials, iters_used)
    if out is None:
        out = torch.empty((rows, cols), dtype=torch.float32, device=W.device)
    _check(lib().tsenor_plan_warm(W.data_ptr(), _dtype_code(W), rows, cols, N, M, float(tau), iters, float(tol),
                                  int(bool(warm)), potentials.data_ptr(), iters_used.data_ptr(), out.data_ptr(),
                                  _stream_handle(stream)))
    return out, potentials, iters_used


def tsenor_plan(W, N: int, M: int, tau: float, iters: int, out=None, stream=None):
    """Fractional plan S (fp32, same shape as W) after `iters` Dykstra iterations."""
    import torch
    _check_2d_cuda(W, "W")
    rows, cols = W.shape
    if out is None:
        out = torch.empty((rows, cols), dtype=torch.float32, device=W.device)
    _check(lib().tsenor_plan(W.data_ptr(), _dtype_code(W), rows, cols, N, M, float(tau), iters,
                             out.data_ptr(), _stream_handle(stream)))
    return out


def tsenor_round(plan, W, N: int, M: int, sweeps: int, out=None, stream=None):
    """Rounding of a given fp32 plan into a mask (int32 words)."""
    import torch
    _check_2d_cuda(W, "W")
    _check_2d_cuda(plan, "plan")
    rows, cols = W.shape
    if plan.shape != W.shape or plan.dtype != torch.float32:
        raise ValueError("plan must be float32 with the shape of W")
    if out is None:
        out = torch.empty((rows, words_per_row(cols)), dtype=torch.int32, device=W.device)
    _check(lib().tsenor_round(plan.data_ptr(), W.data_ptr(), _dtype_code(W), rows, cols, N, M, sweeps,
                              out.data_ptr(), _stream_handle(stream)))
    return out


def tsenor_objective(W, mask, N: int, M: int, out=None, stream=None):
    """Per-block kept sum of |W| (fp64), NaN where a block row/column is not N:M."""
    import torch
    _check_2d_cuda(W, "W")
    rows, cols = W.shape
    if out is None:
        out = torch.empty(((rows // M) * (cols // M),), dtype=torch.float64, device=W.device)
    _check(lib().tsenor_objective(W.data_ptr(), _dtype_code(W), rows, cols, mask.data_ptr(), N, M,
                                  out.data_ptr(), _stream_handle(stream)))
    return out


def tsenor_error_count(stream=None) -> int:
    """Blocks that failed since the previous call (synchronises the stream).

    The C call reports a nonzero count with TSENOR_ERR_DEVICE; here the count
    itself is the result, so that status is not raised.
    """
    n = C.c_int64(0)
    status = lib().tsenor_error_count(_stream_handle(stream), C.byref(n))
    if status != -5:
        _check(status)
    return int(n.value)


__all__ = ["tsenor_mask", "tsenor_mask_host", "tsenor_mask_scores", "tsenor_mask_noalloc", "tsenor_mask_safeguard", "tsenor_mask_padded", "tsenor_mask_warm",
           "tsenor_plan", "tsenor_plan_warm", "tsenor_round", "tsenor_objective", "tsenor_error_count",
           "TsenorError", "lib", "words_per_row", "EXPORTS", "LIB_PATH"]
