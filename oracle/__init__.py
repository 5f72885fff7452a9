"""ctypes wrapper around the CPU oracle (test infrastructure).

Only the test suite, the smoke check and the CPU-baseline leg of the
benchmark use this module.  The CUDA library never imports it.
See tsenor_oracle.c for what each routine computes and which passage of
the TSENOR review it follows.
"""
from __future__ import annotations

import ctypes as C
import os

import numpy as np

from . import build as _build

_lib = None


class Stats(C.Structure):
    _fields_ = [("repairs", C.c_int64), ("ls_swaps", C.c_int64),
                ("failures", C.c_int64), ("short_after_greedy", C.c_int64)]

    def as_dict(self):
        return {k: int(getattr(self, k)) for k, _ in self._fields_}


def lib():
    global _lib
    if _lib is None:
        path = _build.build()
        L = C.CDLL(path)
        p = C.c_void_p
        i64, i32, f64 = C.c_int64, C.c_int, C.c_double
        L.oracle_block_plan.argtypes = [p, i32, i32, f64, i32, p]
        L.oracle_block_round.argtypes = [p, p, i32, i32, i32, i32, p, C.POINTER(Stats)]
        L.oracle_block_opt.argtypes = [p, i32, i32, p]
        L.oracle_block_opt.restype = f64
        L.oracle_plan.argtypes = [p, i64, i64, i32, i32, f64, i32, p, i32]
        L.oracle_round.argtypes = [p, p, i64, i64, i32, i32, i32, p, i32, C.POINTER(Stats)]
        L.oracle_mask.argtypes = [p, i64, i64, i32, i32, f64, i32, i32, p, p, i32, C.POINTER(Stats)]
        L.oracle_objective.argtypes = [p, p, i64, i64, i32, i32, p]
        L.oracle_opt.argtypes = [p, i64, i64, i32, i32, p, p, i32]
        L.oracle_threads_used.argtypes = [i32]
        L.oracle_safeguard.argtypes = [p, p, p, i64, i64, i32, i32, p]
        L.oracle_safeguard.restype = i64
        L.oracle_block_plan_ext.argtypes = [p, i32, i32, f64, i32, f64, i32, p, p]
        L.oracle_solve_ext.argtypes = [p, i64, i64, i32, i32, f64, i32, i32, f64, i32, p, p, p, p, i32,
                                       C.POINTER(Stats)]
        _lib = L
    return _lib


def _f32(x):
    return np.ascontiguousarray(x, dtype=np.float32)


def _ptr(a):
    return a.ctypes.data_as(C.c_void_p) if a is not None else None


def _check(rc):
    if rc != 0:
        raise ValueError(f"oracle rejected the arguments (code {rc})")


def threads_used(threads: int = 0) -> int:
    return lib().oracle_threads_used(threads)


def block_plan(a, N, tau, iters):
    """Plan S (fp64, MxM) of one block of magnitudes ``a``."""
    a = _f32(np.abs(a))
    M = a.shape[0]
    S = np.empty((M, M), dtype=np.float64)
    _check(lib().oracle_block_plan(_ptr(a), N, M, float(tau), iters, _ptr(S)))
    return S


def block_round(key, a, N, sweeps, stage=3):
    """Binary block mask from fp32 keys; stage 1 greedy, 2 +repair, 3 +local search."""
    key = _f32(key); a = _f32(np.abs(a))
    M = a.shape[0]
    s = np.zeros((M, M), dtype=np.uint8)
    st = Stats()
    rc = lib().oracle_block_round(_ptr(key), _ptr(a), N, M, sweeps, stage, _ptr(s), C.byref(st))
    return s, rc, st.as_dict()


def block_opt(a, N):
    """Exact optimum (value, mask) of one block by min-cost flow."""
    a = _f32(np.abs(a))
    M = a.shape[0]
    f = np.zeros((M, M), dtype=np.uint8)
    v = lib().oracle_block_opt(_ptr(a), N, M, _ptr(f))
    return v, f


def plan(W, N, M, tau, iters, threads=0):
    W = _f32(W)
    rows, cols = W.shape
    out = np.empty((rows, cols), dtype=np.float64)
    _check(lib().oracle_plan(_ptr(W), rows, cols, N, M, float(tau), iters, _ptr(out), threads))
    return out


def words_per_row(cols: int) -> int:
    return (cols + 31) // 32


def round_plan(key, W, N, M, sweeps, threads=0):
    """Oracle rounding of a given fp32 plan; returns (mask words, stats)."""
    key = _f32(key); W = _f32(W)
    rows, cols = W.shape
    mask = np.zeros((rows, words_per_row(cols)), dtype=np.uint32)
    st = Stats()
    _check(lib().oracle_round(_ptr(key), _ptr(W), rows, cols, N, M, sweeps, _ptr(mask), threads,
                              C.byref(st)))
    return mask, st.as_dict()


def mask(W, N, M, tau, iters, sweeps, threads=0, want_keys=False):
    """Full pipeline; returns (mask words, keys or None, stats)."""
    W = _f32(W)
    rows, cols = W.shape
    m = np.zeros((rows, words_per_row(cols)), dtype=np.uint32)
    keys = np.empty((rows, cols), dtype=np.float32) if want_keys else None
    st = Stats()
    _check(lib().oracle_mask(_ptr(W), rows, cols, N, M, float(tau), iters, sweeps, _ptr(m),
                             _ptr(keys), threads, C.byref(st)))
    return m, keys, st.as_dict()


def objective(W, mask_words, N, M):
    W = _f32(W)
    rows, cols = W.shape
    mw = np.ascontiguousarray(mask_words, dtype=np.uint32)
    out = np.empty((rows // M) * (cols // M), dtype=np.float64)
    _check(lib().oracle_objective(_ptr(W), _ptr(mw), rows, cols, N, M, _ptr(out)))
    return out


def opt(W, N, M, threads=0, want_mask=False):
    """Exact per-block optimum by min-cost flow; returns (values, mask words or None)."""
    W = _f32(W)
    rows, cols = W.shape
    out = np.empty((rows // M) * (cols // M), dtype=np.float64)
    m = np.zeros((rows, words_per_row(cols)), dtype=np.uint32) if want_mask else None
    _check(lib().oracle_opt(_ptr(W), rows, cols, N, M, _ptr(out), _ptr(m), threads))
    return out, m


def safeguard(W, prev_mask, new_mask, N, M):
    """Per block keep the previous mask if valid and strictly heavier; returns (mask, kept blocks)."""
    W = _f32(W)
    rows, cols = W.shape
    prev = np.ascontiguousarray(prev_mask, dtype=np.uint32)
    new = np.ascontiguousarray(new_mask, dtype=np.uint32)
    out = np.empty_like(new)
    kept = lib().oracle_safeguard(_ptr(W), _ptr(prev), _ptr(new), rows, cols, N, M, _ptr(out))
    if kept < 0:
        raise ValueError("oracle rejected the arguments")
    return out, int(kept)


def block_plan_ext(a, N, tau, iters, tol=0.0, uv=None):
    """Plan of one block with warm start / adaptive stopping.

    uv: starting potentials (2M, U then V, nats) or None for a cold start.
    Returns (S fp64 MxM, final potentials (2M,), iterations run).
    """
    a = _f32(np.abs(a))
    M = a.shape[0]
    S = np.empty((M, M), dtype=np.float64)
    warm = uv is not None
    buf = np.array(uv, dtype=np.float64).copy() if warm else np.zeros(2 * M, dtype=np.float64)
    t = lib().oracle_block_plan_ext(_ptr(a), N, M, float(tau), iters, float(tol), int(warm), _ptr(buf), _ptr(S))
    if t < 0:
        raise ValueError("oracle rejected the arguments")
    return S, buf, int(t)


def solve_ext(W, N, M, tau, iters, sweeps, tol=0.0, potentials=None, want_plan=False, want_mask=True,
              threads=0):
    """Matrix-level warm start / adaptive stopping.

    potentials: None (cold) or (n_blocks, 2M) starting potentials (nats).
    Returns dict(mask, potentials (n_blocks, 2M) fp64, iters_used (n_blocks,), plan, stats).
    """
    W = _f32(W)
    rows, cols = W.shape
    nb = (rows // M) * (cols // M)
    warm = potentials is not None
    uv = (np.array(potentials, dtype=np.float64).reshape(nb, 2 * M).copy() if warm
          else np.zeros((nb, 2 * M), dtype=np.float64))
    used = np.zeros(nb, dtype=np.int32)
    plan_out = np.empty((rows, cols), dtype=np.float64) if want_plan else None
    m = np.zeros((rows, words_per_row(cols)), dtype=np.uint32) if want_mask else None
    st = Stats()
    _check(lib().oracle_solve_ext(_ptr(W), rows, cols, N, M, float(tau), iters, sweeps, float(tol), int(warm),
                                  _ptr(uv), _ptr(used), _ptr(plan_out), _ptr(m), threads, C.byref(st)))
    return {"mask": m, "potentials": uv, "iters_used": used, "plan": plan_out, "stats": st.as_dict()}


def unpack(mask_words, cols):
    """(rows, words) uint32 -> (rows, cols) uint8, bit k of word w = column 32w+k."""
    mw = np.ascontiguousarray(mask_words, dtype=np.uint32)
    bits = np.unpackbits(mw.view(np.uint8), axis=1, bitorder="little")
    return bits[:, :cols]


def pack(bits):
    """(rows, cols) 0/1 -> (rows, words) uint32 with zero padding bits."""
    b = np.ascontiguousarray(bits, dtype=np.uint8)
    rows, cols = b.shape
    wpr = words_per_row(cols)
    padded = np.zeros((rows, wpr * 32), dtype=np.uint8)
    padded[:, :cols] = b
    return np.packbits(padded, axis=1, bitorder="little").view(np.uint32).reshape(rows, wpr)


def blocks_view(x, M):
    """(rows, cols) -> (rows/M, cols/M, M, M) block view."""
    rows, cols = x.shape
    return x.reshape(rows // M, M, cols // M, M).transpose(0, 2, 1, 3)
