"""Seeded synthetic weight matrices for transposable N:M mask search.

This module is the one piece of code that both the CUDA path (tests, bench)
and the CPU oracle (tests) consume.  It holds no arithmetic of the method:
it only draws numbers and rounds them to the storage dtype.

The pages (TSENOR review, "Core claim" and referee comment 1 on Fig. 3)
measure on blocks sampled from LLaMA3 weights, which are not available here.
The workloads below stand in for them with the shapes of a 7B-class
transformer and heavy-tailed value distributions typical of LLM weights.

Random numbers come from numpy's Philox4x32-10 counter-based generator
(Salmon et al., SC'11), keyed by an integer seed.  bf16 matrices are produced
by drawing fp32 values and rounding them to bf16 with round-to-nearest-even.
"""
from __future__ import annotations

import dataclasses
from typing import Iterator

import numpy as np

__all__ = [
    "Workload", "WORKLOADS", "STACK_7B_MATRICES", "rng", "f32_to_bf16_bits",
    "bf16_bits_to_f32", "make_matrix", "random_blocks", "stack_7b_layer",
]


@dataclasses.dataclass(frozen=True)
class Workload:
    """One synthetic matrix plus the solver settings it is measured with."""
    name: str
    rows: int
    cols: int
    dtype: str          # "f32" or "bf16"
    dist: str           # "normal", "t3_outlier_cols", "laplace_outliers"
    scale: float
    N: int
    M: int
    tau: float
    iters: int
    sweeps: int
    seed: int = 0

    @property
    def params(self) -> int:
        return self.rows * self.cols

    @property
    def n_blocks(self) -> int:
        return (self.rows // self.M) * (self.cols // self.M)


# The five measured settings.  Names give shape, dtype, value law and pattern.
WORKLOADS = {
    w.name: w for w in [
        Workload("w256x256_f32_normal_2of4", 256, 256, "f32", "normal", 1.0,
                 2, 4, 10.0, 200, 1),
        Workload("w4096x4096_bf16_normal_8of16", 4096, 4096, "bf16", "normal", 0.02,
                 8, 16, 20.0, 300, 4),
        Workload("w4096x11008_bf16_t3_16of32", 4096, 11008, "bf16", "t3_outlier_cols", 0.02,
                 16, 32, 20.0, 300, 8),
        Workload("w8192x28672_bf16_laplace_32of64", 8192, 28672, "bf16", "laplace_outliers", 0.014,
                 32, 64, 30.0, 400, 8),
        # one matrix of the 7B-shaped stack's settings (the q projection shape, seed 0)
        Workload("w4096x4096_bf16_normal_4of8", 4096, 4096, "bf16", "normal", 0.02,
                 4, 8, 20.0, 200, 4),
    ]
}

# 7B-shaped stack: per layer q,k,v,o (4096x4096), gate,up (11008x4096), down (4096x11008).
STACK_7B_MATRICES = [
    ("q", 4096, 4096), ("k", 4096, 4096), ("v", 4096, 4096), ("o", 4096, 4096),
    ("gate", 11008, 4096), ("up", 11008, 4096), ("down", 4096, 11008),
]
STACK_7B_LAYERS = 32
STACK_7B_SETTINGS = dict(N=4, M=8, tau=20.0, iters=200, sweeps=4)


def rng(seed: int) -> np.random.Generator:
    """Philox4x32-10 stream keyed by ``seed``."""
    return np.random.Generator(np.random.Philox(key=int(seed)))


def f32_to_bf16_bits(x: np.ndarray) -> np.ndarray:
    """Round finite fp32 values to bf16 (round to nearest, ties to even).

    Returns the 16-bit patterns as uint16.  The inputs drawn here are finite,
    so NaN payload handling is not needed.
    """
    u = np.ascontiguousarray(x, dtype=np.float32).view(np.uint32)
    lsb = (u >> np.uint32(16)) & np.uint32(1)
    rounded = u + np.uint32(0x7FFF) + lsb
    return (rounded >> np.uint32(16)).astype(np.uint16)


def bf16_bits_to_f32(b: np.ndarray) -> np.ndarray:
    """Exact widening of bf16 bit patterns to fp32."""
    return (np.asarray(b, dtype=np.uint16).astype(np.uint32) << np.uint32(16)).view(np.float32)


def _draw(g: np.random.Generator, dist: str, rows: int, cols: int, scale: float) -> np.ndarray:
    if dist == "normal":
        return (g.standard_normal((rows, cols), dtype=np.float32) * np.float32(scale))
    if dist == "t3_outlier_cols":
        # Student-t with 3 degrees of freedom, scaled; 1% of the columns
        # (picked by a seeded shuffle) are multiplied by 10.
        w = g.standard_t(3.0, size=(rows, cols)).astype(np.float32) * np.float32(scale)
        n_out = int(cols * 0.01)
        cols_out = g.permutation(cols)[:n_out]
        w[:, cols_out] *= np.float32(10.0)
        return w
    if dist == "laplace_outliers":
        # Laplace(0, scale); each entry independently becomes a x20 outlier
        # with probability 0.001.
        w = g.laplace(0.0, scale, size=(rows, cols)).astype(np.float32)
        hit = g.random((rows, cols), dtype=np.float32) < np.float32(0.001)
        w[hit] *= np.float32(20.0)
        return w
    if dist == "uniform":
        return g.random((rows, cols), dtype=np.float32) * np.float32(scale)
    raise ValueError(f"unknown distribution {dist!r}")


def make_matrix(rows: int, cols: int, dtype: str, dist: str, scale: float, seed: int):
    """Draw one matrix.

    Returns ``(storage, values)``: ``storage`` is what a caller hands to the
    library (uint16 bf16 bit patterns, or float32), ``values`` is the exact
    fp32 value of every stored element (what the oracle consumes).
    """
    w = _draw(rng(seed), dist, rows, cols, scale)
    if dtype == "bf16":
        bits = f32_to_bf16_bits(w)
        return bits, bf16_bits_to_f32(bits)
    if dtype == "f32":
        w = np.ascontiguousarray(w, dtype=np.float32)
        return w, w
    raise ValueError(f"unknown dtype {dtype!r}")


def workload_matrix(w: Workload, seed: int | None = None):
    """The matrix of a named workload (see ``make_matrix`` for the result)."""
    return make_matrix(w.rows, w.cols, w.dtype, w.dist, w.scale, w.seed if seed is None else seed)


def stack_7b_layer(layer: int) -> Iterator[tuple[str, np.ndarray, np.ndarray]]:
    """The seven bf16 matrices of one layer of the 7B-shaped stack.

    Values are N(0, 0.02); matrix ``k`` of layer ``l`` uses seed 1000*l + k.
    """
    for k, (name, r, c) in enumerate(STACK_7B_MATRICES):
        bits, vals = make_matrix(r, c, "bf16", "normal", 0.02, 1000 * layer + k)
        yield name, bits, vals


def random_blocks(n: int, M: int, seed: int, dist: str = "normal", dtype: str = "f32",
                  scale: float = 1.0) -> np.ndarray:
    """``n`` independent MxM blocks laid side by side as an (M, n*M) matrix.

    Returns the exact fp32 values (bf16-rounded when ``dtype == 'bf16'``).
    """
    _, vals = make_matrix(M, n * M, dtype, dist, scale, seed)
    return vals
