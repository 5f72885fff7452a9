"""Build the CUDA libraries in-tree (sm_100a): sparse_mask_search_b200/libtsenor_b200.so, the
solver, and libtsenor_peaks.so, the pipe-throughput probes the benchmark's roofline uses."""
from __future__ import annotations

import glob
import os
import subprocess
import sys

HERE = os.path.dirname(os.path.abspath(__file__))
ROOT = os.path.dirname(HERE)
LIB = os.path.join(HERE, "libtsenor_b200.so")
MAIN = os.path.join(HERE, "csrc", "tsenor_api.cu")
PEAKS_LIB = os.path.join(HERE, "libtsenor_peaks.so")
PEAKS_SRC = os.path.join(HERE, "csrc", "peaks.cu")


def sources() -> list[str]:
    return sorted(glob.glob(os.path.join(HERE, "csrc", "*.cu")) + glob.glob(os.path.join(HERE, "csrc", "*.cuh"))
                  + glob.glob(os.path.join(ROOT, "include", "*.h")))


def nvcc() -> str:
    cand = os.path.join(os.environ.get("CUDA_HOME", "/usr/local/cuda"), "bin", "nvcc")
    return cand if os.path.exists(cand) else "nvcc"


def _compile(src: str, lib: str, deps: list[str], force: bool, verbose: bool) -> str:
    if not force and os.path.exists(lib):
        if os.path.getmtime(lib) >= max(os.path.getmtime(s) for s in deps):
            return lib
    cmd = [nvcc(), "-gencode", "arch=compute_100a,code=sm_100a", "-lineinfo", "-O3", "-std=c++17",
           "-Xcompiler", "-fPIC", "-shared", "-I", os.path.join(ROOT, "include"), src, "-o", lib + ".tmp"]
    if verbose:
        cmd.insert(1, "-Xptxas=-v")
    subprocess.run(cmd, check=True)
    os.replace(lib + ".tmp", lib)
    return lib


def build(force: bool = False, verbose: bool = False) -> str:
    """Both libraries; returns the solver's path."""
    _compile(PEAKS_SRC, PEAKS_LIB, [PEAKS_SRC], force, verbose)
    return _compile(MAIN, LIB, [s for s in sources() if s != PEAKS_SRC], force, verbose)


if __name__ == "__main__":
    print(build(force="--force" in sys.argv, verbose="-v" in sys.argv))
