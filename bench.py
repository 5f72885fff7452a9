#!/usr/bin/env python3
"""Throughput of transposable N:M mask generation on B200 GPUs.

One step = one call of the public entry point tsenor_mask over one whole
synthetic weight matrix (Dykstra plan, sort, greedy, repair, local search,
bit packing).  Default workload: 4096 x 11008 bf16, Student-t(3) x 0.02 with
1% outlier columns x10, transposable 16:32, tau = 20, T = 300, L = 8.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl ours|reference]

Under torchrun every rank solves its own matrix of the same shape (a
different seed): blocks are independent, so there is no data-path
collective and the run scales weakly.  Rank 0 prints one JSON line.
"""
from __future__ import annotations

import argparse
import datetime
import hashlib
import json
import os
import statistics
import subprocess
import sys
import time

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

import numpy as np  # noqa: E402

import synth  # noqa: E402

DEFAULT_WORKLOAD = "w4096x11008_bf16_t3_16of32"
METRIC = "transposable N:M mask Gparams/s at 1 B200 (% of roofline); mean gap to exact opt"
STACK = "stack7b"                  # 32 layers x 7 matrices, 4:8, one pass = one step
SM_COUNT = 148
FP32_LANES_PER_CLK_PER_SM = 128   # fp32 add / mul / fma results per clock per SM (FMA pipe)
MUFU_LANES_PER_CLK_PER_SM = 16    # ex2 / lg2 / rcp results per clock per SM (MUFU pipe)
# The method's work per parameter and Dykstra iteration as the survey of the
# pages counts it: 1 + 2/M exponentials and logarithms (one exponential per
# entry with the row step's exponentials reused for the column sums, M logs
# per row step and M per column step) on the MUFU pipe, and 8 FP32 operations
# (min/max split, subtract, row and column accumulation, row scaling, two
# log-offset adds, clip add).
SURVEY_FP32_OPS_PER_ENTRY_ITER = 8
# This implementation's FMA-pipe work per entry and iteration: the row-sum
# add, the column-sum fma and the column scaling (the row scaling is one
# threshold per row; the clip min(F, th) runs on the ALU pipe and is not
# counted).  Stricter than the survey's count: it measures the kernels
# against the pipe they actually load.
FP32_OPS_PER_ENTRY_ITER = 3
SM_MAX_MHZ_FALLBACK = 1965.0
L2_FLUSH_BYTES = 256 << 20
SECONDARY = ("w256x256_f32_normal_2of4", "w4096x4096_bf16_normal_8of16", "w8192x28672_bf16_laplace_32of64", STACK)


def parse_args(argv=None):
    p = argparse.ArgumentParser(description=__doc__, formatter_class=argparse.RawDescriptionHelpFormatter)
    p.add_argument("--gpus", type=int, default=1)
    p.add_argument("--steps", type=int, default=60)
    p.add_argument("--warmup", type=int, default=5)
    p.add_argument("--impl", choices=["ours", "reference"], default="ours")
    p.add_argument("--workload", default=DEFAULT_WORKLOAD, choices=sorted(synth.WORKLOADS) + [STACK])
    p.add_argument("--layers", type=int, default=synth.STACK_7B_LAYERS, help="layers of the 7B stack")
    p.add_argument("--cpu-seconds", type=float, default=15.0,
                   help="target CPU time of the bounded oracle sample")
    p.add_argument("--no-cpu-baseline", action="store_true")
    p.add_argument("--no-secondary", action="store_true",
                   help="skip the record of the other workloads (2:4, 8:16, 32:64, the 7B-shaped stack)")
    p.add_argument("--no-gap", action="store_true", help="skip the exact-optimum gap of the GPU masks")
    p.add_argument("--mode", choices=["plain", "warm", "gap"], default="plain",
                   help="warm: outer-loop re-solves with warm start and adaptive stopping (tsenor_mask_warm); "
                        "gap: quality only, the GPU masks against the exact optimum on all blocks (or a "
                        "seeded sample of --gap-blocks)")
    p.add_argument("--gap-blocks", type=int, default=0,
                   help="--mode gap: seeded sample size (0 = every block)")
    p.add_argument("--tol", type=float, default=1e-3, help="stop tolerance of --mode warm (nats)")
    p.add_argument("--shape", default=None,
                   help="ROWSxCOLS: the workload's values and settings at another shape (small profiling cases)")
    p.add_argument("--drift", type=float, default=0.01,
                   help="--mode warm: relative change of W between consecutive outer steps")
    return p.parse_args(argv)


# --------------------------------------------------------------------------- helpers

def measured_peaks():
    try:
        with open(os.path.join(ROOT, "MEASURED_PEAKS.json")) as f:
            return json.load(f)
    except OSError:
        return {}


def fp32_peak_tops(sm_mhz):
    return SM_COUNT * FP32_LANES_PER_CLK_PER_SM * sm_mhz * 1e6 / 1e12


def mufu_peak_tops(sm_mhz):
    return SM_COUNT * MUFU_LANES_PER_CLK_PER_SM * sm_mhz * 1e6 / 1e12


def survey_ops_per_param(M, iters):
    """(MUFU ops, FP32 ops) per parameter of one solve, as the survey counts the method's work."""
    return iters * (1.0 + 2.0 / M), float(iters * SURVEY_FP32_OPS_PER_ENTRY_ITER)


def roofline_record(params, M, iters, ms, peaks):
    """Fractions of the binding roofline for one solve of `params` parameters in `ms`.

    peaks: {"fma_tops", "mufu_tops"} (TOP/s).  The survey's bound is the slower
    of the MUFU time (T(1 + 2/M) ops per parameter) and the FP32 time (8T);
    frac_fma counts this implementation's 3T FMA-pipe operations instead.
    """
    t = ms / 1e3
    sfu_pp, fp32_pp = survey_ops_per_param(M, iters)
    t_sfu = params * sfu_pp / (peaks["mufu_tops"] * 1e12)
    t_fp32 = params * fp32_pp / (peaks["fma_tops"] * 1e12)
    t_fma = params * iters * FP32_OPS_PER_ENTRY_ITER / (peaks["fma_tops"] * 1e12)
    sfu_binds = t_sfu >= t_fp32
    ops_pp, peak = (sfu_pp, peaks["mufu_tops"]) if sfu_binds else (fp32_pp, peaks["fma_tops"])
    achieved = params * ops_pp / t / 1e12
    return {"bound": "alu", "binding_pipe": "mufu" if sfu_binds else "fp32", "achieved": achieved, "peak": peak,
            "unit": "TOP/s", "frac": achieved / peak,
            "frac_survey": {"mufu": t_sfu / t, "fp32": t_fp32 / t, "binding": max(t_sfu, t_fp32) / t},
            "frac_fma": t_fma / t,
            "ops": {"mufu_per_param": sfu_pp, "fp32_per_param": fp32_pp,
                    "fma_pipe_per_param": float(iters * FP32_OPS_PER_ENTRY_ITER),
                    "basis": f"survey: T(1+2/M) MUFU and 8T FP32 ops per param; implementation: "
                             f"{FP32_OPS_PER_ENTRY_ITER}T FMA-pipe ops per param (T = {iters}, M = {M})"}}


def measure_pipe_peaks(dev, stream, sampler=None):
    """FP32-FMA and MUFU throughput of this GPU, measured by the repository's own probe
    kernels (libtsenor_peaks.so): independent chains, 8 CTAs of 256 threads per SM, best
    of 5 launches timed with CUDA events on `stream`."""
    import ctypes
    import torch
    import sparse_mask_search_b200.build as lb
    L = ctypes.CDLL(lb.PEAKS_LIB)
    L.tsenor_peak_ops.restype = ctypes.c_longlong
    L.tsenor_peak_ops.argtypes = [ctypes.c_int] * 3
    L.tsenor_peak_launch.argtypes = [ctypes.c_int] * 4 + [ctypes.c_void_p, ctypes.c_void_p]
    blocks, threads = SM_COUNT * 8, 256
    out = torch.empty(blocks, dtype=torch.float32, device=dev)
    res = {}
    t0 = time.time()
    for kind, name, iters in ((0, "fma_tops", 12000), (1, "mufu_tops", 1600)):
        ops = L.tsenor_peak_ops(blocks, threads, iters)
        best = None
        for k in range(7):
            a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
            a.record(stream)
            rc = L.tsenor_peak_launch(kind, blocks, threads, iters, out.data_ptr(), stream.cuda_stream)
            b.record(stream)
            if rc != 0:
                raise RuntimeError(f"peak probe launch failed ({rc})")
            torch.cuda.synchronize(dev)
            if k >= 2:
                ms = a.elapsed_time(b)
                best = ms if best is None else min(best, ms)
        res[name] = ops / (best / 1e3) / 1e12
        res[name.replace("tops", "ms")] = best
    t1 = time.time()
    res["method"] = ("own probe kernels: 8 independent fma.rn.f32 / ex2.approx.ftz.f32 chains per thread, "
                     f"{blocks} CTAs x {threads} threads, best of 5 launches (CUDA events)")
    if sampler is not None:
        res["clocks"] = sampler.window(t0, t1)
    return res


def source_digest():
    """Digest of the kernel sources (the device-code headers); a profiled
    traffic figure is used only while it matches."""
    h = hashlib.sha256()
    csrc = os.path.join(ROOT, "sparse_mask_search_b200", "csrc")
    for fn in sorted(os.listdir(csrc)):
        if not fn.endswith(".cuh"):
            continue
        with open(os.path.join(csrc, fn), "rb") as f:
            h.update(fn.encode() + f.read())
    return h.hexdigest()[:16]


def profiled_traffic(kernel_key):
    """DRAM bytes per launch from a committed ncu summary, if taken on today's sources."""
    path = os.path.join(ROOT, "profiles", "traffic.json")
    try:
        with open(path) as f:
            rec = json.load(f).get(kernel_key)
    except (OSError, ValueError):
        return None
    if not rec or rec.get("source_digest") != source_digest():
        return None
    return rec.get("dram_bytes_per_launch")


class ClockSampler:
    """SM clock and clock-event reasons of one GPU, polled through NVML every
    2 ms by a background thread (nvidia-smi at 100 ms when NVML is missing)."""
    REASONS = (("hw_slowdown", 0x8), ("hw_thermal_slowdown", 0x40), ("sw_thermal_slowdown", 0x20),
               ("sw_power_cap", 0x4), ("hw_power_brake_slowdown", 0x80))

    def __init__(self, uuid):
        import threading
        self.samples = []            # (t, sm_mhz, reasons bits, power W or None)
        self.t0 = self.t1 = None
        self.max_mhz = None
        self.source = "nvml"
        self._stop = threading.Event()
        self._proc = None
        try:
            import pynvml
            pynvml.nvmlInit()
            self._nv = pynvml
            self._h = pynvml.nvmlDeviceGetHandleByUUID(uuid)
            self.max_mhz = float(pynvml.nvmlDeviceGetMaxClockInfo(self._h, pynvml.NVML_CLOCK_SM))
            self._thread = threading.Thread(target=self._poll, daemon=True)
            self._thread.start()
        except Exception:              # no NVML: nvidia-smi, coarser
            self._nv = None
            self.source = "nvidia-smi"
            try:
                self._proc = subprocess.Popen(
                    ["nvidia-smi", "-i", uuid, "--query-gpu=timestamp,clocks.sm,clocks.max.sm,power.draw,"
                     "clocks_event_reasons.active", "--format=csv,noheader,nounits", "-lms", "100"],
                    stdout=subprocess.PIPE, stderr=subprocess.DEVNULL, text=True)
            except OSError:
                self._proc = None

    def _poll(self):
        nv, h = self._nv, self._h
        k = 0
        while not self._stop.is_set():
            t = time.time()
            try:
                mhz = float(nv.nvmlDeviceGetClockInfo(h, nv.NVML_CLOCK_SM))
                bits = int(nv.nvmlDeviceGetCurrentClocksEventReasons(h))
                pw = nv.nvmlDeviceGetPowerUsage(h) / 1000.0 if k % 10 == 0 else None
            except Exception:
                break
            self.samples.append((t, mhz, bits, pw))
            k += 1
            time.sleep(0.002)

    def mark_start(self):
        self.t0 = time.time()

    def mark_end(self):
        self.t1 = time.time()

    def window(self, t0, t1):
        """Summary of the samples taken between t0 and t1 (time.time())."""
        use = [x for x in self.samples if t0 - 0.003 <= x[0] <= t1 + 0.003]
        mhz = [x[1] for x in use]
        reasons = sorted({n for x in use for n, bit in self.REASONS if x[2] & bit})
        pw = [x[3] for x in use if x[3] is not None]
        return {"sm_mhz": statistics.median(mhz) if mhz else None, "sm_mhz_min": min(mhz) if mhz else None,
                "sm_max_mhz": self.max_mhz, "reasons": reasons, "samples": len(use),
                "power_w_max": max(pw) if pw else None}

    def stop(self):
        if self._nv is not None:
            self._stop.set()
            self._thread.join(timeout=2)
            out = self.window(self.t0, self.t1)
            out.update(samples_in_timed_region=out["samples"], source="nvml, 2 ms polling",
                       timed_region_s=self.t1 - self.t0)
            return out
        if self._proc is None:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["clock sampling unavailable"], "samples": 0}
        time.sleep(0.25)
        self._proc.terminate()
        try:
            out, _ = self._proc.communicate(timeout=5)
        except subprocess.TimeoutExpired:
            self._proc.kill()
            out, _ = self._proc.communicate()
        rows = []
        for line in out.splitlines():
            parts = [x.strip() for x in line.split(",")]
            if len(parts) < 5:
                continue
            try:
                ts = datetime.datetime.strptime(parts[0], "%Y/%m/%d %H:%M:%S.%f").timestamp()
                rows.append((ts, float(parts[1]), int(parts[4], 16), float(parts[3])))
                self.max_mhz = float(parts[2])
            except ValueError:
                continue
        self.samples = rows
        inside = self.window(self.t0, self.t1)
        if not inside["samples"]:
            inside = self.window(-1e30, 1e30)
        inside.update(samples_in_timed_region=inside["samples"], source="nvidia-smi, 100 ms")
        return inside


def gpu_uuid(dev):
    import torch
    uuid = str(torch.cuda.get_device_properties(dev).uuid)
    return uuid if uuid.startswith("GPU-") else "GPU-" + uuid


def workload_of(args):
    """The named workload, at --shape ROWSxCOLS when given."""
    w = synth.WORKLOADS[args.workload]
    if args.shape:
        import dataclasses
        r, c = (int(x) for x in args.shape.lower().split("x"))
        if r <= 0 or c <= 0 or r % w.M or c % w.M:
            raise SystemExit(f"--shape {args.shape}: rows and cols must be positive multiples of M = {w.M}")
        w = dataclasses.replace(w, rows=r, cols=c, name=f"{w.name}@{r}x{c}")
    return w


def rank_seed(w, rank: int) -> int:
    """Each rank solves its own matrix of the workload's shape (weak scaling)."""
    return w.seed + rank


def max_over_ranks(value: float, device, world: int) -> float:
    """Max of a per-rank scalar over all ranks (the step time of the slowest rank)."""
    if world <= 1:
        return float(value)
    import torch
    import torch.distributed as dist
    t = torch.tensor([value], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def aggregate_gparams(params_per_rank: int, world: int, max_ms: float) -> float:
    """Whole-job throughput: parameters solved by all ranks over the slowest rank's time."""
    return params_per_rank * world / (max_ms / 1e3) / 1e9


def to_device(storage, dtype, device):
    import torch
    if dtype == "bf16":
        return torch.from_numpy(storage.view(np.int16)).view(torch.bfloat16).to(device)
    return torch.from_numpy(storage).to(device)


# --------------------------------------------------------------------------- CPU (oracle) legs

def oracle_sample(vals, w, seconds, cores=0):
    """Oracle on the first k block-rows of the matrix, k sized for ~`seconds` of CPU work."""
    import oracle
    M = w.M
    nbr = w.rows // M
    t = time.perf_counter()
    oracle.mask(vals[:M], w.N, M, w.tau, w.iters, w.sweeps, threads=cores)
    t1 = max(time.perf_counter() - t, 1e-3)
    k = int(max(1, min(nbr, seconds / t1)))
    sub = np.ascontiguousarray(vals[:k * M])
    t = time.perf_counter()
    m_ref, _, st = oracle.mask(sub, w.N, M, w.tau, w.iters, w.sweeps, threads=cores)
    dt = time.perf_counter() - t
    return sub, k, dt, m_ref, st


def cpu_baseline_leg(vals, w, seconds):
    """The oracle as it stands, timed on a bounded sample of the workload on the host cores."""
    import oracle
    cores = oracle.threads_used(0)
    sub, k, dt, m_ref, st = oracle_sample(vals, w, seconds)
    params = sub.shape[0] * sub.shape[1]
    return {"value": params / dt / 1e9, "unit": "Gparams/s", "cores": cores, "kind": "oracle",
            "sample": f"first {k} of {w.rows // w.M} block-rows ({k * (w.cols // w.M)} blocks, "
                      f"{params} params) of the same matrix; plain C, OpenMP over blocks",
            "seconds": dt}


def gap_record(vals, mask_words, N, M, max_blocks=0, seed=12345):
    """Gap of the GPU masks to the exact per-block optimum (the oracle's min-cost flow):
    every block, or a seeded sample of whole block-rows holding at least max_blocks blocks."""
    import oracle
    rows, cols = vals.shape
    nbr, nbc = rows // M, cols // M
    if max_blocks and max_blocks < nbr * nbc:
        k = -(-max_blocks // nbc)
        sel = np.sort(synth.rng(seed).permutation(nbr)[:k])
    else:
        sel = np.arange(nbr)
    rows_idx = (sel[:, None] * M + np.arange(M)[None, :]).ravel()
    sub = np.ascontiguousarray(vals[rows_idx])
    t0 = time.perf_counter()
    opt, _ = oracle.opt(sub, N, M)
    kept = oracle.objective(sub, np.ascontiguousarray(mask_words[rows_idx]), N, M)
    if np.isnan(kept).any():
        raise RuntimeError("invalid GPU mask block")
    total = oracle.blocks_view(np.abs(sub).astype(np.float64), M).sum(axis=(2, 3)).ravel()
    gap = (opt - kept) / opt
    gp = (opt - kept) / np.maximum(total - opt, 1e-30)
    return {"mean": float(gap.mean()), "max": float(gap.max()), "median": float(np.median(gap)),
            "mean_vs_pruned_mass": float(gp.mean()), "max_vs_pruned_mass": float(gp.max()),
            "blocks": int(opt.size), "of_blocks": int(nbr * nbc),
            "sample": "all blocks" if len(sel) == nbr else f"{len(sel)} seeded whole block-rows",
            "definition": "(opt - kept)/opt per block, opt = exact min-cost-flow optimum",
            "host_seconds": time.perf_counter() - t0, "pages_claim": "1-10% of optimal"}


def run_reference(args, rank, world):
    """The oracle as it stands, on the host cores, on bounded samples of the workload."""
    if rank != 0:
        return
    import oracle
    if args.workload == STACK:
        # a bounded sample of the stack: block-rows of layer 0's first matrix
        st = synth.STACK_7B_SETTINGS
        name, r, c = synth.STACK_7B_MATRICES[0]
        w = synth.Workload(f"stack7b_layer0_{name}", r, c, "bf16", "normal", 0.02, st["N"], st["M"], st["tau"],
                           st["iters"], st["sweeps"], 0)
        _, vals = synth.make_matrix(r, c, "bf16", "normal", 0.02, 0)
    else:
        w = synth.WORKLOADS[args.workload]
        _, vals = synth.workload_matrix(w)
    cores = oracle.threads_used(0)
    M = w.M
    t = time.perf_counter()
    oracle.mask(vals[:M], w.N, M, w.tau, w.iters, w.sweeps)
    t1 = max(time.perf_counter() - t, 1e-3)
    budget = 120.0 / max(1, args.steps + args.warmup)
    k = int(max(1, min(w.rows // M, budget / t1)))
    sub = np.ascontiguousarray(vals[:k * M])
    for _ in range(args.warmup):
        oracle.mask(sub, w.N, M, w.tau, w.iters, w.sweeps)
    times = []
    for _ in range(args.steps):
        t = time.perf_counter()
        oracle.mask(sub, w.N, M, w.tau, w.iters, w.sweeps)
        times.append(time.perf_counter() - t)
    params = sub.shape[0] * sub.shape[1]
    step = statistics.mean(times)
    value = params / step / 1e9
    line = {"impl": "reference", "metric": METRIC,
            "value": value, "unit": "Gparams/s", "n_gpus": world, "steps": args.steps, "warmup": args.warmup,
            "ms_per_step": step * 1e3, "higher_is_better": True, "scaling": "weak", "vs_baseline": None,
            "dtype": "f64", "data": "synthetic",
            "config": {"workload": w.name, "rows": w.rows, "cols": w.cols, "N": w.N, "M": w.M, "tau": w.tau,
                       "iters": w.iters, "sweeps": w.sweeps, "sample_block_rows": k},
            "cpu_baseline": {"value": value, "unit": "Gparams/s", "cores": cores, "kind": "oracle",
                             "sample": f"first {k} block-rows ({params} params) per step"},
            "e2e": {"value": value, "unit": "Gparams/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}}
    print(json.dumps(line), flush=True)


# --------------------------------------------------------------------------- 7B stack

def run_stack(args, rank, world):
    """One step = tsenor_mask over every matrix of the 7B-shaped stack, layer by layer."""
    import torch
    import sparse_mask_search_b200 as tsl
    local = int(os.environ.get("LOCAL_RANK", "0"))
    torch.cuda.set_device(local)
    dev = torch.device("cuda", local)
    st = synth.STACK_7B_SETTINGS
    N, M, tau, iters, sweeps = st["N"], st["M"], st["tau"], st["iters"], st["sweeps"]
    mats = []
    t_gen = time.perf_counter()
    for layer in range(rank * args.layers, (rank + 1) * args.layers):      # ranks split whole layers
        for name, bits, _ in synth.stack_7b_layer(layer):
            Wd = to_device(bits, "bf16", dev)
            mats.append((layer, name, Wd, torch.empty((Wd.shape[0], (Wd.shape[1] + 31) // 32),
                                                     dtype=torch.int32, device=dev)))
    t_gen = time.perf_counter() - t_gen
    stream = torch.cuda.current_stream(dev)
    side = torch.cuda.Stream(dev)
    params = sum(Wd.numel() for _, _, Wd, _ in mats)

    def one_pass():
        # the matrices are independent calls; alternating two streams lets one
        # call's last wave overlap the next call's first
        side.wait_stream(stream)
        for k, (_, _, Wd, out) in enumerate(mats):
            tsl.tsenor_mask(Wd, N, M, tau, iters, sweeps, out=out, stream=stream if k % 2 == 0 else side)
        stream.wait_stream(side)

    for _ in range(max(1, args.warmup)):
        for _, _, Wd, out in mats[:7]:
            tsl.tsenor_mask(Wd, N, M, tau, iters, sweeps, out=out, stream=stream)
    torch.cuda.synchronize(dev)
    sampler = ClockSampler(gpu_uuid(dev))
    time.sleep(0.3)
    if world > 1:
        import torch.distributed as dist
        dist.barrier()
    torch.cuda.synchronize(dev)
    sampler.mark_start()
    ev = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)) for _ in range(args.steps)]
    for a, b in ev:
        a.record(stream)
        one_pass()
        b.record(stream)
    torch.cuda.synchronize(dev)
    sampler.mark_end()
    ms = statistics.mean(a.elapsed_time(b) for a, b in ev)
    ms_max = max_over_ranks(ms, dev, world)
    peaks = measure_pipe_peaks(dev, stream, sampler)
    clocks = sampler.stop()
    tsl.tsenor_error_count()
    roof = roofline_record(params, M, iters, ms, peaks)
    roof.update(traffic=None, kernel="whole pass (one fused_kernel_small<8,bf16> per matrix)", peaks_measured=peaks)
    line = {
        "metric": METRIC,
        "value": aggregate_gparams(params, world, ms_max), "unit": "Gparams/s", "n_gpus": world,
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": ms_max, "higher_is_better": True,
        "scaling": "weak", "vs_baseline": None, "dtype": "f32", "data": "synthetic",
        "config": {"workload": f"stack7b_{args.layers}x7_bf16_4of8", "layers_per_rank": args.layers,
                   "matrices_per_rank": len(mats), "params_per_rank": params, "N": N, "M": M, "tau": tau,
                   "iters": iters, "sweeps": sweeps,
                   "l2": "inputs larger than L2 (13 GB per pass, each matrix read once per pass)",
                   "total_wall_s_per_pass": ms_max / 1e3, "host_generation_s": t_gen},
        "roofline": roof,
        "gpu_launches": len(mats) * args.steps,
        "streams": "the 224 calls alternate between two streams (independent matrices)",
        "clocks": clocks, "cpu_baseline": None,
    }
    if rank == 0:
        print(json.dumps(line), flush=True)


def run_gap(args):
    """Quality report: gap of the GPU masks to the exact (min-cost-flow) optimum, on every block of
    the workload or on a seeded sample of whole block-rows; no timing."""
    import torch
    import sparse_mask_search_b200 as tsl
    dev = torch.device("cuda", int(os.environ.get("LOCAL_RANK", "0")))
    torch.cuda.set_device(dev)
    if args.workload == STACK:
        st = synth.STACK_7B_SETTINGS
        mats = [(f"stack7b_layer0_{name}", bits, vals, st["N"], st["M"], st["tau"], st["iters"], st["sweeps"])
                for name, bits, vals in synth.stack_7b_layer(0)]
    else:
        w = workload_of(args)
        bits, vals = synth.workload_matrix(w)
        mats = [(w.name, bits, vals, w.N, w.M, w.tau, w.iters, w.sweeps)]
    recs = []
    for name, bits, vals, N, M, tau, iters, sweeps in mats:
        Wd = to_device(bits, "bf16" if bits.dtype == np.uint16 else "f32", dev)
        mask = tsl.tsenor_mask(Wd, N, M, tau, iters, sweeps).cpu().numpy().view(np.uint32)
        per_mat = max(1, args.gap_blocks // len(mats)) if args.gap_blocks else 0
        rec = gap_record(vals, mask, N, M, max_blocks=per_mat)
        rec["matrix"] = name
        recs.append(rec)
    blocks = sum(r["blocks"] for r in recs)
    print(json.dumps({"report": "gap", "workload": args.workload, "blocks": blocks,
                      "mean": sum(r["mean"] * r["blocks"] for r in recs) / blocks,
                      "max": max(r["max"] for r in recs), "matrices": recs}), flush=True)


def blocks_identical(mask_a, mask_b, rows, cols, M):
    """Fraction of MxM blocks on which two packed masks agree bit for bit (on the device)."""
    import torch
    diff = torch.bitwise_xor(mask_a, mask_b)
    shifts = torch.arange(32, device=diff.device, dtype=torch.int32)
    bits = ((diff.unsqueeze(-1) >> shifts) & 1).to(torch.uint8).reshape(rows, -1)[:, :cols]
    blk = bits.reshape(rows // M, M, cols // M, M).amax(dim=(1, 3))
    return float((blk == 0).float().mean())


def run_warm(args, rank, world):
    """Outer-loop mode: one step = tsenor_mask_warm on a W that differs from the
    previous step's by a relative drift, started from the previous step's
    potentials, each block stopping at the tolerance (at most T iterations).
    Two matrices W_a, W_b = W_a * (1 + drift * noise) alternate, so every step
    is a genuine re-solve of a nearby matrix.  Quality is reported against the
    plain fixed-T solve of the same matrix."""
    import torch
    import sparse_mask_search_b200 as tsl
    local = int(os.environ.get("LOCAL_RANK", "0"))
    torch.cuda.set_device(local)
    dev = torch.device("cuda", local)
    w = workload_of(args)
    storage, vals = synth.workload_matrix(w, seed=rank_seed(w, rank))
    Wa = to_device(storage, w.dtype, dev)
    g = torch.Generator(device=dev)
    g.manual_seed(rank_seed(w, rank) + 1)
    Wb = (Wa.float() * (1.0 + args.drift * torch.randn(Wa.shape, device=dev, generator=g))).to(Wa.dtype)
    mats = (Wa, Wb)
    nb = (w.rows // w.M) * (w.cols // w.M)
    pot = torch.zeros((nb, 2 * w.M), dtype=torch.float32, device=dev)
    used = torch.zeros(nb, dtype=torch.int32, device=dev)
    wpr = (w.cols + 31) // 32
    mask = torch.empty((w.rows, wpr), dtype=torch.int32, device=dev)
    flush = torch.empty(L2_FLUSH_BYTES, dtype=torch.uint8, device=dev)
    stream = torch.cuda.current_stream(dev)
    # the first solve of the loop is cold with the full T
    tsl.tsenor_mask_warm(Wa, w.N, w.M, w.tau, w.iters, w.sweeps, potentials=pot, iters_used=used, out=mask,
                         stream=stream)

    def step(k):
        tsl.tsenor_mask_warm(mats[(k + 1) % 2], w.N, w.M, w.tau, w.iters, w.sweeps, tol=args.tol, potentials=pot,
                             warm=True, iters_used=used, out=mask, stream=stream)

    for k in range(max(3, args.warmup)):
        step(k)
    torch.cuda.synchronize(dev)
    sampler = ClockSampler(gpu_uuid(dev))
    time.sleep(0.3)
    if world > 1:
        import torch.distributed as dist
        dist.barrier()
    torch.cuda.synchronize(dev)
    sampler.mark_start()
    ev = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)) for _ in range(args.steps)]
    iters_sum = torch.zeros((), dtype=torch.int64, device=dev)
    k0 = max(3, args.warmup)
    for k in range(args.steps):
        flush.zero_()
        ev[k][0].record(stream)
        step(k0 + k)
        ev[k][1].record(stream)
        iters_sum += used.sum()
    torch.cuda.synchronize(dev)
    sampler.mark_end()
    ms = statistics.mean(a.elapsed_time(b) for a, b in ev)
    ms_max = max_over_ranks(ms, dev, world)
    peaks = measure_pipe_peaks(dev, stream, sampler)
    clocks = sampler.stop()
    mean_iters = float(iters_sum.item()) / (args.steps * nb)
    # quality against the plain fixed-T solve of the matrix the last step solved
    last = mats[(k0 + args.steps) % 2]
    ref = tsl.tsenor_mask(last, w.N, w.M, w.tau, w.iters, w.sweeps, stream=stream)
    obj_w = tsl.tsenor_objective(last, mask, w.N, w.M, stream=stream)
    obj_c = tsl.tsenor_objective(last, ref, w.N, w.M, stream=stream)
    same = blocks_identical(mask, ref, w.rows, w.cols, w.M)
    # plain fixed-T step on the same matrices, same flushing, for the speedup
    pev = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)) for _ in range(5)]
    for k, (a, b) in enumerate(pev):
        flush.zero_()
        a.record(stream)
        tsl.tsenor_mask(mats[k % 2], w.N, w.M, w.tau, w.iters, w.sweeps, out=ref, stream=stream)
        b.record(stream)
    torch.cuda.synchronize(dev)
    plain_ms = statistics.mean(a.elapsed_time(b) for a, b in pev)
    tsl.tsenor_error_count()
    params = w.rows * w.cols
    # the work of the iterations actually run (mean per block)
    roof = roofline_record(params, w.M, mean_iters, ms, peaks)
    roof.update(traffic=None, kernel=f"fused_kernel{w.M}<{w.dtype},EXT>" if w.M >= 16 else
                f"fused_kernel_small<{w.M},{w.dtype},EXT>", peaks_measured=peaks)
    line = {
        "metric": METRIC,
        "value": aggregate_gparams(params, world, ms_max), "unit": "Gparams/s", "n_gpus": world,
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": ms_max, "higher_is_better": True,
        "scaling": "weak", "vs_baseline": None, "dtype": "f32", "data": "synthetic",
        "config": {"workload": w.name, "mode": "warm-start outer loop, adaptive stop", "tol_nats": args.tol,
                   "drift": args.drift, "rows": w.rows, "cols": w.cols, "input_dtype": w.dtype, "N": w.N,
                   "M": w.M, "tau": w.tau, "max_iters": w.iters, "sweeps": w.sweeps,
                   "l2": "flushed before every timed step (256 MiB memset outside the events)"},
        "warm": {"mean_iters_per_block": mean_iters, "plain_fixed_T_ms": plain_ms,
                 "speedup_vs_plain": plain_ms / ms, "objective_ratio_vs_plain": float(obj_w.sum() / obj_c.sum()),
                 "blocks_identical_to_plain": same},
        "roofline": roof,
        "gpu_launches": (1 if w.M >= 16 else 2) * args.steps,
        "clocks": clocks, "cpu_baseline": None, "e2e": None,
    }
    if rank == 0:
        print(json.dumps(line), flush=True)


# --------------------------------------------------------------------------- GPU leg

def time_calls(fn, flush, stream, steps, warmup):
    """Per-call milliseconds of fn() over `steps` calls after `warmup`, CUDA events on
    `stream`, L2 flushed (a 256 MiB memset outside the events) before every call."""
    import torch
    for _ in range(warmup):
        fn()
    ev = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)) for _ in range(steps)]
    for a, b in ev:
        flush.zero_()
        a.record(stream)
        fn()
        b.record(stream)
    torch.cuda.synchronize()
    return [a.elapsed_time(b) for a, b in ev]


def time_e2e(host_w, w, host_mask, flush, stream, steps):
    """tsenor_mask_host calls (host W in, host mask out, copies inside the events)."""
    import sparse_mask_search_b200 as tsl
    return statistics.mean(time_calls(
        lambda: tsl.tsenor_mask_host(host_w, w.N, w.M, w.tau, w.iters, w.sweeps, out=host_mask, stream=stream),
        flush, stream, steps, 2))


def pinned_host(storage, dtype):
    import torch
    t = torch.from_numpy(storage.view(np.int16) if dtype == "bf16" else storage).pin_memory()
    return t.view(torch.bfloat16) if dtype == "bf16" else t


def secondary_workload(name, dev, stream, flush, steps, peaks, want_gap):
    """Device time, roofline fractions, end-to-end time and gap of one other workload."""
    import torch
    import sparse_mask_search_b200 as tsl
    w = synth.WORKLOADS[name]
    storage, vals = synth.workload_matrix(w)
    Wd = to_device(storage, w.dtype, dev)
    wpr = (w.cols + 31) // 32
    mask = torch.empty((w.rows, wpr), dtype=torch.int32, device=dev)
    ms = statistics.mean(time_calls(lambda: tsl.tsenor_mask(Wd, w.N, w.M, w.tau, w.iters, w.sweeps, out=mask,
                                                             stream=stream), flush, stream, steps, 3))
    plan = torch.empty((w.rows, w.cols), dtype=torch.float32, device=dev)
    plan_ms = statistics.mean(time_calls(lambda: tsl.tsenor_plan(Wd, w.N, w.M, w.tau, w.iters, out=plan,
                                                                  stream=stream), flush, stream, max(3, steps // 2), 2))
    del plan
    host_w, host_mask = pinned_host(storage, w.dtype), torch.empty((w.rows, wpr), dtype=torch.int32).pin_memory()
    e2e_ms = time_e2e(host_w, w, host_mask, flush, stream, max(3, steps // 2))
    gpu_mask = mask.cpu().numpy().view(np.uint32)
    if not np.array_equal(host_mask.numpy().view(np.uint32), gpu_mask):
        raise RuntimeError(f"{name}: tsenor_mask_host and tsenor_mask disagree")
    params = w.rows * w.cols
    rec = {"workload": w.name, "rows": w.rows, "cols": w.cols, "input_dtype": w.dtype, "N": w.N, "M": w.M,
           "tau": w.tau, "iters": w.iters, "sweeps": w.sweeps, "steps": steps, "ms_per_step": ms,
           "value": params / (ms / 1e3) / 1e9, "unit": "Gparams/s",
           "roofline": roofline_record(params, w.M, w.iters, ms, peaks),
           "dykstra_plan_kernel_alone_ms": plan_ms,
           "e2e": {"value": params / (e2e_ms / 1e3) / 1e9, "unit": "Gparams/s", "ms_per_step": e2e_ms,
                   "h2d_bytes_per_step": int(storage.nbytes), "d2h_bytes_per_step": int(host_mask.numel() * 4)}}
    if want_gap:
        rec["gap"] = gap_record(vals, gpu_mask, w.N, w.M, max_blocks=0 if w.M <= 32 else 8192)
    return rec


def secondary_stack(dev, stream, peaks, want_gap, passes=3):
    """The 7B-shaped stack (32 layers x 7 matrices, 4:8): one pass = tsenor_mask on all 224 matrices.
    Values N(0, 0.02) are drawn on the device (torch's Philox generator, seed 1000*layer + k)."""
    import torch
    import sparse_mask_search_b200 as tsl
    st = synth.STACK_7B_SETTINGS
    N, M, tau, iters, sweeps = st["N"], st["M"], st["tau"], st["iters"], st["sweeps"]
    mats = []
    g = torch.Generator(device=dev)
    for layer in range(synth.STACK_7B_LAYERS):
        for k, (name, r, c) in enumerate(synth.STACK_7B_MATRICES):
            g.manual_seed(1000 * layer + k)
            Wd = (0.02 * torch.randn((r, c), device=dev, generator=g)).to(torch.bfloat16)
            mats.append((Wd, torch.empty((r, (c + 31) // 32), dtype=torch.int32, device=dev)))
    params = sum(Wd.numel() for Wd, _ in mats)
    side = torch.cuda.Stream(dev)

    def one_pass():
        side.wait_stream(stream)
        for k, (Wd, out) in enumerate(mats):
            tsl.tsenor_mask(Wd, N, M, tau, iters, sweeps, out=out, stream=stream if k % 2 == 0 else side)
        stream.wait_stream(side)

    for _ in range(2):
        one_pass()
    torch.cuda.synchronize(dev)
    ev = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)) for _ in range(passes)]
    for a, b in ev:
        a.record(stream)
        one_pass()
        b.record(stream)
    torch.cuda.synchronize(dev)
    ms = statistics.mean(a.elapsed_time(b) for a, b in ev)
    # end to end: every layer's matrices go through tsenor_mask_host from pinned host
    # copies of layer 0's seven matrices (the same bytes per pass as the stack)
    host = [(mats[k][0].cpu().pin_memory(),
             torch.empty(tuple(mats[k][1].shape), dtype=torch.int32).pin_memory()) for k in range(7)]

    def one_pass_host():
        for k in range(len(mats)):
            hw, hm = host[k % 7]
            tsl.tsenor_mask_host(hw, N, M, tau, iters, sweeps, out=hm, stream=stream)

    one_pass_host()
    torch.cuda.synchronize(dev)
    ev = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)) for _ in range(2)]
    for a, b in ev:
        a.record(stream)
        one_pass_host()
        b.record(stream)
    torch.cuda.synchronize(dev)
    e2e_ms = statistics.mean(a.elapsed_time(b) for a, b in ev)
    if not torch.equal(host[0][1], mats[0][1].cpu()):
        raise RuntimeError("stack: tsenor_mask_host and tsenor_mask disagree")
    rec = {"workload": "stack7b_32x7_bf16_4of8", "matrices": len(mats), "params": params, "N": N, "M": M,
           "tau": tau, "iters": iters, "sweeps": sweeps, "passes": passes, "ms_per_step": ms,
           "value": params / (ms / 1e3) / 1e9, "unit": "Gparams/s",
           "data": "values drawn on the device: N(0, 0.02), torch Philox, seed 1000*layer + matrix index",
           "streams": "the 224 calls alternate between two streams (independent matrices)",
           "roofline": roofline_record(params, M, iters, ms, peaks),
           "e2e": {"value": params / (e2e_ms / 1e3) / 1e9, "unit": "Gparams/s", "ms_per_step": e2e_ms,
                   "h2d_bytes_per_step": int(params * 2), "d2h_bytes_per_step": int(sum(m.numel() for _, m in mats) * 4),
                   "call": "tsenor_mask_host per matrix; host buffers: layer 0's seven matrices, pinned, "
                           "reused for every layer"}}
    if want_gap:
        W0 = mats[0][0].float().cpu().numpy()
        rec["gap"] = gap_record(W0, mats[0][1].cpu().numpy().view(np.uint32), N, M, max_blocks=8192)
        rec["gap"]["matrix"] = "layer 0, q (4096 x 4096)"
    del mats
    torch.cuda.empty_cache()
    return rec


def main(argv=None):
    args = parse_args(argv)
    rank = int(os.environ.get("RANK", "0"))
    world = int(os.environ.get("WORLD_SIZE", "1"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    if args.impl == "reference":
        run_reference(args, rank, world)
        return 0
    if args.mode == "gap":
        if rank == 0:
            run_gap(args)
        return 0
    if args.mode == "warm" and args.workload != STACK:
        if world > 1:
            import torch
            import torch.distributed as dist
            torch.cuda.set_device(local)
            dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=300),
                                    device_id=torch.device("cuda", local))
        run_warm(args, rank, world)
        if world > 1:
            dist.barrier()
            dist.destroy_process_group()
        return 0
    if args.workload == STACK:
        if world > 1:
            import torch
            import torch.distributed as dist
            torch.cuda.set_device(local)
            dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=300),
                                    device_id=torch.device("cuda", local))
        run_stack(args, rank, world)
        if world > 1:
            dist.barrier()
            dist.destroy_process_group()
        return 0

    import torch
    import torch.distributed as dist
    import sparse_mask_search_b200 as tsl

    torch.cuda.set_device(local)
    dev = torch.device("cuda", local)
    if world > 1:
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=300), device_id=dev)

    w = workload_of(args)
    storage, vals = synth.workload_matrix(w, seed=rank_seed(w, rank))
    Wd = to_device(storage, w.dtype, dev)
    wpr = (w.cols + 31) // 32
    mask = torch.empty((w.rows, wpr), dtype=torch.int32, device=dev)
    flush = torch.empty(L2_FLUSH_BYTES, dtype=torch.uint8, device=dev)
    stream = torch.cuda.current_stream(dev)

    def step():
        tsl.tsenor_mask(Wd, w.N, w.M, w.tau, w.iters, w.sweeps, out=mask, stream=stream)

    for _ in range(args.warmup):                    # the same launches as a timed step
        flush.zero_()
        step()
    torch.cuda.synchronize(dev)

    sampler = ClockSampler(gpu_uuid(dev))
    time.sleep(0.3)

    # ---- timed region: K steps, L2 flushed before each (outside the events)
    if world > 1:
        dist.barrier()
    torch.cuda.synchronize(dev)
    sampler.mark_start()
    ev = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)) for _ in range(args.steps)]
    for k in range(args.steps):
        flush.zero_()
        ev[k][0].record(stream)
        step()
        ev[k][1].record(stream)
    torch.cuda.synchronize(dev)
    sampler.mark_end()
    if world > 1:
        dist.barrier()
    step_ms = [a.elapsed_time(b) for a, b in ev]
    mean_ms = sum(step_ms) / len(step_ms)
    mean_ms_max = max_over_ranks(mean_ms, dev, world)
    gpu_mask = mask.cpu().numpy().view(np.uint32)

    # ---- the pipes' throughput on this GPU (roofline denominators)
    peaks = measure_pipe_peaks(dev, stream, sampler)
    clocks = sampler.stop()

    # ---- the Dykstra phase alone (the plan kernel), same stream, same input
    plan = torch.empty((w.rows, w.cols), dtype=torch.float32, device=dev)
    plan_ms = statistics.mean(time_calls(lambda: tsl.tsenor_plan(Wd, w.N, w.M, w.tau, w.iters, out=plan,
                                                                  stream=stream), flush, stream, 10, 3))
    round_ms = max(mean_ms - plan_ms, 0.0)
    del plan

    # ---- end to end through the public API with host buffers: tsenor_mask_host
    # copies W in row chunks and the mask back, overlapped with the solve
    host_w = pinned_host(storage, w.dtype)
    host_mask = torch.empty((w.rows, wpr), dtype=torch.int32).pin_memory()
    e2e_ms = time_e2e(host_w, w, host_mask, flush, stream, max(3, min(args.steps, 20)))
    if not np.array_equal(host_mask.numpy().view(np.uint32), gpu_mask):
        raise RuntimeError("tsenor_mask_host and tsenor_mask disagree")
    e2e_ms = max_over_ranks(e2e_ms, dev, world)

    params = w.rows * w.cols
    value = aggregate_gparams(params, world, mean_ms_max)
    # tsenor_mask is one fused kernel per call for every M: the dominant kernel is
    # the whole step; the plan-only kernel gives the Dykstra phase alone
    kernel_key = f"fused_kernel{w.M}<{w.dtype}>" if w.M >= 16 else f"fused_kernel_small<{w.M},{w.dtype}>"
    roof = roofline_record(params, w.M, w.iters, mean_ms, peaks)
    unit_peaks = {"fma_tops": fp32_peak_tops(SM_MAX_MHZ_FALLBACK), "mufu_tops": mufu_peak_tops(SM_MAX_MHZ_FALLBACK)}
    roof.update(traffic=profiled_traffic(kernel_key), kernel=kernel_key, kernel_ms=mean_ms,
                peaks_measured=peaks,
                peak_basis="measured by this run's own probe kernels (peaks_measured)",
                vs_unit_count_peaks={"peaks": unit_peaks,
                                     "basis": f"{SM_COUNT} SMs x ({FP32_LANES_PER_CLK_PER_SM} FP32, "
                                              f"{MUFU_LANES_PER_CLK_PER_SM} MUFU) lanes/clk x "
                                              f"{SM_MAX_MHZ_FALLBACK:.0f} MHz",
                                     "frac": roofline_record(params, w.M, w.iters, mean_ms, unit_peaks)["frac"]})
    plan_roof = roofline_record(params, w.M, w.iters, plan_ms, peaks)
    line = {
        "metric": METRIC,
        "value": value, "unit": "Gparams/s", "n_gpus": world, "steps": args.steps, "warmup": args.warmup,
        "ms_per_step": mean_ms_max, "higher_is_better": True, "scaling": "weak", "vs_baseline": None,
        "dtype": "f32", "data": "synthetic",
        "config": {"workload": w.name, "rows": w.rows, "cols": w.cols, "input_dtype": w.dtype, "N": w.N,
                   "M": w.M, "tau": w.tau, "iters": w.iters, "sweeps": w.sweeps,
                   "l2": "flushed before every timed step (256 MiB memset outside the events)",
                   "parallelism": f"replicas x{world}: each rank solves its own matrix, no collective"},
        "roofline": roof,
        "breakdown_ms": {"dykstra_plan_kernel_alone": plan_ms, "rest_of_step": round_ms,
                         "dykstra_frac_survey": plan_roof["frac_survey"]["binding"],
                         "dykstra_frac_fma": plan_roof["frac_fma"]},
        "e2e": {"value": aggregate_gparams(params, world, e2e_ms), "unit": "Gparams/s",
                "h2d_bytes_per_step": int(storage.nbytes), "d2h_bytes_per_step": int(host_mask.numel() * 4),
                "ms_per_step": e2e_ms, "call": "tsenor_mask_host (pinned host W and mask, chunked, copies overlapped)"},
        "gpu_launches": args.steps,
        "clocks": clocks,
        "cpu_baseline": None,
        "hbm": {"algorithmic_bytes_per_step": int(storage.nbytes + mask.numel() * 4),
                "achieved_gbs": (storage.nbytes + mask.numel() * 4) / (mean_ms_max / 1e3) / 1e9,
                "measured_peak_gbs": measured_peaks().get("hbm_gbs")},
    }
    if rank == 0 and world == 1 and not args.no_gap:
        line["gap"] = gap_record(vals, gpu_mask, w.N, w.M)
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        line["cpu_baseline"] = cpu_baseline_leg(vals, w, args.cpu_seconds)
    if rank == 0 and world == 1 and not args.no_secondary and not args.shape:
        recs = []
        for name in SECONDARY:
            if name == w.name:
                continue
            if name == STACK:
                recs.append(secondary_stack(dev, stream, peaks, not args.no_gap))
            else:
                heavy = synth.WORKLOADS[name].params > 10 ** 8
                recs.append(secondary_workload(name, dev, stream, flush, min(args.steps, 10 if heavy else 20),
                                               peaks, not args.no_gap))
        line["other_workloads"] = recs
    if world > 1:
        dist.barrier()
        dist.destroy_process_group()
    if rank == 0:
        print(json.dumps(line), flush=True)
    return 0


if __name__ == "__main__":
    sys.exit(main())
