"""Helpers shared by the GPU tests: device copies and parity statistics."""
import json
import os

import numpy as np

import oracle

PLAN_TOL = 1e-4          # max |S_gpu - S_oracle| (fp32 plan vs fp64 plan)
# A block may differ from the oracle's only through a near-tie: every pair of
# entries that the two key sets order differently has oracle keys within this
# relative distance, |S_e - S_f| / max(S_e, S_f).
NEAR_TIE = 1e-6


def to_device(storage, dtype):
    import torch
    if dtype == "bf16":
        return torch.from_numpy(np.ascontiguousarray(storage).view(np.int16)).view(torch.bfloat16).cuda()
    return torch.from_numpy(np.ascontiguousarray(storage, dtype=np.float32)).cuda()


def mask_to_np(t):
    return t.cpu().numpy().view(np.uint32)


def block_bits(mask_words, cols, M):
    return oracle.blocks_view(oracle.unpack(mask_words, cols), M)


def order(S, a):
    """Rounding order of one block: S desc, |W| desc, flat index asc."""
    E = S.size
    return np.lexsort((np.arange(E), -a.ravel().astype(np.float64), -S.ravel().astype(np.float64)))


def max_inverted_gap(S_ref, S_gpu, a):
    """Largest relative gap |S_ref[e] - S_ref[f]| / max(S_ref[e], S_ref[f]) over the
    entry pairs that the two key sets order differently (0 when none is)."""
    o = order(S_ref, a)
    pos = np.empty(S_ref.size, dtype=np.int64)
    pos[order(S_gpu, a)] = np.arange(S_ref.size)
    P = pos[o]
    ks = S_ref.ravel().astype(np.float64)[o]
    E = len(P)
    best = 0.0
    for u0 in range(0, E, 512):
        u = np.arange(u0, min(E, u0 + 512))
        inv = (P[u][:, None] > P[None, :]) & (u[:, None] < np.arange(E)[None, :])
        if inv.any():
            d = np.abs(ks[u][:, None] - ks[None, :])
            scale = np.maximum(np.abs(ks[u][:, None]), np.abs(ks[None, :]))
            rel = np.divide(d, scale, out=np.zeros_like(d), where=scale > 0)
            best = max(best, float(rel[inv].max()))
    return best


def record(name, stats):
    path = os.environ.get("TSENOR_PARITY_LOG")
    if path:
        with open(path, "a") as f:
            f.write(json.dumps({"case": name, **stats}) + "\n")
