"""Full-size workloads, in the launch configuration the benchmark times.

Every block of the full matrix is checked for validity on the device
(tsenor_objective); a seeded sample of at least 2048 blocks is solved again by
the CPU oracle and compared block by block: at least 99.9% of the sampled
blocks identical, every differing one through a near-tie of the oracle's keys
(relative gap below 1e-6), the summed objective within 1e-6 relative.  The
sample's exact optimum gives the quality gap, which must stay inside the
pages' stated 1-10% relative error.
"""
import numpy as np
import pytest

import oracle
import synth
from gpu_util import NEAR_TIE, block_bits, mask_to_np, max_inverted_gap, record, to_device

torch = pytest.importorskip("torch")
pytestmark = pytest.mark.gpu

import sparse_mask_search_b200 as tsl  # noqa: E402


def gather_blocks(W, M, ids):
    nbc = W.shape[1] // M
    return np.concatenate([W[(b // nbc) * M:(b // nbc + 1) * M, (b % nbc) * M:(b % nbc + 1) * M] for b in ids],
                          axis=1)


def check_sampled(name, stor, W, dtype, N, M, tau, iters, sweeps, n_sample, seed=0, min_identical=0.999):
    rows, cols = W.shape
    Wd = to_device(stor, dtype)
    tsl.tsenor_error_count()
    m_t = tsl.tsenor_mask(Wd, N, M, tau, iters, sweeps)
    obj = tsl.tsenor_objective(Wd, m_t, N, M).cpu().numpy()
    assert tsl.tsenor_error_count() == 0
    assert not np.isnan(obj).any()                       # every block valid
    nb = obj.size
    ids = np.sort(np.random.default_rng(seed).choice(nb, size=min(n_sample, nb), replace=False))
    sub = gather_blocks(W, M, ids)
    m_gpu = block_bits(mask_to_np(m_t), cols, M).reshape(-1, M, M)[ids]
    m_ref_w, keys_ref, _ = oracle.mask(sub, N, M, tau, iters, sweeps, want_keys=True)
    m_ref = block_bits(m_ref_w, sub.shape[1], M).reshape(-1, M, M)
    same = (m_gpu == m_ref).all(axis=(1, 2))
    gaps = []
    if not same.all():
        plan = tsl.tsenor_plan(Wd, N, M, tau, iters).cpu().numpy()
        Pg = oracle.blocks_view(plan, M).reshape(-1, M, M)[ids]
        Pr = oracle.blocks_view(keys_ref, M).reshape(-1, M, M)
        A = oracle.blocks_view(np.abs(sub), M).reshape(-1, M, M)
        gaps = [max_inverted_gap(Pr[k], Pg[k], A[k]) for k in np.where(~same)[0]]
    obj_ref = oracle.objective(sub, m_ref_w, N, M)
    rel = abs(obj[ids].sum() - obj_ref.sum()) / obj_ref.sum()
    opt, _ = oracle.opt(sub, N, M)
    gap = (opt - obj[ids]) / opt
    stats = {"blocks": int(nb), "sampled": int(len(ids)), "identical": float(same.mean()),
             "max_inverted_key_gap": max(gaps) if gaps else 0.0, "objective_rel": float(rel),
             "gap_mean": float(gap.mean()), "gap_max": float(gap.max())}
    record(name, stats)
    assert same.mean() >= min_identical, stats
    assert all(g <= NEAR_TIE for g in gaps), stats
    assert rel <= 1e-6, stats
    assert (gap >= -1e-12).all() and gap.mean() <= 0.10, stats
    return stats


@pytest.mark.parametrize("name,n_sample", [("w4096x4096_bf16_normal_8of16", 4096),
                                           ("w4096x11008_bf16_t3_16of32", 4096),
                                           ("w8192x28672_bf16_laplace_32of64", 4096)])
def test_full_workload_sampled(name, n_sample):
    w = synth.WORKLOADS[name]
    stor, W = synth.workload_matrix(w)
    check_sampled(w.name, stor, W, w.dtype, w.N, w.M, w.tau, w.iters, w.sweeps, n_sample)


def test_stack_7b_layer_sampled():
    s = synth.STACK_7B_SETTINGS
    for k, (name, stor, W) in enumerate(synth.stack_7b_layer(0)):
        check_sampled(f"stack7b_layer0_{name}", stor, W, "bf16", s["N"], s["M"], s["tau"], s["iters"],
                      s["sweeps"], 2048, seed=k)
