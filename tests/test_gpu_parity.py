"""CUDA path vs the CPU oracle on identical seeded inputs (through the C ABI).

Bars (the target stated for this method): the fp32 plan within 1e-4 of the
oracle's; every block's mask valid, bit-exact; rounding bit-exact on an
identical plan; >= 99.9% identical blocks, each differing block traced to a
near-tie of the sort keys; per-matrix objective within 1e-6 relative.
"""
import numpy as np
import pytest

import oracle
import synth
from gpu_util import (NEAR_TIE, PLAN_TOL, block_bits, mask_to_np, max_inverted_gap, record,
                      to_device)

torch = pytest.importorskip("torch")
pytestmark = pytest.mark.gpu

import sparse_mask_search_b200 as tsl  # noqa: E402

# (M, N, dtype, rows, cols, tau, iters, sweeps, dist): block counts leave a ragged
# last CTA (128 blocks per CTA for M <= 8, 16 for M = 16, 4 for M = 32, 1 for M = 64)
CASES = [
    (4, 2, "f32", 64, 100, 10.0, 200, 1, "normal"),
    (4, 1, "bf16", 36, 132, 10.0, 50, 3, "laplace_outliers"),
    (8, 4, "bf16", 64, 200, 20.0, 200, 4, "normal"),
    (8, 3, "f32", 40, 72, 20.0, 120, 2, "t3_outlier_cols"),
    (16, 8, "bf16", 64, 176, 20.0, 300, 4, "normal"),
    (16, 5, "f32", 48, 80, 15.0, 100, 3, "laplace_outliers"),
    (32, 16, "bf16", 96, 160, 20.0, 300, 8, "t3_outlier_cols"),
    (32, 7, "f32", 64, 96, 20.0, 150, 8, "normal"),
    (64, 32, "bf16", 128, 192, 30.0, 400, 8, "laplace_outliers"),
    (64, 20, "f32", 64, 128, 30.0, 100, 8, "normal"),
]


def _ids(c):
    return f"M{c[0]}N{c[1]}_{c[2]}_{c[3]}x{c[4]}"


def _matrix(c, seed=0):
    M, N, dtype, rows, cols, tau, iters, sweeps, dist = c
    scale = 1.0 if dtype == "f32" and dist == "normal" else 0.02
    return synth.make_matrix(rows, cols, dtype, dist, scale, seed=1234 + M * 7 + N + seed)


@pytest.mark.parametrize("c", CASES, ids=_ids)
def test_plan_matches_oracle(c):
    M, N, dtype, rows, cols, tau, iters, sweeps, dist = c
    stor, W = _matrix(c)
    P_gpu = tsl.tsenor_plan(to_device(stor, dtype), N, M, tau, iters).cpu().numpy()
    P_ref = oracle.plan(W, N, M, tau, iters)
    err = np.abs(P_gpu.astype(np.float64) - P_ref)
    record("plan_" + _ids(c), {"max_abs": float(err.max()), "mean_abs": float(err.mean())})
    assert err.max() <= PLAN_TOL
    assert (P_gpu <= 1.0).all() and (P_gpu >= 0.0).all()


@pytest.mark.parametrize("c", CASES, ids=_ids)
def test_rounding_bit_exact_on_identical_plan(c):
    M, N, dtype, rows, cols, tau, iters, sweeps, dist = c
    stor, W = _matrix(c)
    Wd = to_device(stor, dtype)
    plan = tsl.tsenor_plan(Wd, N, M, tau, iters)
    m_gpu = mask_to_np(tsl.tsenor_round(plan, Wd, N, M, sweeps))
    m_ref, st = oracle.round_plan(plan.cpu().numpy(), W, N, M, sweeps)
    assert (m_gpu == m_ref).all()
    # random keys independent of |W| stress repair and local search; coarse
    # keys (3 levels) stress the tie-breaking
    g = np.random.default_rng(M + N)
    for keys in (g.random((rows, cols)).astype(np.float32),
                 (g.integers(0, 3, (rows, cols)) / 2.0).astype(np.float32)):
        kd = torch.from_numpy(keys).cuda()
        m_gpu = mask_to_np(tsl.tsenor_round(kd, Wd, N, M, sweeps))
        m_ref, st = oracle.round_plan(keys, W, N, M, sweeps)
        assert st["failures"] == 0
        assert (m_gpu == m_ref).all(), _ids(c)


def check_pipeline(name, stor, W, dtype, N, M, tau, iters, sweeps, min_identical=0.999):
    Wd = to_device(stor, dtype)
    tsl.tsenor_error_count()
    m_gpu_t = tsl.tsenor_mask(Wd, N, M, tau, iters, sweeps)
    obj_gpu = tsl.tsenor_objective(Wd, m_gpu_t, N, M).cpu().numpy()
    assert tsl.tsenor_error_count() == 0
    m_gpu = mask_to_np(m_gpu_t)
    m_ref, keys_ref, st = oracle.mask(W, N, M, tau, iters, sweeps, want_keys=True)
    # validity, bit-exact, on every block
    assert not np.isnan(obj_gpu).any()
    obj_ref_of_gpu = oracle.objective(W, m_gpu, N, M)
    assert not np.isnan(obj_ref_of_gpu).any()
    np.testing.assert_allclose(obj_gpu, obj_ref_of_gpu, rtol=1e-12)
    obj_ref = oracle.objective(W, m_ref, N, M)
    rows, cols = W.shape
    bg, br = block_bits(m_gpu, cols, M), block_bits(m_ref, cols, M)
    same = (bg == br).all(axis=(2, 3)).ravel()
    diff = np.where(~same)[0]
    gaps = []
    if len(diff):
        plan = tsl.tsenor_plan(Wd, N, M, tau, iters).cpu().numpy()
        Pg, Pr = oracle.blocks_view(plan, M), oracle.blocks_view(keys_ref, M)
        A = oracle.blocks_view(np.abs(W), M)
        nbc = cols // M
        for b in diff[:50]:
            r, c = divmod(int(b), nbc)
            gaps.append(max_inverted_gap(Pr[r, c], Pg[r, c], A[r, c]))
    rel = abs(obj_gpu.sum() - obj_ref.sum()) / obj_ref.sum()
    stats = {"blocks": int(same.size), "identical": float(same.mean()), "differing": int(len(diff)),
             "max_inverted_key_gap": max(gaps) if gaps else 0.0, "objective_rel": float(rel)}
    record(name, stats)
    assert same.mean() >= min_identical, stats
    assert all(g <= NEAR_TIE for g in gaps), stats
    assert rel <= 1e-6, stats
    return stats


@pytest.mark.parametrize("c", CASES, ids=_ids)
def test_mask_matches_oracle(c):
    M, N, dtype, rows, cols, tau, iters, sweeps, dist = c
    stor, W = _matrix(c)
    nb = (rows // M) * (cols // M)
    # with few blocks one near-tie is more than 0.1%; the near-tie check still applies
    check_pipeline("mask_" + _ids(c), stor, W, dtype, N, M, tau, iters, sweeps,
                   min_identical=0.999 if nb >= 1000 else 0.0)


def test_full_256x256_2of4():
    w = synth.WORKLOADS["w256x256_f32_normal_2of4"]
    stor, W = synth.workload_matrix(w)
    check_pipeline(w.name, stor, W, w.dtype, w.N, w.M, w.tau, w.iters, w.sweeps)


@pytest.mark.parametrize("M,N,dtype", [(8, 4, "f32"), (16, 8, "bf16"), (32, 16, "bf16"), (64, 32, "bf16")])
def test_largest_tau(M, N, dtype):
    """tau = 80 (the largest accepted): the block's kernel spans 2^115, near the edge
    of the fp32 range the linear-form exponentials live in.  Plan within the plan
    bar; masks valid and equal to the oracle's but for near-ties."""
    rows, cols = 2 * M, 8 * M
    stor, W = synth.make_matrix(rows, cols, dtype, "laplace_outliers", 0.02, seed=500 + M)
    check = (M, N, dtype, rows, cols, 80.0, 300, 4, "laplace_outliers")
    Wd = to_device(stor, dtype)
    P_gpu = tsl.tsenor_plan(Wd, N, M, 80.0, 300).cpu().numpy()
    P_ref = oracle.plan(W, N, M, 80.0, 300)
    assert np.abs(P_gpu.astype(np.float64) - P_ref).max() <= PLAN_TOL
    check_pipeline("mask_tau80_" + _ids(check), stor, W, dtype, N, M, 80.0, 300, 4, min_identical=0.0)
    with pytest.raises(tsl.TsenorError):
        tsl.tsenor_mask(Wd, N, M, 80.5, 300, 4)


def test_objective_matches_oracle_on_oracle_masks():
    stor, W = synth.make_matrix(64, 128, "bf16", "normal", 0.02, seed=3)
    m_ref, _, _ = oracle.mask(W, 8, 16, 20.0, 50, 2)
    m_ref[0, 0] ^= 1                                    # break block 0
    md = torch.from_numpy(m_ref.view(np.int32)).cuda()
    got = tsl.tsenor_objective(to_device(stor, "bf16"), md, 8, 16).cpu().numpy()
    ref = oracle.objective(W, m_ref, 8, 16)
    assert np.isnan(got[0]) and np.isnan(ref[0])
    np.testing.assert_allclose(got[1:], ref[1:], rtol=1e-12)


@pytest.mark.parametrize("M,N", [(4, 2), (8, 4), (16, 8), (32, 16), (64, 32)])
def test_non_finite_blocks_fail_alone(M, N):
    stor, W = synth.make_matrix(2 * M, 3 * M, "f32", "normal", 1.0, seed=M)
    stor = stor.copy()
    stor[1, M + 2] = np.nan          # block 1
    stor[M + 3, 2 * M] = np.inf      # block 5
    tsl.tsenor_error_count()
    Wd = to_device(stor, "f32")
    m = mask_to_np(tsl.tsenor_mask(Wd, N, M, 10.0, 40, 2))
    assert tsl.tsenor_error_count() == 2
    bits = block_bits(m, 3 * M, M)
    assert (bits[0, 1] == 0).all() and (bits[1, 2] == 0).all()
    for (r, c) in ((0, 0), (0, 2), (1, 0), (1, 1)):
        assert (bits[r, c].sum(axis=0) == N).all() and (bits[r, c].sum(axis=1) == N).all()
    plan = tsl.tsenor_plan(Wd, N, M, 10.0, 40).cpu().numpy()
    P = oracle.blocks_view(plan, M)
    assert np.isnan(P[0, 1]).all() and np.isnan(P[1, 2]).all()
    assert np.isfinite(P[0, 0]).all()


@pytest.mark.parametrize("M", [4, 8, 16, 32, 64])
def test_degenerate_blocks(M):
    """All-zero block, constant block (every key and weight tied), N = M, N = 1."""
    rows, cols = M, 4 * M
    W = np.zeros((rows, cols), np.float32)
    W[:, M:2 * M] = 0.5
    W[:, 2 * M:] = synth.make_matrix(rows, 2 * M, "f32", "normal", 1.0, seed=9)[1]
    Wd = to_device(W, "f32")
    for N in sorted({1, max(1, M // 2), M}):
        m = mask_to_np(tsl.tsenor_mask(Wd, N, M, 20.0, 60, 3))
        m_ref, _, _ = oracle.mask(W, N, M, 20.0, 60, 3)
        bits = block_bits(m, cols, M)
        assert (bits.sum(axis=3) == N).all() and (bits.sum(axis=2) == N).all()
        # zero and constant blocks are exact ties everywhere: index order decides
        assert (block_bits(m_ref, cols, M)[0, :2] == bits[0, :2]).all()
        if N == M:
            assert (bits == 1).all()


def test_empty_and_bad_arguments():
    W = torch.zeros((0, 64), dtype=torch.bfloat16, device="cuda")
    out = tsl.tsenor_mask(W, 2, 4, 10.0, 5, 1)
    assert out.shape == (0, 2)
    W = torch.zeros((64, 60), dtype=torch.bfloat16, device="cuda")
    with pytest.raises(tsl.TsenorError) as e:
        tsl.tsenor_mask(W, 2, 8, 10.0, 5, 1)
    assert e.value.status == -2
    with pytest.raises(tsl.TsenorError):
        tsl.tsenor_mask(torch.zeros((64, 64), dtype=torch.bfloat16, device="cuda"), 2, 12, 10.0, 5, 1)


def test_stream_ordering_on_side_stream():
    stor, W = synth.make_matrix(64, 256, "bf16", "normal", 0.02, seed=77)
    s = torch.cuda.Stream()
    with torch.cuda.stream(s):
        Wd = to_device(stor, "bf16")
        m = tsl.tsenor_mask(Wd, 16, 32, 20.0, 100, 4, stream=s)
    s.synchronize()
    m_ref, _, _ = oracle.mask(W, 16, 32, 20.0, 100, 4)
    bits = block_bits(mask_to_np(m), 256, 32)
    assert (bits.sum(axis=3) == 16).all()
    assert (block_bits(m_ref, 256, 32) == bits).all(axis=(2, 3)).mean() >= 0.5


@pytest.mark.parametrize("c", CASES, ids=_ids)
def test_mask_equals_rounding_of_exported_plan(c):
    """tsenor_mask (fused for M = 32) == tsenor_round(tsenor_plan(W)), bit for bit."""
    M, N, dtype, rows, cols, tau, iters, sweeps, dist = c
    stor, W = _matrix(c, seed=1)
    Wd = to_device(stor, dtype)
    m1 = tsl.tsenor_mask(Wd, N, M, tau, iters, sweeps)
    m2 = tsl.tsenor_round(tsl.tsenor_plan(Wd, N, M, tau, iters), Wd, N, M, sweeps)
    assert torch.equal(m1, m2)


@pytest.mark.parametrize("M,N,rows,cols", [(4, 2, 64, 128), (8, 4, 64, 128), (16, 8, 128, 128), (32, 16, 128, 256),
                                             (64, 32, 256, 512)])
def test_rounding_bit_exact_on_adversarial_keys(M, N, rows, cols):
    """The bf16 sort's 32-bit keys keep a bucket of the plan (an exponent window
    and upper mantissa bits) and settle same-bucket runs with the full key: keys
    spread over many binades (below the window too), keys one or two ulps apart
    (same bucket, any order), keys on bucket edges and exact ties of plan and
    |W| must all round as the oracle does."""
    g = np.random.default_rng(M * 31 + N)
    stor, W = synth.make_matrix(rows, cols, "bf16", "laplace_outliers", 0.02, seed=77 + M)
    Wd = to_device(stor, "bf16")
    wide = np.exp2(g.uniform(-24.0, 0.0, (rows, cols))).astype(np.float32)
    base = g.uniform(0.25, 0.5, (rows, cols)).astype(np.float32)
    near = (base.view(np.uint32) & ~np.uint32(3) | g.integers(0, 4, (rows, cols)).astype(np.uint32)).view(np.float32)
    edges = np.exp2(g.integers(-16, 1, (rows, cols)).astype(np.float32)) * \
        np.where(g.random((rows, cols)) < 0.5, np.float32(1.0), np.float32(1.0 - 2.0 ** -24))
    edges = np.minimum(edges, np.float32(1.0)).astype(np.float32)
    few = (g.integers(0, 40, (rows, cols)) / 39.0).astype(np.float32)
    for name, keys in (("wide", wide), ("near", near), ("edges", edges), ("few", few)):
        kd = torch.from_numpy(keys).cuda()
        m_gpu = mask_to_np(tsl.tsenor_round(kd, Wd, N, M, 8))
        m_ref, st = oracle.round_plan(keys, W, N, M, 8)
        assert st["failures"] == 0
        assert (m_gpu == m_ref).all(), name
