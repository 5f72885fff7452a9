"""Pins for the oracle's rounding: greedy, feasibility repair, local search.

Hand-worked fixtures (tests/golden/rounding_4x4.json) follow the TSENOR
review's description of the rounding ("What carries the argument", Fig. 2
caption).  Properties that hold for any input are checked on random blocks:
  - after the greedy every (short row, short column) pair is already taken;
  - after the repair every row and column holds exactly N ones;
  - the local search never lowers the objective and, run to convergence,
    leaves no exchange between two rows that gains;
  - the result never beats the exact optimum.
"""
import json
import os

import numpy as np
import pytest

import oracle
import synth


def load_fixtures(golden_dir):
    with open(os.path.join(golden_dir, "rounding_4x4.json")) as f:
        return json.load(f)


def test_hand_worked_fixtures(golden_dir):
    for fx in load_fixtures(golden_dir):
        key = np.array(fx["key"], np.float32)
        a = np.array(fx["a"], np.float32)
        for stage, name in ((1, "after_greedy"), (2, "after_repair"), (3, "after_ls")):
            s, rc, st = oracle.block_round(key, a, fx["N"], fx["sweeps"], stage)
            assert rc == 0, fx["name"]
            assert (s == np.array(fx[name])).all(), (fx["name"], name, s)
        assert st["repairs"] == fx["repairs"], fx["name"]
        assert st["ls_swaps"] == fx["ls_swaps"], fx["name"]
        assert float((s * a.astype(np.float64)).sum()) == fx["objective"]


def _rand_case(M, seed, dist="normal"):
    g = np.random.default_rng(seed)
    a = np.abs(synth.random_blocks(1, M, seed=seed, dist=dist, dtype="bf16", scale=0.02)).reshape(M, M)
    # keys drawn independently of |W| make the greedy leave deficits often
    key = g.random((M, M)).astype(np.float32)
    return key, a


@pytest.mark.parametrize("M", [4, 8, 16, 32, 64])
def test_greedy_deficits_pair_up(M):
    for seed in range(20):
        N = 1 + seed % (M - 1)
        key, a = _rand_case(M, 1000 * M + seed)
        s, rc, _ = oracle.block_round(key, a, N, 0, stage=1)
        r, c = s.sum(axis=1), s.sum(axis=0)
        assert (r <= N).all() and (c <= N).all()
        assert r.sum() == c.sum()
        short_r, short_c = np.where(r < N)[0], np.where(c < N)[0]
        assert len(short_r) > 0 or len(short_c) == 0
        assert (s[np.ix_(short_r, short_c)] == 1).all()


@pytest.mark.parametrize("M", [4, 8, 16, 32, 64])
def test_repair_and_local_search_properties(M):
    for seed in range(12):
        N = 1 + (seed * 7) % M
        key, a = _rand_case(M, 2000 * M + seed, dist="t3_outlier_cols")
        s2, rc2, st2 = oracle.block_round(key, a, N, 0, stage=2)
        assert rc2 == 0
        assert (s2.sum(axis=0) == N).all() and (s2.sum(axis=1) == N).all()
        s3, rc3, st3 = oracle.block_round(key, a, N, 60, stage=3)
        assert rc3 == 0
        assert (s3.sum(axis=0) == N).all() and (s3.sum(axis=1) == N).all()
        a64 = a.astype(np.float64)
        o2, o3 = (s2 * a64).sum(), (s3 * a64).sum()
        assert o3 >= o2 * (1 - 1e-6)
        opt, _ = oracle.block_opt(a, N)
        assert o3 <= opt * (1 + 1e-12)
        if st3["ls_swaps"] < 60 * M:
            # converged: no exchange of one entry between two rows gains
            for i in range(M):
                for ip in range(M):
                    if ip == i:
                        continue
                    give = np.where((s3[i] == 1) & (s3[ip] == 0))[0]
                    take = np.where((s3[i] == 0) & (s3[ip] == 1))[0]
                    if len(give) == 0:
                        continue
                    best = max(float(np.float32(a[ip, j] - a[i, j])) for j in give) + \
                        max(float(np.float32(a[i, j] - a[ip, j])) for j in take)
                    assert np.float32(best) <= 0.0


@pytest.mark.parametrize("M", [4, 8, 32])
def test_all_ones_when_N_equals_M(M):
    key, a = _rand_case(M, 77)
    s, rc, st = oracle.block_round(key, a, M, 4, stage=3)
    assert rc == 0 and (s == 1).all() and st["repairs"] == 0


def test_full_256x256_2of4_pipeline():
    w = synth.WORKLOADS["w256x256_f32_normal_2of4"]
    _, W = synth.workload_matrix(w)
    m, keys, st = oracle.mask(W, w.N, w.M, w.tau, w.iters, w.sweeps, want_keys=True)
    assert st["failures"] == 0
    obj = oracle.objective(W, m, w.N, w.M)
    assert not np.isnan(obj).any()
    opt, _ = oracle.opt(W, w.N, w.M)
    assert (obj <= opt * (1 + 1e-12)).all()
    gap = (opt - obj) / opt
    # the pages claim 1-10% relative error; the oracle must stay inside it
    assert gap.mean() <= 0.01 and gap.max() <= 0.10
    # rounding the oracle's own keys again gives the same masks
    m2, st2 = oracle.round_plan(keys, W, w.N, w.M, w.sweeps)
    assert (m2 == m).all()


@pytest.mark.parametrize("name", ["w4096x4096_bf16_normal_8of16", "w4096x11008_bf16_t3_16of32",
                                  "w8192x28672_bf16_laplace_32of64"])
def test_config_samples_quality(name):
    w = synth.WORKLOADS[name]
    nb = 16 if w.M == 64 else 64
    _, W = synth.make_matrix(w.M, nb * w.M, w.dtype, w.dist, w.scale, 5)
    m, _, st = oracle.mask(W, w.N, w.M, w.tau, w.iters, w.sweeps)
    obj = oracle.objective(W, m, w.N, w.M)
    opt, _ = oracle.opt(W, w.N, w.M)
    assert st["failures"] == 0 and not np.isnan(obj).any()
    assert (obj <= opt * (1 + 1e-12)).all()
    assert ((opt - obj) / opt).max() <= 0.10


def test_non_finite_block_fails_alone():
    W = synth.random_blocks(3, 8, seed=9)
    W[2, 9] = np.nan          # block 1
    W[5, 20] = np.inf         # block 2
    m, _, st = oracle.mask(W, 4, 8, 20.0, 50, 2)
    assert st["failures"] == 2
    bits = oracle.unpack(m, W.shape[1])
    assert (bits[:, 8:24] == 0).all()
    assert (bits[:, :8].sum(axis=0) == 4).all()


def test_argument_errors():
    W = np.zeros((8, 12), np.float32)
    with pytest.raises(ValueError):
        oracle.mask(W, 2, 8, 10.0, 5, 1)      # 12 is not a multiple of 8
    with pytest.raises(ValueError):
        oracle.mask(W[:, :8], 9, 8, 10.0, 5, 1)   # N > M
