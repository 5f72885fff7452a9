"""Pins for the oracle's exact optimum (min-cost flow b-matching).

The TSENOR review states that the block problem's LP relaxation is exact
(Core claim: bipartite matching polytope; "Assumptions & free parameters":
standard math, integral optimum), so the flow optimum must equal
  - the maximum over every feasible mask (brute force: 90 masks for 2:4,
    297,200 for 3:6 -- the counts themselves are checked),
  - the optimum of the LP relaxation solved by an independent LP solver
    (scipy HiGHS),
  - for N = 1, the assignment-problem optimum (scipy's Hungarian-type solver),
  - for N = M - 1, total mass minus a minimum-weight perfect matching,
  - for N = M, the total mass.
"""
import itertools

import numpy as np
import pytest
from scipy.optimize import linear_sum_assignment, linprog

import oracle
import synth


def feasible_masks(M, N):
    """Every MxM 0/1 matrix with all row and column sums equal to N."""
    pats = np.array([[1 if j in c else 0 for j in range(M)]
                     for c in itertools.combinations(range(M), N)], dtype=np.int8)
    states = np.zeros((1, 0), dtype=np.int8)
    counts = np.zeros((1, M), dtype=np.int8)
    for _ in range(M - 1):
        ns = states.shape[0]
        new_counts = (counts[:, None, :] + pats[None, :, :]).reshape(-1, M)
        keep = (new_counts <= N).all(axis=1)
        rows = np.broadcast_to(pats[None], (ns, len(pats), M)).reshape(-1, M)
        prev = np.repeat(states, len(pats), axis=0)
        states = np.concatenate([prev, rows], axis=1)[keep]
        counts = new_counts[keep]
    last = (N - counts).astype(np.int8)
    ok = ((last == 0) | (last == 1)).all(axis=1)
    return np.concatenate([states[ok], last[ok]], axis=1)


def test_feasible_mask_counts():
    # 2n x 2n binary matrices with all line sums n: 2, 90, 297200 for n = 1, 2, 3.
    assert len(feasible_masks(2, 1)) == 2
    assert len(feasible_masks(4, 2)) == 90
    assert len(feasible_masks(6, 3)) == 297200


def _blocks(W, M):
    return oracle.blocks_view(np.abs(W), M).reshape(-1, M * M)


def test_opt_equals_brute_force_2of4_full_256():
    w = synth.WORKLOADS["w256x256_f32_normal_2of4"]
    _, W = synth.workload_matrix(w)
    masks = feasible_masks(4, 2).astype(np.float64)
    bf = (_blocks(W, 4).astype(np.float64) @ masks.T).max(axis=1)
    opt, m = oracle.opt(W, 2, 4, want_mask=True)
    np.testing.assert_allclose(opt, bf, rtol=1e-12, atol=0)
    # the returned mask is feasible and attains the value
    obj = oracle.objective(W, m, 2, 4)
    np.testing.assert_allclose(obj, opt, rtol=1e-12)


def test_opt_equals_brute_force_3of6():
    W = synth.random_blocks(200, 6, seed=7, dist="laplace_outliers", scale=0.014)
    masks = feasible_masks(6, 3).astype(np.float64)
    bf = (_blocks(W, 6).astype(np.float64) @ masks.T).max(axis=1)
    opt, _ = oracle.opt(W, 3, 6)
    np.testing.assert_allclose(opt, bf, rtol=1e-12, atol=0)


def _lp_opt(a, N):
    M = a.shape[0]
    A_eq = np.zeros((2 * M, M * M))
    for i in range(M):
        A_eq[i, i * M:(i + 1) * M] = 1
        A_eq[M + i, i::M] = 1
    res = linprog(-a.ravel().astype(np.float64), A_eq=A_eq, b_eq=np.full(2 * M, N),
                  bounds=(0, 1), method="highs")
    assert res.status == 0
    return -res.fun


@pytest.mark.parametrize("M,N,dist", [(8, 3, "normal"), (8, 4, "t3_outlier_cols"),
                                      (16, 5, "normal"), (16, 8, "laplace_outliers"),
                                      (32, 16, "normal")])
def test_opt_equals_lp_relaxation(M, N, dist):
    W = synth.random_blocks(6, M, seed=100 + M + N, dist=dist, dtype="bf16", scale=0.02)
    opt, _ = oracle.opt(W, N, M)
    blocks = oracle.blocks_view(np.abs(W), M).reshape(-1, M, M)
    for b, a in enumerate(blocks):
        assert opt[b] == pytest.approx(_lp_opt(a, N), rel=1e-9)


@pytest.mark.parametrize("M", [4, 16, 32, 64])
def test_opt_assignment_N1(M):
    W = synth.random_blocks(5, M, seed=3 * M, dist="normal")
    opt, _ = oracle.opt(W, 1, M)
    for b, a in enumerate(oracle.blocks_view(np.abs(W), M).reshape(-1, M, M)):
        r, c = linear_sum_assignment(a.astype(np.float64), maximize=True)
        assert opt[b] == pytest.approx(a[r, c].astype(np.float64).sum(), rel=1e-12)


@pytest.mark.parametrize("M", [8, 32])
def test_opt_complement_N_minus_1(M):
    W = synth.random_blocks(4, M, seed=5 * M, dist="uniform")
    opt, _ = oracle.opt(W, M - 1, M)
    for b, a in enumerate(oracle.blocks_view(np.abs(W), M).reshape(-1, M, M)):
        a64 = a.astype(np.float64)
        r, c = linear_sum_assignment(a64, maximize=False)
        assert opt[b] == pytest.approx(a64.sum() - a64[r, c].sum(), rel=1e-12)


def test_opt_N_equals_M():
    W = synth.random_blocks(3, 8, seed=11)
    opt, m = oracle.opt(W, 8, 8, want_mask=True)
    for b, a in enumerate(oracle.blocks_view(np.abs(W), 8).reshape(-1, 8, 8)):
        assert opt[b] == pytest.approx(a.astype(np.float64).sum(), rel=1e-12)
    assert (oracle.unpack(m, W.shape[1]) == 1).all()


def test_objective_bit_layout():
    # word w of row r holds columns 32w..32w+31, bit k = column 32w+k
    rng = np.random.default_rng(0)
    W = rng.standard_normal((8, 40)).astype(np.float32)
    bits = np.zeros((8, 40), dtype=np.uint8)
    bits[0, 0] = bits[0, 31] = bits[0, 32] = bits[0, 39] = 1
    words = oracle.pack(bits)
    assert words.shape == (8, 2)
    assert words[0, 0] == (1 | (1 << 31)) and words[0, 1] == (1 | (1 << 7))
    assert (oracle.unpack(words, 40) == bits).all()
    # a single-entry mask is never feasible for 1:8 blocks -> NaN
    obj = oracle.objective(W, words, 1, 8)
    assert np.isnan(obj).all()
    # the identity pattern inside every 8x8 block is feasible for N=1
    eye = np.zeros((8, 40), dtype=np.uint8)
    for bc in range(5):
        eye[np.arange(8), bc * 8 + np.arange(8)] = 1
    obj = oracle.objective(W, oracle.pack(eye), 1, 8)
    for bc in range(5):
        assert obj[bc] == pytest.approx(np.abs(W[np.arange(8), bc * 8 + np.arange(8)]).astype(np.float64).sum())
