"""CPU checks of the algebraic forms the rounding kernels use in place of the
pages' definitions (2-in/1-out local search, "What carries the argument"):

  - pair gains in max-plus form: with C_x[j] = a_xj off row x's support
    (-inf on it) and Bn_x[j] = a_xj on it (+inf off it),
        max over j in O_x \\ O_y of (a_yj - a_xj) = max_j (C_y[j] - Bn_x[j])
        max over j in O_y \\ O_x of (a_xj - a_yj) = max_j (C_x[j] - Bn_y[j])
    as the same fp32 differences (no rounding step differs);
  - the best-partner rescan by quads over a gain row whose diagonal holds
    -inf equals the sequential scan that skips the row itself (lowest
    partner index on ties) whenever some partner gain is finite;
  - with N < M every row of a valid N:M block has a partner of finite gain
    (two rows with the same support in every pair would put M ones in those
    columns), which is what lets the rescan drop the test for the row itself.

Plain numpy, fp32 where the kernels are fp32; nothing here calls the CUDA path.
"""
import itertools

import numpy as np
import pytest

F32 = np.float32


def random_valid_mask(M, N, rng):
    """A random valid N:M block mask: a circulant pattern ((j - i) mod M in a
    random N-subset) with rows and columns randomly permuted."""
    S = rng.choice(M, size=N, replace=False)
    base = np.isin((np.arange(M)[None, :] - np.arange(M)[:, None]) % M, S)
    mask = base[rng.permutation(M)][:, rng.permutation(M)]
    assert (mask.sum(0) == N).all() and (mask.sum(1) == N).all()
    return mask


def pair_terms_bit_tested(a, mask, x, y):
    t1 = -np.inf
    t2 = -np.inf
    for j in range(a.shape[1]):
        d = F32(a[y, j] - a[x, j])                  # fp32 difference, as the kernels take it
        if mask[x, j] and not mask[y, j]:
            t1 = max(t1, d)
        if mask[y, j] and not mask[x, j]:
            t2 = max(t2, F32(a[x, j] - a[y, j]))
    return t1, t2


def pair_terms_max_plus(a, mask, x, y):
    C = np.where(mask, -np.inf, a).astype(F32)
    Bn = np.where(mask, a, np.inf).astype(F32)
    with np.errstate(invalid="raise"):
        t1 = (C[y] - Bn[x]).max()
        t2 = (C[x] - Bn[y]).max()
    return t1, t2


@pytest.mark.parametrize("M,N", [(4, 2), (8, 4), (16, 8), (32, 16), (32, 31)])
def test_max_plus_pair_gains_equal_bit_tested(M, N):
    rng = np.random.default_rng(M * 100 + N)
    for trial in range(6):
        a = np.abs(rng.standard_normal((M, M))).astype(F32)
        if trial % 2:
            a = np.round(a * 4).astype(F32) / F32(4)       # ties and exact zeros
        mask = random_valid_mask(M, N, rng)
        for x, y in itertools.permutations(range(M), 2):
            ref = pair_terms_bit_tested(a, mask, x, y)
            got = pair_terms_max_plus(a, mask, x, y)
            assert got[0] == ref[0] and got[1] == ref[1]


def rescan_sequential(g, x):
    bv, bp = -np.inf, -1
    for y in range(len(g)):
        if y == x:
            continue
        if bp < 0 or g[y] > bv:
            bv, bp = g[y], y
    return bv, bp


def rescan_quads(g, x):
    g = g.copy()
    g[x] = -np.inf                                     # the table's diagonal
    bv, bp = -np.inf, -1
    for q in range(len(g) // 4):
        g0, g1, g2, g3 = g[4 * q:4 * q + 4]
        v01, i01 = (g1, 4 * q + 1) if g1 > g0 else (g0, 4 * q)
        v23, i23 = (g3, 4 * q + 3) if g3 > g2 else (g2, 4 * q + 2)
        vq, iq = (v23, i23) if v23 > v01 else (v01, i01)
        if q == 0 or vq > bv:
            bv, bp = vq, iq
    return bv, bp


@pytest.mark.parametrize("M", [4, 8, 16, 32])
def test_quad_rescan_equals_sequential_scan(M):
    rng = np.random.default_rng(7 + M)
    for _ in range(400):
        g = rng.integers(-3, 3, M).astype(F32)         # many ties
        g[rng.random(M) < 0.3] = -np.inf               # partners with no exchange
        x = int(rng.integers(M))
        if np.isneginf(np.delete(g, x)).all():
            g[(x + 1) % M] = F32(0)                    # some partner finite (see the next test)
        assert rescan_quads(g, x) == rescan_sequential(g, x)


@pytest.mark.parametrize("M,N", [(4, 1), (4, 3), (8, 7), (16, 15), (32, 31), (64, 32)])
def test_every_row_has_a_partner_with_another_support(M, N):
    rng = np.random.default_rng(M + N)
    for _ in range(20):
        mask = random_valid_mask(M, N, rng)
        for x in range(M):
            assert any((mask[x] != mask[y]).any() for y in range(M) if y != x)
