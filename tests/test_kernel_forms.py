"""CPU checks of the algebraic and floating-point forms the kernels use in
place of the pages' definitions.  Dykstra ("What carries the argument"):

  - the anchor points rebuild the linear-form exponentials as a product of
    fp32 factors, which keeps a few ulps where the fp32 sum of the exponent's
    terms does not (below).

Rounding (2-in/1-out local search, "What carries the argument"):

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


# --- the anchor points of the kernels' linear-form exponentials --------------
# The kernels rebuild E = 2^(y0 + U_i + V_j) every 64 iterations.  The terms
# y0 and U_i + V_j are each of size up to tau * log2(e) and cancel; as a
# product, (E0_ij * 2^U_i) * 2^V_j with E0 = 2^y0 taken once from an fp64 y0,
# every entry carries a few fp32 roundings whatever the size of the terms.
# These checks emulate both forms in numpy (fp32 roundings explicit, the
# hardware exponential replaced by the correctly rounded one) against exact
# fp64 values.

def _exp2_wide(y):
    """fp32 2^y for fp64 y in [-126, 126]: y = n + f, n the nearest integer, the
    fp32 2^f scaled by the exact 2^n (the kernels' split)."""
    y = np.clip(np.asarray(y, np.float64), -126.0, 126.0)
    n = np.rint(y)
    f = (y - n).astype(np.float32)
    return (np.exp2(f.astype(np.float64)).astype(np.float32) * np.exp2(n).astype(np.float32)).astype(np.float32)


def test_exp2_split_is_within_two_roundings():
    rng = np.random.default_rng(0)
    y = np.concatenate([rng.uniform(-60.0, 60.0, 20000), rng.uniform(-0.5, 0.5, 2000), [-43.28, 0.0, 17.5]])
    got = _exp2_wide(y).astype(np.float64)
    rel = np.abs(got / np.exp2(y) - 1.0)
    assert rel.max() <= 2.0 ** -23          # f rounded (<= 2^-26 in the exponent) + one fp32 rounding


def test_product_anchor_keeps_a_few_ulps_where_the_fp32_sum_does_not():
    rng = np.random.default_rng(1)
    tau2 = 30.0 * 1.4426950408889634
    q = rng.uniform(0.0, 1.0, 50000)                # a / max|W|
    y0 = tau2 * q - tau2                            # in [-tau2, 0], fp64
    U = rng.uniform(0.0, tau2, q.size)              # row potentials of weak rows: large
    V = rng.uniform(-2.0, 2.0, q.size)
    exact = np.exp2(y0 + U + V)
    E0 = _exp2_wide(y0)
    prod = ((E0 * _exp2_wide(U)).astype(np.float32) * _exp2_wide(V)).astype(np.float32)
    rel_prod = np.abs(prod.astype(np.float64) / exact - 1.0)
    # fp32 sum of the terms, then the exponential (the form kept for very large tau)
    s = (y0.astype(np.float32) + (U.astype(np.float32) + V.astype(np.float32))).astype(np.float32)
    rel_sum = np.abs(np.exp2(s.astype(np.float64)) / exact - 1.0)
    assert rel_prod.max() <= 5 * 2.0 ** -24       # E0, 2^U, 2^V and two products
    assert rel_sum.max() >= 20 * 2.0 ** -24       # cancellation of terms of size ~tau2
    assert np.median(rel_sum) > 4 * np.median(rel_prod)


# --- the rounding sort's 32-bit keys (bf16 inputs, blocks of 256, 1024, 4096) ---
# The kernels sort on a 32-bit image of the rounding key (plan desc, |W| desc,
# flat index asc): the IB = log2 E low bits hold E-1-idx, the bits above them a
# bucket of the plan - nibble 15 and the |W| bits for a plan of exactly 1,
# nibble e-112 and the upper 28-IB mantissa bits for a plan in [2^-14, 1) (e
# its biased exponent), nibble 0 and the plan's bits shifted right by 2+IB
# below 2^-14; then odd-even transposition passes with the full key settle the
# runs that share a bucket; a block not settled after 8 passes, or holding a
# plan above 1, is sorted on the full key.

def _full_key(S, a, idx):
    return ((S.view(np.uint32).astype(np.uint64) << np.uint64(32))
            | (a.view(np.uint32).astype(np.uint64) & np.uint64(0xffff0000))
            | (np.uint64(0xffff) - idx.astype(np.uint64)))


def _key32(kb, E):
    IB = E.bit_length() - 1
    MB = 28 - IB
    u = np.uint64
    s = (kb >> u(32)) & u(0xffffffff)
    inv = kb & u(E - 1)
    a16 = (kb >> u(16)) & u(0xffff)
    ex = s >> u(23)
    bucket = np.where(s >= u(0x3F800000), (u(15) << u(MB)) | a16,
                      np.where(ex > u(112), ((ex - np.minimum(ex, u(112))) << u(MB)) | ((s >> u(23 - MB)) & u((1 << MB) - 1)),
                               s >> u(30 - MB)))
    return (bucket << u(IB)) | inv


def _clipped32(x):
    return (x >> 28) == 15


def _sort32_then_settle(S, a, E, passes=8):
    """The kernels' order by the 32-bit keys and the settling passes; None = not settled."""
    kb = _full_key(S, a, np.arange(E))
    k = sorted((int(v) for v in _key32(kb, E)), reverse=True)
    full = [int(v) for v in kb]
    idx = lambda x: (E - 1) - (x & (E - 1))

    def later_first(x, y):
        if _clipped32(x) or ((x ^ y) & ~(E - 1)):
            return False
        return full[idx(y)] > full[idx(x)]
    for _ in range(passes):
        moved = False
        for start in (0, 1):
            for q in range(start, E - 1, 2):
                if later_first(k[q], k[q + 1]):
                    k[q], k[q + 1] = k[q + 1], k[q]
                    moved = True
        if not moved:
            return [idx(v) for v in k]
    return None


@pytest.mark.parametrize("E", [256, 1024, 4096])
def test_32bit_sort_keys_give_the_rounding_order(E):
    rng = np.random.default_rng(E)
    settled = 0
    for t in range(12):
        S = rng.random(E).astype(np.float32)
        if t % 3 == 0:
            S[rng.random(E) < 0.3] = 1.0                     # clipped entries
        if t % 2 == 1:
            S = (np.round(S * 500) / 500).astype(np.float32)  # many equal and near-equal plans
        a = (np.abs(rng.standard_normal(E)).astype(np.float32).view(np.uint32) & 0xffff0000).view(np.float32)
        if t % 4 == 0:
            a[rng.random(E) < 0.5] = 0.0                     # ties of |W|
        kb = _full_key(S, a, np.arange(E))
        truth = sorted(range(E), key=lambda i: -int(kb[i]))
        got = _sort32_then_settle(S, a, E)
        if got is not None:
            settled += 1
            assert got == truth
    assert settled >= 1
    # a constant block: the index decides, as in the 32-bit keys, and nothing moves
    assert _sort32_then_settle(np.full(E, 0.5, np.float32), np.full(E, 1.0, np.float32), E) == list(range(E))
    # equal plans with |W| rising along the index reverse the whole block: it does not
    # settle in 8 passes, and the 64-bit sort takes it
    ramp = ((np.arange(E, dtype=np.float32) + 1.0).view(np.uint32) & 0xffff0000).view(np.float32)
    assert _sort32_then_settle(np.full(E, 0.5, np.float32), ramp, E) is None


@pytest.mark.parametrize("E", [256, 1024, 4096])
def test_32bit_key_buckets_are_monotone_in_the_full_key(E):
    """A larger full key never gets a smaller bucket: so two keys can only be
    out of order within a bucket, which is all the settling passes look at."""
    rng = np.random.default_rng(7 + E)
    n = 200000
    # plans over every range the bucket treats apart: 1, the window's binades,
    # below 2^-14 down to subnormals and 0, and the window's edges
    S = np.concatenate([
        np.ones(1000, np.float32),
        rng.random(n // 2).astype(np.float32),
        np.exp2(rng.uniform(-30, 0, n // 2)).astype(np.float32),
        np.array([0.0, 1e-45, 2.0 ** -126, 2.0 ** -14, np.nextafter(np.float32(2.0 ** -14), np.float32(0)),
                  np.nextafter(np.float32(1), np.float32(0)), 0.5], np.float32)])
    a = (np.abs(rng.standard_normal(S.size)).astype(np.float32).view(np.uint32) & 0xffff0000).view(np.float32)
    a[:50] = 0.0
    idx = rng.integers(0, E, S.size)
    kb = _full_key(S, a, idx)
    k32 = _key32(kb, E)
    order = np.argsort(kb, kind="stable")
    b = (k32 >> np.uint64(E.bit_length() - 1))[order]
    assert (np.diff(b.astype(np.int64)) >= 0).all()
    # the clipped bucket sits above every other, and is exact among its own entries
    clipped = S == 1.0
    assert k32[clipped].min() > k32[~clipped].max()
    assert _clipped32(int(k32[clipped][0])) and not _clipped32(int(k32[~clipped].max()))
    # the window keeps 28 - log2 E mantissa bits: plans one step of that size apart differ
    MB = 28 - (E.bit_length() - 1)
    x = np.float32(0.3)
    y = (x.view(np.uint32) + np.uint32(1 << (23 - MB))).view(np.float32)
    kx, ky = _key32(_full_key(np.array([x, y]), np.zeros(2, np.float32), np.zeros(2, np.int64)), E)
    assert (ky >> np.uint64(E.bit_length() - 1)) == (kx >> np.uint64(E.bit_length() - 1)) + np.uint64(1)


def test_bc_swizzle_is_a_permutation_and_spreads_bank_groups():
    """The M = 64 local search stores logical 16-byte chunk c of row r at
    c ^ (r % 16) ^ (4 if c >= 8): a permutation of each row's 16 chunks; chunk
    c of 4 consecutive rows and chunks c, c + 8 of one row (the two threads of
    a row) land in distinct bank groups (a bank group: 4 banks = chunk mod 8)."""
    def phys(r, c):
        return (c ^ (r % 16) ^ (4 if c >= 8 else 0)) & 15

    for r in range(64):
        assert sorted(phys(r, c) for c in range(16)) == list(range(16))
        for q in range(8):
            assert phys(r, q) % 8 != phys(r, q + 8) % 8              # one row, both halves
    for r0 in range(64):
        for q in range(8):
            rows = [(r0 + k) % 64 for k in range(4)]               # a quarter warp: 4 rows, 2 threads each
            groups = [phys(r, q) % 8 for r in rows] + [phys(r, q + 8) % 8 for r in rows]
            assert len(set(groups)) == 8


def test_best_partner_update_without_rescan_equals_rescan():
    """After a swap of rows i and bp only the gains g(y, i), g(y, bp) of a row y
    change.  The local search rescans row y only when its best partner was i or
    bp AND its new gain with that partner fell below the old best; otherwise it
    compares the old best with the two new gains (lowest partner on ties).  On
    random tie-heavy gain tables that must equal a full rescan."""
    rng = np.random.default_rng(3)

    def rescan(G, y):
        bv, bp = -np.inf, -1
        for x in range(G.shape[0]):
            if bp < 0 or G[y, x] > bv:
                bv, bp = G[y, x], x
        return bv, bp

    checked = 0
    for t in range(900):
        M = (8, 16, 32)[t % 3]
        lv = int(rng.integers(1, 5))
        G = np.triu(rng.integers(-lv, lv + 1, (M, M)).astype(float), 1)
        G = G + G.T
        np.fill_diagonal(G, -np.inf)
        old = [rescan(G, y) for y in range(M)]
        i, bp = (int(v) for v in rng.choice(M, 2, replace=False))
        for y in range(M):
            if y != i:
                G[i, y] = G[y, i] = float(rng.integers(-lv, lv + 1))
        for y in range(M):
            if y not in (i, bp):
                G[bp, y] = G[y, bp] = float(rng.integers(-lv, lv + 1))
        for y in range(M):
            if y in (i, bp):
                continue
            ov, op = old[y]
            gi, gb = G[y, i], G[y, bp]
            if op in (i, bp) and (gi if op == i else gb) < ov:
                continue                                       # rescanned
            bv, b2 = ov, op
            c1, c2 = min(i, bp), max(i, bp)
            for c, g in ((c1, gi if c1 == i else gb), (c2, gi if c2 == i else gb)):
                if g > bv or (g == bv and c < b2):
                    bv, b2 = g, c
            assert (bv, b2) == rescan(G, y)
            checked += 1
    assert checked > 10000
