"""Pins for the oracle's warm start and adaptive stopping of the Dykstra loop.

The TSENOR review fixes the iteration count T and gives no convergence test
("Assumptions & free parameters"); the extension rests on the fact that the
row and column steps only add potentials and the clip only moves an amount
between x and its correction, so x + q = x0 - tau + U_i + V_j after every
clip.  None of the pins below restates the oracle's loop:
  - shift invariance: a cold start of the extended loop (x = x0 - tau) gives
    the plan of the literal start x0 at every iteration count;
  - the exported potentials reproduce the plan in closed form,
    S = exp(min(x0 - tau + U_i + V_j, 0));
  - restarting from the potentials of T1 iterations and running T2 more is
    the same as running T1 + T2 (the potentials are the whole state);
  - an independent linear-space (multiplicative) iteration started from the
    same potentials agrees at every finite iteration count;
  - from ANY starting potentials the loop converges to the unique KL
    projection, computed here by a quasi-Newton solve of its dual;
  - the stop rule: the reported count t is the first iteration whose largest
    potential step is <= tol, with the steps read off the potentials of
    separate runs of t-1 and t iterations.
"""
import numpy as np
import pytest
from scipy.optimize import minimize

import oracle
import synth


def x0_of(a, tau):
    m = float(a.max())
    return tau * (a.astype(np.float64) / m) if m > 0 else np.zeros(a.shape)


def blocks(M, n, seed, dist="t3_outlier_cols"):
    W = synth.random_blocks(n, M, seed=seed, dist=dist, dtype="bf16", scale=0.02)
    return list(oracle.blocks_view(np.abs(W), M).reshape(-1, M, M))


@pytest.mark.parametrize("M,N,tau,iters", [(4, 2, 10.0, 1), (4, 1, 20.0, 57), (8, 4, 20.0, 200),
                                           (16, 5, 20.0, 33), (32, 16, 20.0, 120), (64, 32, 30.0, 20)])
def test_cold_start_equals_literal_start(M, N, tau, iters):
    for a in blocks(M, 2, seed=M + iters):
        S_lit = oracle.block_plan(a, N, tau, iters)
        S, uv, t = oracle.block_plan_ext(a, N, tau, iters)
        assert t == iters
        np.testing.assert_allclose(S, S_lit, rtol=0, atol=1e-12)


@pytest.mark.parametrize("M,N,tau,iters", [(4, 2, 10.0, 3), (8, 3, 20.0, 150), (16, 8, 20.0, 80),
                                           (32, 16, 20.0, 60), (64, 32, 30.0, 15)])
def test_potentials_give_the_plan_in_closed_form(M, N, tau, iters):
    for a in blocks(M, 2, seed=3 * M + N):
        S, uv, _ = oracle.block_plan_ext(a, N, tau, iters)
        U, V = uv[:M], uv[M:]
        y = x0_of(a, tau) - tau + U[:, None] + V[None, :]
        np.testing.assert_allclose(S, np.exp(np.minimum(y, 0.0)), rtol=0, atol=1e-12)


def test_zero_block_potentials():
    M, N = 8, 3
    S, uv, t = oracle.block_plan_ext(np.zeros((M, M), np.float32), N, 20.0, 4)
    np.testing.assert_allclose(S, N / M, atol=1e-12)
    # y0 = -tau everywhere; the plan N/M needs U_i + V_j = tau + ln(N/M)
    np.testing.assert_allclose(uv[:M, None] + uv[None, M:], 20.0 + np.log(N / M), atol=1e-12)


@pytest.mark.parametrize("M,N,tau,t1,t2", [(4, 2, 10.0, 1, 1), (8, 4, 20.0, 37, 63), (16, 8, 20.0, 100, 5),
                                           (32, 16, 20.0, 150, 150), (64, 32, 30.0, 9, 11)])
def test_restart_from_potentials_continues_the_run(M, N, tau, t1, t2):
    for a in blocks(M, 2, seed=t1 + t2 + M):
        S_all, uv_all, _ = oracle.block_plan_ext(a, N, tau, t1 + t2)
        _, uv1, _ = oracle.block_plan_ext(a, N, tau, t1)
        S2, uv2, t = oracle.block_plan_ext(a, N, tau, t2, uv=uv1)
        assert t == t2
        np.testing.assert_allclose(S2, S_all, rtol=0, atol=1e-12)
        np.testing.assert_allclose(uv2, uv_all, rtol=1e-12, atol=1e-10)


def linear_space_from_potentials(a, N, tau, iters, U, V):
    """Multiplicative form of the three KL projections, started at the state
    S * Q = exp(x0 - tau) * exp(U_i) * exp(V_j) with S = min(that, 1)."""
    St = np.exp(x0_of(a, tau) - tau) * np.exp(U)[:, None] * np.exp(V)[None, :]
    S = np.minimum(St, 1.0)
    Q = St / S
    for _ in range(iters):
        S = S * (N / S.sum(axis=1))[:, None]
        S = S * (N / S.sum(axis=0))[None, :]
        St = S * Q
        S = np.minimum(St, 1.0)
        Q = St / S
    return S


@pytest.mark.parametrize("M,N,tau,iters", [(4, 2, 10.0, 1), (4, 2, 10.0, 30), (8, 4, 20.0, 100),
                                           (16, 6, 20.0, 40)])
def test_warm_start_matches_linear_space(M, N, tau, iters):
    rng = np.random.default_rng(M * 100 + iters)
    for a in blocks(M, 2, seed=M * 7 + iters):
        uv0 = rng.uniform(-3.0, 3.0, 2 * M)   # arbitrary starting potentials, some entries clipped
        S, _, _ = oracle.block_plan_ext(a, N, tau, iters, uv=uv0)
        ref = linear_space_from_potentials(a, N, tau, iters, uv0[:M], uv0[M:])
        np.testing.assert_allclose(S, ref, rtol=0, atol=1e-9)


def kl_projection(a, N, tau):
    """argmin KL(S || exp(x0)) over {rows = N, cols = N, S <= 1} via its dual
    (quasi-Newton on the potentials; the clip bound enters as max(z, 0))."""
    M = a.shape[0]
    x0 = x0_of(a, tau)

    def fun(p):
        z = x0 + p[:M, None] + p[None, M:]
        ez = np.exp(np.minimum(z, 0.0))
        f = np.where(z <= 0, ez, 1.0 + z)
        g = np.minimum(ez, 1.0)
        return f.sum() - N * p.sum(), np.concatenate([g.sum(axis=1) - N, g.sum(axis=0) - N])

    p0 = np.concatenate([np.full(M, -x0.mean()), np.zeros(M)])
    res = minimize(fun, p0, jac=True, method="BFGS", options={"gtol": 1e-13, "maxiter": 20000})
    z = x0 + res.x[:M, None] + res.x[None, M:]
    return np.exp(np.minimum(z, 0.0))


@pytest.mark.parametrize("M,N,tau,seed", [(4, 2, 10.0, 0), (8, 3, 10.0, 2), (8, 4, 20.0, 3)])
def test_any_warm_start_converges_to_the_kl_projection(M, N, tau, seed):
    a = np.abs(synth.random_blocks(1, M, seed=seed)).reshape(M, M)
    ref = kl_projection(a, N, tau)
    rng = np.random.default_rng(seed)
    for uv0 in (None, rng.uniform(-5.0, 5.0, 2 * M), rng.uniform(0.0, 10.0, 2 * M)):
        S, _, t = oracle.block_plan_ext(a, N, tau, 50000, tol=1e-13, uv=uv0)
        assert t < 50000
        np.testing.assert_allclose(S, ref, atol=2e-6)


@pytest.mark.parametrize("M,N,tau,tol", [(4, 2, 10.0, 1e-3), (8, 4, 20.0, 1e-4), (16, 8, 20.0, 1e-5),
                                         (32, 16, 20.0, 1e-3)])
def test_stop_rule_is_the_first_small_step(M, N, tau, tol):
    for a in blocks(M, 2, seed=int(-np.log10(tol)) + M):
        _, _, t = oracle.block_plan_ext(a, N, tau, 100000, tol=tol)
        assert 2 <= t < 100000

        def step(k):
            """Largest |r_i|, |c_j| of iteration k: potentials after k minus after k-1."""
            _, uk, _ = oracle.block_plan_ext(a, N, tau, k)
            _, ukm, _ = oracle.block_plan_ext(a, N, tau, k - 1) if k > 1 else (None, None, None)
            if ukm is None:
                return np.inf
            return float(np.abs(uk - ukm).max())

        # the per-iteration step of each potential is a single r_i or c_j
        assert step(t) <= tol * (1 + 1e-6)
        assert step(t - 1) > tol * (1 - 1e-6)


def test_converged_warm_start_stops_at_once():
    M, N, tau = 16, 8, 20.0
    for a in blocks(M, 2, seed=5):
        S, uv, t = oracle.block_plan_ext(a, N, tau, 100000, tol=1e-10)
        S2, uv2, t2 = oracle.block_plan_ext(a, N, tau, 100000, tol=1e-6, uv=uv)
        assert t2 == 1
        np.testing.assert_allclose(S2, S, atol=1e-8)


def test_matrix_level_matches_block_level():
    M, N, tau, iters, tol = 8, 4, 20.0, 300, 1e-4
    storage, W = synth.make_matrix(32, 48, "bf16", "t3_outlier_cols", 0.02, seed=9)
    W = W.copy()
    W[8:16, 16:24] = 0.0                     # a zero block
    W[0, 40] = np.nan                        # a non-finite block (block row 0, block col 5)
    res = oracle.solve_ext(W, N, M, tau, iters, sweeps=2, tol=tol, want_plan=True)
    nbc = 48 // M
    for b, a in enumerate(oracle.blocks_view(np.abs(W), M).reshape(-1, M, M)):
        if not np.isfinite(a).all():
            assert res["iters_used"][b] == 0 and np.isnan(res["potentials"][b]).all()
            continue
        S, uv, t = oracle.block_plan_ext(a, N, tau, iters, tol=tol)
        assert res["iters_used"][b] == t
        np.testing.assert_array_equal(res["potentials"][b], uv)
        br, bc = divmod(b, nbc)
        np.testing.assert_array_equal(res["plan"][br * M:(br + 1) * M, bc * M:(bc + 1) * M], S)
    # tol = 0 and a cold start: the masks of the literal pipeline
    res0 = oracle.solve_ext(W, N, M, tau, iters, sweeps=2)
    ref, _, _ = oracle.mask(W, N, M, tau, iters, 2)
    np.testing.assert_array_equal(res0["mask"], ref)
    assert (res0["iters_used"][np.isfinite(oracle.blocks_view(W, M)).all(axis=(2, 3)).reshape(-1)] == iters).all()
