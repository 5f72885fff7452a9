"""Pins for the oracle's entropic transport plan (Dykstra in log space).

What the TSENOR review fixes ("What carries the argument", "Core claim",
minor comment 2): the relaxed block problem with an entropy term is solved by
Dykstra's alternating KL projections onto {row sums = N}, {column sums = N}
and {S <= 1}.  The pins below do not restate the oracle's loop:
  - closed form: for an additive kernel the plan is N/M everywhere after one
    iteration, and the clip never binds;
  - the limit of Dykstra's algorithm is the KL projection of the kernel onto
    the intersection (Bregman/Dykstra theory), characterised by its dual;
    the dual is minimised here by a generic quasi-Newton solver;
  - an independent linear-space (multiplicative) formulation of the same
    iteration agrees at every finite iteration count, and so does the form
    the kernels carry (row scalings as clip thresholds, column factors on
    the exponentials, re-anchored from the accumulated potentials);
  - the entropic suboptimality bound 0 <= opt - <S,|W|> <= (m/tau) * F(S)
    with F(S) = -sum S log S <= N*M*log(M/N), which fixes the sign and the
    scale of tau in the kernel x0 = tau*|W|/max|W|.
"""
import numpy as np
import pytest
from scipy.optimize import minimize

import oracle
import synth


def kernel(a, tau):
    m = a.max()
    return tau * (a.astype(np.float64) / m) if m > 0 else np.zeros_like(a, dtype=np.float64)


@pytest.mark.parametrize("M,N", [(4, 2), (8, 3), (16, 8), (32, 16), (64, 32)])
@pytest.mark.parametrize("iters", [1, 7])
def test_additive_kernel_gives_uniform_plan(M, N, iters):
    rng = np.random.default_rng(M * 10 + N)
    # dyadic u, v so that u_i + v_j is exact in fp32
    u = rng.integers(0, 64, M) / 64.0; v = rng.integers(0, 64, M) / 64.0
    a = (u[:, None] + v[None, :]).astype(np.float32)
    assert (a.astype(np.float64) == u[:, None] + v[None, :]).all()
    S = oracle.block_plan(a, N, tau=20.0, iters=iters)
    np.testing.assert_allclose(S, N / M, rtol=0, atol=1e-9)


@pytest.mark.parametrize("M,N", [(4, 1), (16, 5)])
def test_zero_block_gives_uniform_plan(M, N):
    S = oracle.block_plan(np.zeros((M, M), np.float32), N, tau=20.0, iters=3)
    np.testing.assert_allclose(S, N / M, atol=1e-12)


def test_small_tau_tends_to_uniform():
    a = np.abs(synth.random_blocks(1, 8, seed=4)).reshape(8, 8)
    S = oracle.block_plan(a, 3, tau=1e-7, iters=50)
    np.testing.assert_allclose(S, 3 / 8, atol=1e-6)


def dual_plan(a, N, tau):
    """KL projection of exp(x0) onto {rows = N, cols = N, S <= 1} via its dual.

    The projection is S_ij = min(1, exp(x0_ij + u_i + v_j)) where (u, v)
    minimises sum_ij f(x0_ij + u_i + v_j) - N sum u - N sum v with
    f(z) = exp(z) for z <= 0 and 1 + z for z > 0 (convex, C^1).
    """
    M = a.shape[0]
    x0 = kernel(a, tau)

    def fun(p):
        z = x0 + p[:M, None] + p[None, M:]
        ez = np.exp(np.minimum(z, 0.0))
        f = np.where(z <= 0, ez, 1.0 + z)
        g = np.minimum(ez, 1.0)
        val = f.sum() - N * p.sum()
        grad = np.concatenate([g.sum(axis=1) - N, g.sum(axis=0) - N])
        return val, grad

    p0 = np.concatenate([np.full(M, -x0.mean()), np.zeros(M)])
    res = minimize(fun, p0, jac=True, method="BFGS", options={"gtol": 1e-13, "maxiter": 20000})
    z = x0 + res.x[:M, None] + res.x[None, M:]
    return np.minimum(np.exp(np.minimum(z, 0.0)), 1.0)


@pytest.mark.parametrize("M,N,tau,seed", [(4, 2, 10.0, 0), (4, 1, 5.0, 1), (8, 3, 10.0, 2),
                                          (8, 4, 20.0, 3)])
def test_converged_plan_is_the_kl_projection(M, N, tau, seed):
    a = np.abs(synth.random_blocks(1, M, seed=seed)).reshape(M, M)
    S = oracle.block_plan(a, N, tau=tau, iters=20000)
    ref = dual_plan(a, N, tau)
    # the dual solution is feasible to the solver's gradient tolerance
    np.testing.assert_allclose(ref.sum(axis=1), N, atol=1e-7)
    np.testing.assert_allclose(S, ref, atol=2e-6)
    # and the oracle's limit satisfies the constraints itself
    np.testing.assert_allclose(S.sum(axis=0), N, atol=1e-7)
    np.testing.assert_allclose(S.sum(axis=1), N, atol=1e-7)
    assert S.max() <= 1.0


def linear_space_dykstra(a, N, tau, iters):
    """Multiplicative (linear-space) form of the three KL projections."""
    S = np.exp(kernel(a, tau))
    Q = np.ones_like(S)
    for _ in range(iters):
        S = S * (N / S.sum(axis=1))[:, None]
        S = S * (N / S.sum(axis=0))[None, :]
        St = S * Q
        S = np.minimum(St, 1.0)
        Q = St / S
    return S


@pytest.mark.parametrize("M,N,tau,iters", [(4, 2, 10.0, 200), (8, 4, 20.0, 200), (16, 8, 20.0, 300),
                                           (32, 16, 20.0, 300), (64, 32, 30.0, 40)])
def test_log_space_matches_linear_space(M, N, tau, iters):
    W = synth.random_blocks(3, M, seed=M + iters, dist="t3_outlier_cols", dtype="bf16", scale=0.02)
    for a in oracle.blocks_view(np.abs(W), M).reshape(-1, M, M):
        S = oracle.block_plan(a, N, tau=tau, iters=iters)
        ref = linear_space_dykstra(a, N, tau, iters)
        np.testing.assert_allclose(S, ref, rtol=0, atol=1e-9)


def threshold_form_dykstra(a, N, tau, iters, anchor_every):
    """The same iteration in the form the kernels carry it: the state is
    y = y0 + U_i + V_j; between anchor points E = exp(y) = F / th_i, the row
    step replaces the row's clip threshold th_i by S_i / N (S_i the row sum of
    min(F, th_i)), the column step weighs min(F, th_i) by N / S_i and multiplies
    F by N / C_j; at an anchor point the logarithms of the thresholds and of
    the column factors' products move into U and V and F = exp(y0 + U + V)."""
    M = a.shape[0]
    y0 = kernel(a, tau) - tau
    U = np.zeros(M); V = np.zeros(M)
    F = np.exp(y0); th = np.ones(M); pv = np.ones(M)
    for t in range(iters):
        if t > 0 and t % anchor_every == 0:
            U -= np.log(th); V += np.log(pv)
            th = np.ones(M); pv = np.ones(M)
            F = np.exp(y0 + U[:, None] + V[None, :])
        e = np.minimum(F, th[:, None])
        S_row = e.sum(axis=1)
        C = (e * (N / S_row)[:, None]).sum(axis=0)
        u = N / C
        th = S_row / N
        F = F * u[None, :]
        pv = pv * u
    return np.minimum(F / th[:, None], 1.0)


@pytest.mark.parametrize("M,N,tau,iters", [(4, 2, 10.0, 200), (8, 4, 20.0, 200), (16, 8, 20.0, 300),
                                           (32, 16, 20.0, 300), (64, 32, 30.0, 40)])
@pytest.mark.parametrize("anchor_every", [1, 3, 64, 10 ** 9])
def test_log_space_matches_threshold_form(M, N, tau, iters, anchor_every):
    W = synth.random_blocks(3, M, seed=M + iters + 1, dist="t3_outlier_cols", dtype="bf16", scale=0.02)
    for a in oracle.blocks_view(np.abs(W), M).reshape(-1, M, M):
        S = oracle.block_plan(a, N, tau=tau, iters=iters)
        ref = threshold_form_dykstra(a, N, tau, iters, anchor_every)
        np.testing.assert_allclose(S, ref, rtol=0, atol=1e-9)


@pytest.mark.parametrize("M,N,tau", [(4, 2, 10.0), (8, 4, 20.0), (8, 2, 50.0), (16, 8, 100.0)])
def test_entropic_suboptimality_bound(M, N, tau):
    W = synth.random_blocks(4, M, seed=int(tau) + M, dist="normal")
    opt, _ = oracle.opt(W, N, M)
    for b, a in enumerate(oracle.blocks_view(np.abs(W), M).reshape(-1, M, M)):
        S = oracle.block_plan(a, N, tau=tau, iters=20000)
        val = float((S * a.astype(np.float64)).sum())
        F = float(-(S * np.log(np.maximum(S, 1e-300))).sum())
        m = float(a.max())
        gap = opt[b] - val
        assert gap >= -1e-7 * opt[b]
        assert gap <= m / tau * F + 1e-7 * opt[b]
        assert F <= N * M * np.log(M / N) + 1e-9


def test_gap_shrinks_as_tau_grows():
    a = np.abs(synth.random_blocks(1, 8, seed=21)).reshape(8, 8)
    opt, _ = oracle.block_opt(a, 4)
    gaps = []
    for tau in (2.0, 8.0, 32.0, 128.0):
        S = oracle.block_plan(a, 4, tau=tau, iters=20000)
        gaps.append(opt - float((S * a.astype(np.float64)).sum()))
    assert all(g1 > g2 for g1, g2 in zip(gaps, gaps[1:]))
    assert gaps[-1] >= -1e-9


def test_plan_bounds_at_finite_iterations():
    w = synth.WORKLOADS["w256x256_f32_normal_2of4"]
    _, W = synth.workload_matrix(w)
    P = oracle.plan(W[:64, :64], w.N, w.M, w.tau, w.iters)
    assert (P <= 1.0).all() and (P > 0.0).all()
    # a fixed T with no stopping test (free parameter T) leaves the plans
    # close to, but not exactly on, the transport constraints
    B = oracle.blocks_view(P, 4)
    err = np.maximum(np.abs(B.sum(axis=3) - 2.0).max(axis=2), np.abs(B.sum(axis=2) - 2.0).max(axis=2))
    assert err.max() < 0.05
    assert np.median(err) < 1e-4

