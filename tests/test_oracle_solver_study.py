"""Pins of the oracle's solver study (ai.info page, Key Contributions 2 and Main
Findings: CH against gradient descent, accelerated gradient descent and conjugate
gradient; pith.science page, Fig. 1a and Fig. 8: residual norms per iteration).

Each solver is fixed by something outside the oracle's code:
  * gradient descent with step 1/d and Nesterov's method with step 1/L and momentum
    (sqrt(kappa) - 1)/(sqrt(kappa) + 1) act on each eigen-direction of A by a scalar
    recurrence, evaluated here with numpy's eigendecomposition;
  * conjugate gradient equals SciPy's implementation iterate by iterate, and ends
    within D steps in exact arithmetic;
  * Chebyshev equals the oracle's pinned r-step solve for every r;
  * the layer-level study equals the per-system routine on each token's explicit
    A_t = H_t + a ||H_t||_F I built from the oracle's pinned forward states.
"""
import numpy as np
import pytest
import scipy.sparse.linalg as spla

import oracle


def rng(seed):
    return np.random.default_rng(seed)


def _system(D, mu, L, seed):
    g = rng(seed)
    Q, _ = np.linalg.qr(g.standard_normal((D, D)))
    eigs = np.concatenate([[mu, L], g.uniform(mu, L, D - 2)])
    return Q @ np.diag(eigs) @ Q.T, Q, eigs, g.standard_normal(D)


def _rel_res(A, q, x):
    return np.linalg.norm(q - A @ x) / np.linalg.norm(q)


@pytest.mark.parametrize("a", [0.5, 0.05])
def test_gradient_descent_per_eigen_direction(a):
    D, r = 10, 15
    mu, L = a, 1 + a
    A, Q, eigs, q = _system(D, mu, L, 1)
    d = (L + mu) / 2
    c0 = Q.T @ q
    # residual component along eigenvector j after i steps: (1 - lam_j / d)^i c0_j
    ref = [np.linalg.norm((1 - eigs / d) ** i * c0) / np.linalg.norm(q) for i in range(r + 1)]
    np.testing.assert_allclose(oracle.solver_residuals(A, q, mu, L, r, "gd"), ref, rtol=1e-10)


@pytest.mark.parametrize("a", [0.5, 0.05])
def test_nesterov_per_eigen_direction(a):
    D, r = 10, 15
    mu, L = a, 1 + a
    A, Q, eigs, q = _system(D, mu, L, 2)
    kap = L / mu
    m = (np.sqrt(kap) - 1) / (np.sqrt(kap) + 1)
    # error e = x - x*, per eigen-direction: y = e_i + m (e_i - e_{i-1}), e_{i+1} = (1 - lam/L) y
    xs = Q.T @ np.linalg.solve(A, q)
    e_prev = -xs.copy()
    e = -xs.copy()
    ref = [1.0]
    for _ in range(r):
        y = e + m * (e - e_prev)
        e_prev, e = e, (1 - eigs / L) * y
        ref.append(np.linalg.norm(eigs * e) / np.linalg.norm(q))
    np.testing.assert_allclose(oracle.solver_residuals(A, q, mu, L, r, "agd"), ref, rtol=1e-9)


@pytest.mark.parametrize("a", [0.5, 0.05])
def test_conjugate_gradient_matches_scipy_and_terminates(a):
    D, r = 12, 12
    mu, L = a, 1 + a
    A, _, _, q = _system(D, mu, L, 3)
    got = oracle.solver_residuals(A, q, mu, L, r, "cg")
    for i in range(1, 7):
        x, _ = spla.cg(A, q, x0=np.zeros(D), maxiter=i, rtol=0.0, atol=0.0)
        assert got[i] == pytest.approx(_rel_res(A, q, x), rel=1e-6, abs=1e-12), i
    assert got[D] < 1e-9


@pytest.mark.parametrize("r", [1, 2, 5, 10])
def test_chebyshev_matches_the_pinned_solve(r):
    D, a = 9, 0.3
    mu, L = a, 1 + a
    A, _, _, q = _system(D, mu, L, 4)
    got = oracle.solver_residuals(A, q, mu, L, r, "chebyshev")
    for i in range(1, r + 1):
        x = oracle.cheb_solve(A, q, mu, L, i)
        assert got[i] == pytest.approx(_rel_res(A, q, x), rel=1e-10), i


@pytest.mark.parametrize("solver", ["chebyshev", "gd", "agd", "cg"])
def test_layer_study_uses_each_tokens_system(solver):
    g = rng(5)
    B, H, T, D, a, r = 1, 2, 12, 6, 0.1, 8
    q = g.standard_normal((B, H, T, D))
    k = g.standard_normal((B, H, T, D))
    k /= np.linalg.norm(k, axis=-1, keepdims=True)
    beta = g.uniform(0.5, 1.0, (B, H, T))
    gate = g.uniform(0.2, 1.0, (B, H, T))
    got = oracle.solver_study(q, k, beta, a, r, solver, gate=gate)
    for t in (0, 5, 11):
        st = oracle.forward(q[:, :, :t + 1], k[:, :, :t + 1], k[:, :, :t + 1], beta[:, :, :t + 1],
                            a, 1, gate=gate[:, :, :t + 1], want_final_state=True)["final_state"]
        for h in range(H):
            Ht = st[0, h, 0]
            n = np.linalg.norm(Ht)
            ref = oracle.solver_residuals(Ht + a * n * np.eye(D), q[0, h, t], a * n, (1 + a) * n,
                                          r, solver)
            np.testing.assert_allclose(got[0, h, t], ref, rtol=1e-10, atol=1e-14)


def test_study_on_the_solver_study_shape_orders_the_methods():
    # the paper's observation on its random-regression setup: CG drops fastest in the
    # first iterations and CH reaches the smallest residuals by the end
    g = rng(6)
    B, H, T, D, a, r = 1, 2, 48, 16, 0.1, 30
    q = g.standard_normal((B, H, T, D))
    k = g.standard_normal((B, H, T, D))
    k /= np.linalg.norm(k, axis=-1, keepdims=True)
    beta = 1 / (1 + np.exp(-g.normal(3.0, 1.0, (B, H, T))))
    res = {s: oracle.solver_study(q, k, beta, a, r, s).mean(axis=(0, 1, 2)) for s in oracle.SOLVERS}
    assert res["cg"][3] < res["chebyshev"][3] < res["gd"][3]
    assert res["chebyshev"][r] < res["gd"][r] and res["chebyshev"][r] < res["agd"][r]
