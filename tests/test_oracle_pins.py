"""Pins of the float64 oracle to facts fixed by the paper and by mathematics,
not by the oracle itself.

Source: "Gated KalmaNet: A Fading Memory Layer Through Test-Time Ridge
Regression" (arXiv 2511.21016).
  * weighted ridge objective (Eq. 3) with weights eta_{t,i} = prod gamma_j and
    lambda_t = a ||H_t||_F -> exact least-squares solve (ai.info page, Main
    Findings and Methodology; pith.science appendix, "Adaptive weighting");
  * condition-number bound (a+1)/a (ai.info, Key Contributions 2);
  * Chebyshev iteration: error polynomial T_r and its bound, the weight
    schedule of Lemma 3 / Lemma 4 and the printed rate table for kappa = 51
    (pith.science appendix fragments);
  * chunk-wise ||H_t||_F equals the token-wise one (ai.info, Methodology).
"""
import json
import math
import os

import numpy as np
import numpy.polynomial.chebyshev as npcheb
import pytest

import oracle

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")


def T_r(r, x):
    """Chebyshev polynomial of the first kind (numpy's routine)."""
    return npcheb.chebval(x, [0.0] * r + [1.0])


def rng(seed):
    return np.random.default_rng(seed)


def unit_rows(x):
    return x / np.linalg.norm(x, axis=-1, keepdims=True)


# --------------------------------------------------------------------------
# Chebyshev weight schedule and the printed rate table
# --------------------------------------------------------------------------

def test_rate_table_kappa51_matches_page():
    g = json.load(open(os.path.join(GOLDEN, "cheb_rates_kappa51.json")))
    kappa = g["L"] / g["mu"]
    assert kappa == pytest.approx(g["kappa"], rel=1e-12)
    sk = math.sqrt(kappa)
    R = (kappa - 1) / (kappa + 1) * (sk - 1) / (sk + 1)
    Ra = (sk - 1) / (sk + 1)
    # each printed value carries 1-4 significant digits: allow one unit of its last digit
    for p, (val, unit) in g["R"].items():
        assert abs(R ** int(p) - val) <= unit, ("R", p, R ** int(p))
    for p, (val, unit) in g["R_a"].items():
        assert abs(Ra ** int(p) - val) <= unit, ("R_a", p, Ra ** int(p))


@pytest.mark.parametrize("a", [0.02, 0.1, 0.5, 2.0])
def test_omega_schedule_lemmas(a):
    # interval [a n, (1+a) n]: kappa = (1+a)/a, rho = (L-mu)/(L+mu) = 1/(1+2a)
    kappa = (1 + a) / a
    rho = (kappa - 1) / (kappa + 1)
    assert rho == pytest.approx(1 / (1 + 2 * a), rel=1e-14)
    n = 40
    w = oracle.omegas(rho, n)
    assert w[0] == 2.0
    w_star = 2 * (1 - math.sqrt(1 - rho ** 2)) / rho ** 2
    # fixed point of omega -> 1/(1 - rho^2 omega/4)
    assert 1 / (1 - rho ** 2 * w_star / 4) == pytest.approx(w_star, rel=1e-14)
    sk = math.sqrt(kappa)
    R = (kappa - 1) / (kappa + 1) * (sk - 1) / (sk + 1)
    for i in range(1, n):
        assert 1.0 <= w[i] <= 2.0                      # Lemma 3
        assert w[i] <= w[i - 1] + 1e-15                # monotone
        assert w[i] >= w_star * (1 - 1e-14)
        assert w[i] - w_star <= R ** i * (w[0] - w_star) * (1 + 1e-9) + 1e-15   # Lemma 4


@pytest.mark.parametrize("a", [0.1, 0.5])
def test_omega_equals_chebyshev_ratio(a):
    # textbook semi-iteration: omega_{k+1} = 2 tau_k / (rho tau_{k+1}), tau_k = T_k(1/rho);
    # the pages' omega_i (i >= 1) is the textbook omega_{i+1}
    rho = 1 / (1 + 2 * a)
    w = oracle.omegas(rho, 25)
    for i in range(1, 25):
        tau_i = T_r(i, 1 / rho)
        tau_n = T_r(i + 1, 1 / rho)
        assert w[i] == pytest.approx(2 * tau_i / (rho * tau_n), rel=1e-12)


# --------------------------------------------------------------------------
# Chebyshev solve: exact error polynomial and bound
# --------------------------------------------------------------------------

def _spd_with_spectrum(D, eigs, seed):
    Q, _ = np.linalg.qr(rng(seed).standard_normal((D, D)))
    return Q @ np.diag(eigs) @ Q.T, Q


@pytest.mark.parametrize("r", [1, 2, 3, 7, 10, 20])
def test_cheb_error_is_chebyshev_polynomial(r):
    D = 12
    mu, L = 0.3, 1.7
    eigs = np.linspace(mu, L, D)
    A, Q = _spd_with_spectrum(D, eigs, 11 + r)
    q = rng(5).standard_normal(D)
    x = oracle.cheb_solve(A, q, mu, L, r)
    xs = np.linalg.solve(A, q)
    d, c = (L + mu) / 2, (L - mu) / 2
    rho = c / d
    # e_r = P_r(I - A/d) e_0 with P_r(t) = T_r(t/rho)/T_r(1/rho), e_0 = -x*
    e0 = Q.T @ (-xs)
    er = Q.T @ (x - xs)
    pred = np.array([T_r(r, (1 - lam / d) / rho) / T_r(r, 1 / rho) for lam in eigs]) * e0
    np.testing.assert_allclose(er, pred, rtol=1e-9, atol=1e-13 * np.abs(xs).max())


@pytest.mark.parametrize("a,r", [(0.5, 10), (0.1, 30), (0.1, 5), (0.02, 20)])
def test_cheb_error_bound(a, r):
    D = 24
    mu, L = a, 1 + a
    eigs = np.concatenate([[mu, L], rng(3).uniform(mu, L, D - 2)])
    A, _ = _spd_with_spectrum(D, eigs, 7)
    q = rng(8).standard_normal(D)
    x = oracle.cheb_solve(A, q, mu, L, r)
    xs = np.linalg.solve(A, q)
    kappa = L / mu
    Ra = (math.sqrt(kappa) - 1) / (math.sqrt(kappa) + 1)
    bound = 2 * Ra ** r / (1 + Ra ** (2 * r))
    assert bound == pytest.approx(1 / T_r(r, (kappa + 1) / (kappa - 1)), rel=1e-9)
    assert np.linalg.norm(x - xs) <= np.linalg.norm(xs) * bound * (1 + 1e-9) + 1e-15


# --------------------------------------------------------------------------
# The layer against the weighted ridge regression it approximates
# --------------------------------------------------------------------------

def _ridge_outputs(q, k, v, beta, a):
    """o*_t = S_t q_t, S_t = argmin_S sum_i eta_{t,i}||S k_i - v_i||^2 + lambda_t ||S||_F^2,
    eta_{t,i} = prod_{j=i+1..t} beta_j, lambda_t = a ||sum_i eta_{t,i} k_i k_i^T||_F,
    solved as a stacked least-squares problem (numpy lstsq)."""
    T, D = q.shape
    out = np.zeros((T, D))
    norms = np.zeros(T)
    for t in range(T):
        eta = np.array([np.prod(beta[i + 1:t + 1]) for i in range(t + 1)])
        Hdef = sum(eta[i] * np.outer(k[i], k[i]) for i in range(t + 1))
        lam = a * np.linalg.norm(Hdef, "fro")
        norms[t] = lam / a
        Arows = np.vstack([np.sqrt(eta)[:, None] * k[:t + 1], math.sqrt(lam) * np.eye(D)])
        rhs = np.vstack([np.sqrt(eta)[:, None] * v[:t + 1], np.zeros((D, D))])
        St, *_ = np.linalg.lstsq(Arows, rhs, rcond=None)   # D x D, maps k -> v as k @ St
        out[t] = q[t] @ St
    return out, norms


@pytest.mark.parametrize("a,r,seed", [(0.5, 60, 0), (0.1, 160, 1), (1.0, 40, 2)])
def test_layer_equals_exact_ridge_regression(a, r, seed):
    g = rng(seed)
    T, D = 14, 5
    q = g.standard_normal((T, D))
    k = unit_rows(g.standard_normal((T, D))) * g.uniform(0.5, 2.0, (T, 1))
    v = g.standard_normal((T, D))
    beta = 1 / (1 + np.exp(-g.normal(1.0, 1.5, T)))
    ref, ref_norms = _ridge_outputs(q, k, v, beta, a)
    out = oracle.forward(q[None, None], k[None, None], v[None, None], beta[None, None], a, r,
                         want_norms=True)
    np.testing.assert_allclose(out["norms"][0, 0], ref_norms, rtol=1e-12)
    np.testing.assert_allclose(out["o"][0, 0], ref, rtol=1e-8, atol=1e-10)


@pytest.mark.parametrize("a,r", [(0.5, 10), (0.5, 11), (0.1, 30), (0.1, 3), (2.0, 1)])
def test_first_token_closed_form(a, r):
    # At t = 0, H = k k^T has eigenvalues exactly at mu = a||k||^2 and L = (1+a)||k||^2,
    # so x_r = x* - (x*_perp + (-1)^r x*_par)/T_r(1/rho) and, by Sherman-Morrison,
    # o_0 = v (k.q)/((1+a)||k||^2) (1 - (-1)^r / T_r(1/rho)).
    g = rng(100 + r)
    B, H, D = 2, 3, 16
    q = g.standard_normal((B, H, 1, D))
    k = g.standard_normal((B, H, 1, D))
    v = g.standard_normal((B, H, 1, D))
    beta = g.uniform(0, 1, (B, H, 1))
    o = oracle.forward(q, k, v, beta, a, r)["o"]
    rho = 1 / (1 + 2 * a)
    fac = 1 - (-1) ** r / T_r(r, 1 / rho)
    kk = (k * k).sum(-1, keepdims=True)
    kq = (k * q).sum(-1, keepdims=True)
    np.testing.assert_allclose(o, v * kq / ((1 + a) * kk) * fac, rtol=1e-11, atol=1e-14)


def test_beta_zero_resets_state():
    g = rng(7)
    T, D, a, r = 9, 8, 0.5, 6
    q = g.standard_normal((1, 1, T, D))
    k = unit_rows(g.standard_normal((1, 1, T, D)))
    v = g.standard_normal((1, 1, T, D))
    beta = g.uniform(0.3, 1.0, (1, 1, T))
    beta[0, 0, 5] = 0.0
    o = oracle.forward(q, k, v, beta, a, r)["o"][0, 0]
    rho = 1 / (1 + 2 * a)
    fac = 1 - (-1) ** r / T_r(r, 1 / rho)
    kk, kq = k[0, 0, 5] @ k[0, 0, 5], k[0, 0, 5] @ q[0, 0, 5]
    np.testing.assert_allclose(o[5], v[0, 0, 5] * kq / ((1 + a) * kk) * fac, rtol=1e-11)


def test_condition_number_bound_and_state():
    # tiny fp32 workload shape: B=1, heads=2, D=32, a=0.5 (prefixes of the sequence)
    g = rng(21)
    B, H, T, D, a = 1, 2, 48, 32, 0.5
    k = unit_rows(g.standard_normal((B, H, T, D)))
    q = unit_rows(g.standard_normal((B, H, T, D)))
    v = g.standard_normal((B, H, T, D))
    beta = 1 / (1 + np.exp(-g.normal(2.0, 0.5, (B, H, T))))
    full = oracle.forward(q, k, v, beta, a, 10, want_norms=True)
    for t in [0, 1, 5, 17, 47]:
        pre = oracle.forward(q[:, :, :t + 1], k[:, :, :t + 1], v[:, :, :t + 1],
                             beta[:, :, :t + 1], a, 10, want_final_state=True)
        for h in range(H):
            Ht = pre["final_state"][0, h, 0]
            n = full["norms"][0, h, t]
            assert np.linalg.norm(Ht, "fro") == pytest.approx(n, rel=1e-13)
            ev = np.linalg.eigvalsh(Ht + a * n * np.eye(D))
            assert ev.min() >= a * n * (1 - 1e-12)
            assert ev.max() <= (1 + a) * n * (1 + 1e-12)
            assert ev.max() / ev.min() <= (1 + a) / a * (1 + 1e-12)


# --------------------------------------------------------------------------
# Chunk-wise norm, chunk states, invariances, decode
# --------------------------------------------------------------------------

@pytest.mark.parametrize("C", [1, 4, 16, 32])
def test_chunked_norm_equals_tokenwise(C):
    g = rng(C)
    B, H, T, D = 1, 2, 64, 8
    k = unit_rows(g.standard_normal((B, H, T, D)))
    beta = 1 / (1 + np.exp(-g.normal(1.0, 1.0, (B, H, T))))
    beta[0, 1, 20] = 0.0   # a reset inside a chunk
    ref = oracle.forward(k, k, k, beta, 0.5, 1, want_norms=True)["norms"]
    got = oracle.chunked_norms(k, beta, C)
    np.testing.assert_allclose(got, ref, rtol=1e-12)


def test_chunk_states_are_prefix_states():
    g = rng(4)
    B, H, T, D, C = 1, 2, 32, 6, 8
    q, k, v = (g.standard_normal((B, H, T, D)) for _ in range(3))
    beta = g.uniform(0.2, 1.0, (B, H, T))
    out = oracle.forward(q, k, v, beta, 0.5, 4, chunk=C, want_chunk_states=True)
    cs = out["chunk_states"]
    assert np.all(cs[:, :, 0] == 0)
    for n in range(1, T // C):
        pre = oracle.forward(q[:, :, :n * C], k[:, :, :n * C], v[:, :, :n * C],
                             beta[:, :, :n * C], 0.5, 4, want_final_state=True)
        np.testing.assert_array_equal(cs[:, :, n], pre["final_state"])


def test_invariances():
    g = rng(9)
    B, H, T, D, a, r = 1, 2, 20, 8, 0.5, 8
    q1, q2, v1, v2 = (g.standard_normal((B, H, T, D)) for _ in range(4))
    k = unit_rows(g.standard_normal((B, H, T, D)))
    beta = g.uniform(0.3, 1.0, (B, H, T))
    f = lambda q, k, v: oracle.forward(q, k, v, beta, a, r)["o"]
    base = f(q1, k, v1)
    np.testing.assert_allclose(f(2.5 * q1 + q2, k, v1), 2.5 * base + f(q2, k, v1), rtol=1e-10,
                               atol=1e-12)
    np.testing.assert_allclose(f(q1, k, -1.5 * v1 + v2), -1.5 * base + f(q1, k, v2),
                               rtol=1e-10, atol=1e-12)
    s = 3.0
    np.testing.assert_allclose(f(q1, s * k, v1), base / s, rtol=1e-10, atol=1e-12)


def test_decode_steps_continue_the_forward():
    g = rng(12)
    B, H, T, D, a, r = 2, 2, 10, 8, 0.5, 7
    q, v = (g.standard_normal((B, H, T, D)) for _ in range(2))
    k = unit_rows(g.standard_normal((B, H, T, D)))
    beta = g.uniform(0.3, 1.0, (B, H, T))
    ref = oracle.forward(q, k, v, beta, a, r)["o"]
    pre = oracle.forward(q[:, :, :6], k[:, :, :6], v[:, :, :6], beta[:, :, :6], a, r,
                         want_final_state=True)
    st = pre["final_state"]
    for t in range(6, T):
        o, st = oracle.decode_step(st, q[:, :, t], k[:, :, t], v[:, :, t], beta[:, :, t], a, r)
        np.testing.assert_allclose(o, ref[:, :, t], rtol=1e-13, atol=1e-15)


def test_solve_from_skips_only_outputs():
    g = rng(13)
    B, H, T, D = 1, 1, 16, 4
    q, k, v = (g.standard_normal((B, H, T, D)) for _ in range(3))
    beta = g.uniform(0.3, 1.0, (B, H, T))
    full = oracle.forward(q, k, v, beta, 0.5, 5)["o"]
    part = oracle.forward(q, k, v, beta, 0.5, 5, solve_from=11)["o"]
    np.testing.assert_array_equal(part[:, :, 11:], full[:, :, 11:])
    assert np.all(part[:, :, :11] == 0)
