"""Pins of the oracle's write-gated recurrence (the paper's beta_t-augmented
variant: a per-token input-selectivity gate in [0, 1] scales each token's write
into H_t and U_t; ai.info page, Main Findings, and Future Directions).  Here the
gate is g_t and the decay beta_t:
    H_t = beta_t H_{t-1} + g_t k_t k_t^T,   M_t = beta_t M_{t-1} + g_t v_t k_t^T.

What fixes the gated layer independently of the oracle's own code:
  * it is the weighted ridge regression of Eq. 3 with token i's weight
    eta_{t,i} g_i (exact least squares on tiny inputs, numpy lstsq);
  * g k k^T = (sqrt(g) k)(sqrt(g) k)^T and g v k^T = (sqrt(g) v)(sqrt(g) k)^T, so it
    equals the ungated layer (pinned in test_oracle_pins) on rescaled keys and values;
  * a constant gate c scales H, M and lambda by c and leaves o unchanged;
  * g = 1 everywhere is the ungated layer, bit for bit.
"""
import math

import numpy as np
import pytest

import oracle


def rng(seed):
    return np.random.default_rng(seed)


def unit_rows(x):
    return x / np.linalg.norm(x, axis=-1, keepdims=True)


def sigmoid(x):
    return 1 / (1 + np.exp(-x))


def _case(seed, B=1, H=2, T=24, D=8):
    g = rng(seed)
    q = g.standard_normal((B, H, T, D))
    k = unit_rows(g.standard_normal((B, H, T, D)))
    v = g.standard_normal((B, H, T, D))
    beta = sigmoid(g.normal(1.5, 1.0, (B, H, T)))
    gate = sigmoid(g.normal(0.0, 1.5, (B, H, T)))
    return q, k, v, beta, gate


def _weighted_ridge(q, k, v, beta, gate, a):
    """o*_t = S_t q_t with S_t = argmin_S sum_i eta_{t,i} g_i ||S k_i - v_i||^2
    + lambda_t ||S||_F^2, eta_{t,i} = prod_{j=i+1..t} beta_j, lambda_t = a ||H_t||_F,
    H_t = sum_i eta_{t,i} g_i k_i k_i^T; stacked least squares (numpy lstsq)."""
    T, D = q.shape
    out = np.zeros((T, D))
    norms = np.zeros(T)
    for t in range(T):
        wt = np.array([np.prod(beta[i + 1:t + 1]) * gate[i] for i in range(t + 1)])
        Hdef = sum(wt[i] * np.outer(k[i], k[i]) for i in range(t + 1))
        norms[t] = np.linalg.norm(Hdef, "fro")
        lam = a * norms[t]
        Arows = np.vstack([np.sqrt(wt)[:, None] * k[:t + 1], math.sqrt(lam) * np.eye(D)])
        rhs = np.vstack([np.sqrt(wt)[:, None] * v[:t + 1], np.zeros((D, D))])
        St, *_ = np.linalg.lstsq(Arows, rhs, rcond=None)
        out[t] = q[t] @ St
    return out, norms


@pytest.mark.parametrize("a,r,seed", [(0.5, 60, 0), (0.1, 160, 1)])
def test_gated_layer_equals_weighted_ridge_regression(a, r, seed):
    g = rng(seed)
    T, D = 14, 5
    q = g.standard_normal((T, D))
    k = unit_rows(g.standard_normal((T, D))) * g.uniform(0.5, 2.0, (T, 1))
    v = g.standard_normal((T, D))
    beta = sigmoid(g.normal(1.0, 1.5, T))
    gate = sigmoid(g.normal(0.0, 1.5, T))
    gate[3] = 0.0          # a token that writes nothing
    ref, ref_norms = _weighted_ridge(q, k, v, beta, gate, a)
    out = oracle.forward(q[None, None], k[None, None], v[None, None], beta[None, None], a, r,
                         gate=gate[None, None], want_norms=True)
    np.testing.assert_allclose(out["norms"][0, 0], ref_norms, rtol=1e-12)
    np.testing.assert_allclose(out["o"][0, 0], ref, rtol=1e-8, atol=1e-10)


def test_unit_gate_is_the_ungated_layer_bit_for_bit():
    q, k, v, beta, _ = _case(1)
    ones = np.ones(beta.shape)
    a, r = 0.5, 9
    f0 = oracle.forward(q, k, v, beta, a, r, want_norms=True, want_final_state=True)
    f1 = oracle.forward(q, k, v, beta, a, r, gate=ones, want_norms=True, want_final_state=True)
    for key in ("o", "norms", "final_state"):
        np.testing.assert_array_equal(f0[key], f1[key])
    np.testing.assert_array_equal(oracle.chunked_norms(k, beta, 8),
                                  oracle.chunked_norms(k, beta, 8, gate=ones))
    st = f0["final_state"]
    o0, s0 = oracle.decode_step(st, q[:, :, 0], k[:, :, 0], v[:, :, 0], beta[:, :, 0], a, r)
    o1, s1 = oracle.decode_step(st, q[:, :, 0], k[:, :, 0], v[:, :, 0], beta[:, :, 0], a, r,
                                gate=ones[:, :, 0])
    np.testing.assert_array_equal(o0, o1)
    np.testing.assert_array_equal(s0, s1)


@pytest.mark.parametrize("c", [0.37, 1e-3, 4.0])
def test_constant_gate_leaves_output_unchanged(c):
    # H, M and lambda all scale by c; the Chebyshev iterate by 1/c; o = M x does not move
    q, k, v, beta, _ = _case(2)
    a, r = 0.5, 12
    f0 = oracle.forward(q, k, v, beta, a, r, want_norms=True, want_final_state=True)
    fc = oracle.forward(q, k, v, beta, a, r, gate=np.full(beta.shape, c), want_norms=True,
                        want_final_state=True)
    np.testing.assert_allclose(fc["o"], f0["o"], rtol=1e-10, atol=1e-13)
    np.testing.assert_allclose(fc["norms"], c * f0["norms"], rtol=1e-12)
    np.testing.assert_allclose(fc["final_state"], c * f0["final_state"], rtol=1e-12, atol=1e-15)


@pytest.mark.parametrize("a,r", [(0.5, 10), (0.1, 30)])
def test_gate_equals_rescaled_keys_and_values(a, r):
    q, k, v, beta, gate = _case(3, B=2, H=2, T=40, D=8)
    gate[0, 1, 7] = 0.0
    gate[1, 0, 0] = 1.0
    s = np.sqrt(gate)[..., None]
    fg = oracle.forward(q, k, v, beta, a, r, gate=gate, want_norms=True, want_final_state=True)
    fs = oracle.forward(q, s * k, s * v, beta, a, r, want_norms=True, want_final_state=True)
    np.testing.assert_allclose(fg["norms"], fs["norms"], rtol=1e-12)
    np.testing.assert_allclose(fg["final_state"], fs["final_state"], rtol=1e-12, atol=1e-14)
    np.testing.assert_allclose(fg["o"], fs["o"], rtol=1e-9, atol=1e-12)


def test_zero_gate_with_unit_decay_keeps_the_state():
    q, k, v, beta, gate = _case(4, T=12)
    beta[:, :, 6] = 1.0
    gate[:, :, 6] = 0.0
    a, r = 0.5, 8
    s5 = oracle.forward(q[:, :, :6], k[:, :, :6], v[:, :, :6], beta[:, :, :6], a, r,
                        gate=gate[:, :, :6], want_final_state=True)["final_state"]
    s6 = oracle.forward(q[:, :, :7], k[:, :, :7], v[:, :, :7], beta[:, :, :7], a, r,
                        gate=gate[:, :, :7], want_final_state=True)["final_state"]
    np.testing.assert_array_equal(s6, s5)


@pytest.mark.parametrize("a,r", [(0.5, 10), (0.1, 7)])
def test_gated_first_token_closed_form(a, r):
    # one token: H = g k k^T, M = g v k^T; the gate cancels in o (see the constant-gate case)
    g = rng(50 + r)
    B, H, D = 2, 3, 16
    q = g.standard_normal((B, H, 1, D))
    k = g.standard_normal((B, H, 1, D))
    v = g.standard_normal((B, H, 1, D))
    beta = g.uniform(0, 1, (B, H, 1))
    gate = g.uniform(0.05, 1, (B, H, 1))
    o = oracle.forward(q, k, v, beta, a, r, gate=gate)["o"]
    rho = 1 / (1 + 2 * a)
    Tr = np.polynomial.chebyshev.chebval(1 / rho, [0.0] * r + [1.0])
    fac = 1 - (-1) ** r / Tr
    kk = (k * k).sum(-1, keepdims=True)
    kq = (k * q).sum(-1, keepdims=True)
    np.testing.assert_allclose(o, v * kq / ((1 + a) * kk) * fac, rtol=1e-11, atol=1e-14)


@pytest.mark.parametrize("C", [1, 4, 16])
def test_gated_chunked_norm_equals_tokenwise(C):
    _, k, _, beta, gate = _case(10 + C, T=64)
    beta[0, 1, 20] = 0.0
    gate[0, 0, 5] = 0.0
    ref = oracle.forward(k, k, k, beta, 0.5, 1, gate=gate, want_norms=True)["norms"]
    got = oracle.chunked_norms(k, beta, C, gate=gate)
    np.testing.assert_allclose(got, ref, rtol=1e-12)


def test_gated_decode_steps_continue_the_forward():
    q, k, v, beta, gate = _case(20, B=2, H=2, T=10)
    a, r = 0.5, 7
    ref = oracle.forward(q, k, v, beta, a, r, gate=gate)["o"]
    st = oracle.forward(q[:, :, :6], k[:, :, :6], v[:, :, :6], beta[:, :, :6], a, r,
                        gate=gate[:, :, :6], want_final_state=True)["final_state"]
    for t in range(6, 10):
        o, st = oracle.decode_step(st, q[:, :, t], k[:, :, t], v[:, :, t], beta[:, :, t], a, r,
                                   gate=gate[:, :, t])
        np.testing.assert_allclose(o, ref[:, :, t], rtol=1e-13, atol=1e-15)
