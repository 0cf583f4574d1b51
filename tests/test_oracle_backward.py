"""Pins of the oracle's backward pass (implicit differentiation; ai.info page,
Key Contributions 3, Main Findings (Lemma 2: dq_t = dq^_t) and Methodology;
pith.science appendix, Eq. 50) against PyTorch float64 autograd, which is
independent of the oracle's code:

  * with the Chebyshev iteration converged (r large), implicit differentiation
    is the exact gradient of the layer with an exact solve: autograd through
    torch.linalg.solve of (H_t + a ||H_t||_F I) x = q_t, o_t = M_t x_t, token by
    token, gives the same dq, dk, dv, dbeta and write-gate gradient;
  * Lemma 2 for any r: the r-step iterate is x_r = P_r(A) q with P_r(A)
    symmetric, so dq equals autograd through the r-step iteration itself;
  * as r grows, the implicit gradients and autograd through the iteration
    approach each other (both tend to the exact gradient).
"""
import numpy as np
import pytest
import torch

import oracle


def rng(seed):
    return np.random.default_rng(seed)


def _inputs(seed, B=1, H=2, T=9, D=5, gate=False):
    g = rng(seed)
    q = g.standard_normal((B, H, T, D))
    k = g.standard_normal((B, H, T, D))
    k /= np.linalg.norm(k, axis=-1, keepdims=True)
    k *= g.uniform(0.6, 1.6, (B, H, T, 1))
    v = g.standard_normal((B, H, T, D))
    beta = 1 / (1 + np.exp(-g.normal(1.0, 1.5, (B, H, T))))
    dout = g.standard_normal((B, H, T, D))
    gt = g.uniform(0.05, 1.0, (B, H, T)) if gate else None
    return q, k, v, beta, dout, gt


def _torch_layer(q, k, v, beta, a, gate=None, solver=None):
    """Token-by-token layer in torch float64; solver(A, q) -> x (default: exact)."""
    B, H, T, D = q.shape
    Hs = torch.zeros(B, H, D, D, dtype=torch.float64)
    Ms = torch.zeros(B, H, D, D, dtype=torch.float64)
    eye = torch.eye(D, dtype=torch.float64)
    outs = []
    for t in range(T):
        g = 1.0 if gate is None else gate[:, :, t, None, None]
        kt, vt = k[:, :, t], v[:, :, t]
        Hs = beta[:, :, t, None, None] * Hs + g * kt[..., :, None] * kt[..., None, :]
        Ms = beta[:, :, t, None, None] * Ms + g * vt[..., :, None] * kt[..., None, :]
        n = torch.sqrt((Hs * Hs).sum(dim=(-2, -1)))
        A = Hs + a * n[..., None, None] * eye
        if solver is None:
            x = torch.linalg.solve(A, q[:, :, t, :, None])[..., 0]
        else:
            x = solver(A, q[:, :, t], n, a)
        outs.append((Ms @ x[..., None])[..., 0])
    return torch.stack(outs, dim=2)


def _cheb_torch(r):
    """r-step three-term Chebyshev iteration on [a n, (1+a) n] from x = 0, with the
    weights of the oracle's schedule (pinned in test_oracle_pins)."""
    def solve(A, q, n, a):
        mu, L = a * n, (1 + a) * n
        d = ((L + mu) / 2)[..., None]
        rho = 1.0 / (1.0 + 2.0 * a)
        om = oracle.omegas(rho, r)
        xp = torch.zeros_like(q)
        x = q / d
        for i in range(1, r):
            Ax = (A @ x[..., None])[..., 0]
            xn = xp + om[i] * ((q - Ax) / d + x - xp)
            xp, x = x, xn
        return x
    return solve


def _autograd(q, k, v, beta, dout, a, gate=None, solver=None):
    ts = [torch.tensor(x, dtype=torch.float64, requires_grad=True) for x in (q, k, v, beta)]
    gt = None if gate is None else torch.tensor(gate, dtype=torch.float64, requires_grad=True)
    o = _torch_layer(*ts, a, gate=gt, solver=solver)
    (o * torch.tensor(dout)).sum().backward()
    out = {n: t.grad.numpy() for n, t in zip(("dq", "dk", "dv", "dbeta"), ts)}
    if gt is not None:
        out["dgate"] = gt.grad.numpy()
    return out, o.detach().numpy()


@pytest.mark.parametrize("a,seed,gate", [(0.5, 0, False), (0.5, 1, True), (1.0, 2, False)])
def test_converged_backward_equals_exact_solve_autograd(a, seed, gate):
    q, k, v, beta, dout, gt = _inputs(seed, gate=gate)
    beta[0, 1, 4] = 0.0                       # a reset inside the sequence
    ref, o_exact = _autograd(q, k, v, beta, dout, a, gate=gt)
    r = 60                                    # R_a^r below 1e-30 for a >= 0.5
    got = oracle.backward(q, k, v, beta, dout, a, r, gate=gt)
    np.testing.assert_allclose(oracle.forward(q, k, v, beta, a, r, gate=gt)["o"], o_exact,
                               rtol=1e-10, atol=1e-12)
    for name in ref:
        scale = np.abs(ref[name]).max()
        np.testing.assert_allclose(got[name], ref[name], rtol=1e-8, atol=1e-10 * scale,
                                   err_msg=name)


@pytest.mark.parametrize("r", [1, 2, 3, 7])
def test_lemma2_dq_equals_autograd_through_the_iteration(r):
    q, k, v, beta, dout, _ = _inputs(10 + r)
    a = 0.5
    ref, o_cheb = _autograd(q, k, v, beta, dout, a, solver=_cheb_torch(r))
    # the torch iteration is the oracle's forward
    np.testing.assert_allclose(oracle.forward(q, k, v, beta, a, r)["o"], o_cheb, rtol=1e-11,
                               atol=1e-13)
    got = oracle.backward(q, k, v, beta, dout, a, r)
    np.testing.assert_allclose(got["dq"], ref["dq"], rtol=1e-10, atol=1e-12)


def test_implicit_and_iteration_autograd_meet_as_r_grows():
    q, k, v, beta, dout, gt = _inputs(30, gate=True)
    a = 0.5
    diffs = []
    for r in (4, 8, 16):
        ref, _ = _autograd(q, k, v, beta, dout, a, gate=gt, solver=_cheb_torch(r))
        got = oracle.backward(q, k, v, beta, dout, a, r, gate=gt)
        diffs.append(max(np.abs(got[n] - ref[n]).max() / np.abs(ref[n]).max()
                         for n in ("dk", "dv", "dbeta", "dgate")))
    assert diffs[0] > diffs[1] > diffs[2] and diffs[2] < 1e-6, diffs


def test_zero_key_tokens_contribute_nothing():
    # a zero key at the start leaves H = 0: x = 0, o = 0, and no gradient through it
    q, k, v, beta, dout, _ = _inputs(40)
    k[:, :, 0] = 0.0
    got = oracle.backward(q, k, v, beta, dout, 0.5, 60)
    assert np.all(got["dq"][:, :, 0] == 0)
    ref, _ = _autograd(q[:, :, 1:], k[:, :, 1:], v[:, :, 1:], beta[:, :, 1:], dout[:, :, 1:], 0.5)
    np.testing.assert_allclose(got["dk"][:, :, 1:], ref["dk"], rtol=1e-8, atol=1e-12)
    np.testing.assert_allclose(got["dv"][:, :, 1:], ref["dv"], rtol=1e-8, atol=1e-12)
    # the state before token 1 is zero, so beta_1 gets no gradient
    assert np.all(got["dbeta"][:, :, 1] == 0)
