"""Host-side checks (CPU, float64) of three reformulations the tensor-core backward uses,
each against the sequential recurrence it replaces, on random inputs.

1. dbeta's prefix sums over a chunk as 32 x 32 matrix products (the gradient kernel)
   against the per-column recurrences of the CUDA-core gradient kernel.
2. The adjoint pass's e_i = sum_{s>=i} b_s c_s w_si by a lane-parallel suffix scan of the
   linear recurrence e_i = b_i c_i + w_{i+1,i} e_{i+1}.
3. Per-token decays relative to groups of two chunks, built chunk by chunk from a running
   offset (the state pass at 32-token chunks feeding a solve at 64), against the prefix
   over each group directly.
"""
import numpy as np

C = 32


def _decays(rng, C=C):
    ell = np.cumsum(np.log(rng.uniform(0.6, 1.0, C)))       # chunk-relative cumulative logs
    W = np.zeros((C, C))                                    # W[l][s] = w_sl, s >= l
    for l in range(C):
        for s in range(l, C):
            W[l, s] = np.exp(ell[s] - ell[l])
    step = np.exp(np.diff(np.concatenate([[0.0], ell])))    # beta_t within the chunk
    return ell, W, step


def test_dbeta_matrix_form_matches_recurrences():
    rng = np.random.default_rng(5)
    ell, W, step = _decays(rng)
    w = rng.uniform(0.2, 1.0, C)                 # write gates
    KX, KY, VG, GK = (rng.standard_normal((C, C)) for _ in range(4))
    GK = (GK + GK.T) / 2                         # k_l . k_i is symmetric
    c, b = rng.standard_normal(C), np.exp(ell)
    uk, yhx, gmx, qe_tok, X1 = (rng.standard_normal(C) for _ in range(5))
    bm1 = np.concatenate([[1.0], np.exp(ell[:-1])])
    wend = np.exp(ell[-1] - ell)
    hs2, eh = 1.7, -0.4

    # recurrences (lane s over j <= s; lane i over s; lane j for the sums)
    Q = np.zeros((C, C))
    for i in range(C):
        qv = 0.0
        for s in range(C):
            qv = (0.0 if s == 0 else step[s]) * qv + w[s] * w[i] * GK[s, i] ** 2
            Q[i, s] = qv
    PH = np.zeros((C, C))
    for s in range(C):
        t1 = t2 = t3 = u1 = 0.0
        for j in range(s + 1):
            if j > 0:
                i = j - 1
                t1 = step[i] * t1 + w[i] * KY[i, s] * KX[i, s]
                t3 = step[i] * t3 + w[i] * VG[i, s] * KX[i, s]
                t2 = step[i] * t2 + Q[i, s]
                u1 = step[i] * u1 + w[i] * uk[i]
            bm = bm1[j]
            phi = (-(bm * yhx[s] + t1) - c[s] * (b[s] * bm * hs2 + b[s] * u1 + bm * X1[s] + t2)
                   + (bm * gmx[s] + t3))
            PH[j, s] = W[j, s] * phi
    ref = np.zeros(C)
    for j in range(C):
        qe = 0.0
        for i in range(j):
            qe = step[i] * qe + w[i] * qe_tok[i]
        ref[j] = PH[j, j:].sum() + wend[j] * (bm1[j] * eh + qe)

    # matrix form: L[j][i] = w_{j-1,i} for i < j
    L = np.zeros((C, C))
    for j in range(1, C):
        L[j, :] = W[:, j - 1]
    Qm = ((w[:, None] * GK ** 2) * w[None, :]).T @ W
    T1 = L @ (w[:, None] * KY * KX)
    T2 = L @ Qm
    T3 = L @ (w[:, None] * VG * KX)
    U1, QE = L @ (w * uk), L @ (w * qe_tok)
    phi = (-(bm1[:, None] * yhx[None, :] + T1)
           - c[None, :] * (b[None, :] * bm1[:, None] * hs2 + b[None, :] * U1[:, None]
                           + bm1[:, None] * X1[None, :] + T2)
           + (bm1[:, None] * gmx[None, :] + T3))
    got = (W * phi).sum(axis=1) + wend * (bm1 * eh + QE)
    assert np.allclose(Qm, Q, rtol=1e-12, atol=1e-12)
    assert np.allclose(got, ref, rtol=1e-11, atol=1e-11)


def test_adjoint_weights_suffix_scan():
    rng = np.random.default_rng(6)
    ell, W, step = _decays(rng)
    b, c = np.exp(ell), rng.standard_normal(C)
    # the definition and the sequential recurrence
    e_def = np.array([sum(b[s] * c[s] * W[i, s] for s in range(i, C)) for i in range(C)])
    e_seq = np.zeros(C)
    acc = 0.0
    for i in range(C - 1, -1, -1):
        acc = b[i] * c[i] + (step[i + 1] * acc if i + 1 < C else 0.0)
        e_seq[i] = acc
    # lane-parallel: (A, B) = (w_{t+1,t}, b_t c_t) composed with the lane o steps down
    A = np.array([step[t + 1] if t + 1 < C else 0.0 for t in range(C)])
    B = b * c
    o = 1
    while o < C:
        A2 = np.array([A[t + o] if t + o < C else 0.0 for t in range(C)])
        B2 = np.array([B[t + o] if t + o < C else 0.0 for t in range(C)])
        live = np.arange(C) + o < C
        B = np.where(live, A * B2 + B, B)
        A = np.where(live, A * A2, A)
        o *= 2
    assert np.allclose(e_seq, e_def, rtol=1e-12, atol=1e-13)
    assert np.allclose(B, e_def, rtol=1e-12, atol=1e-13)


def test_group_relative_decays_from_running_offset():
    rng = np.random.default_rng(7)
    Cs, tdc, nchunks = 32, 2, 8
    logb = np.maximum(np.log(rng.uniform(0.3, 1.0, Cs * nchunks)), -150.0)
    # per chunk: the chunk-relative prefix plus the group offset, reset every tdc chunks
    got = np.zeros_like(logb)
    goff = 0.0
    for n in range(nchunks):
        seg = logb[n * Cs:(n + 1) * Cs]
        got[n * Cs:(n + 1) * Cs] = np.cumsum(seg) + goff
        goff = 0.0 if (n + 1) % tdc == 0 else goff + seg.sum()
    # directly: the prefix over each group of tdc chunks
    G = Cs * tdc
    ref = np.concatenate([np.cumsum(logb[g:g + G]) for g in range(0, len(logb), G)])
    assert np.allclose(got, ref, rtol=1e-13, atol=1e-12)
