"""ctypes front end of the float64 oracle in ``gka_oracle.c``.

TEST INFRASTRUCTURE ONLY (tests, smoke check, CPU baseline).  Arrays are numpy
float64, C-contiguous.  Inputs of lower precision (bf16, fp32) are upcast
exactly by the caller before they reach these functions.

Source: "Gated KalmaNet: A Fading Memory Layer Through Test-Time Ridge
Regression" (arXiv 2511.21016); see the C file for the passages each routine
follows.
"""
from __future__ import annotations

import ctypes
import os
import subprocess
from pathlib import Path

import numpy as np

_HERE = Path(__file__).resolve().parent
_SRC = _HERE / "gka_oracle.c"
_LIB = _HERE / "libgka_oracle.so"
_lib = None

_dp = ctypes.POINTER(ctypes.c_double)


def build(force: bool = False) -> Path:
    """Compile the oracle with gcc (-O2, OpenMP, strict IEEE float64)."""
    if force or not _LIB.exists() or _LIB.stat().st_mtime < _SRC.stat().st_mtime:
        tmp = _LIB.with_suffix(f".so.{os.getpid()}.tmp")
        subprocess.check_call(
            ["gcc", "-O2", "-fopenmp", "-fPIC", "-shared", "-std=c11",
             "-fno-fast-math", "-ffp-contract=off",
             str(_SRC), "-o", str(tmp), "-lm"])
        os.replace(tmp, _LIB)
    return _LIB


def _load():
    global _lib
    if _lib is None:
        build()
        lib = ctypes.CDLL(str(_LIB))
        i, d = ctypes.c_int, ctypes.c_double
        lib.gka_oracle_omegas.argtypes = [d, i, _dp]
        lib.gka_oracle_omegas.restype = None
        lib.gka_oracle_cheb_solve.argtypes = [_dp, _dp, i, d, d, i, _dp, _dp]
        lib.gka_oracle_cheb_solve.restype = None
        lib.gka_oracle_forward.argtypes = [_dp, _dp, _dp, _dp, _dp, i, i, i, i, d, i,
                                           _dp, i, _dp, _dp, _dp, i, _dp, i]
        lib.gka_oracle_forward.restype = i
        lib.gka_oracle_decode_step.argtypes = [_dp, _dp, _dp, _dp, _dp, _dp, i, i, i,
                                               d, i, _dp, i]
        lib.gka_oracle_decode_step.restype = i
        lib.gka_oracle_chunked_norms.argtypes = [_dp, _dp, _dp, i, i, i, i, i, _dp, i]
        lib.gka_oracle_chunked_norms.restype = i
        lib.gka_oracle_backward.argtypes = [_dp, _dp, _dp, _dp, _dp, _dp, i, i, i, i, d, i,
                                            _dp, _dp, _dp, _dp, _dp, i]
        lib.gka_oracle_backward.restype = i
        lib.gka_oracle_solver_study.argtypes = [_dp, _dp, _dp, _dp, i, i, i, i, d, i, i, _dp, i]
        lib.gka_oracle_solver_study.restype = i
        lib.gka_oracle_solver_residuals.argtypes = [_dp, _dp, i, d, d, i, i, _dp]
        lib.gka_oracle_solver_residuals.restype = None
        lib.gka_oracle_max_threads.argtypes = []
        lib.gka_oracle_max_threads.restype = i
        _lib = lib
    return _lib


def _f64(x) -> np.ndarray:
    if hasattr(x, "detach"):  # torch tensor: exact upcast on the host
        x = x.detach().to("cpu").double().numpy()
    return np.ascontiguousarray(x, dtype=np.float64)


def _ptr(a):
    return None if a is None else a.ctypes.data_as(_dp)


def max_threads() -> int:
    return int(_load().gka_oracle_max_threads())


def omegas(rho: float, n: int) -> np.ndarray:
    """Chebyshev weights omega_0..omega_{n-1} (omega_0 = 2)."""
    out = np.zeros(max(n, 1), dtype=np.float64)
    _load().gka_oracle_omegas(float(rho), int(n), _ptr(out))
    return out[:n]


def cheb_solve(A, q, mu: float, L: float, r: int) -> np.ndarray:
    """r-step Chebyshev iterate for A x = q, spectrum of A in [mu, L], x_0 = 0."""
    A = _f64(A)
    q = _f64(q)
    D = q.shape[0]
    assert A.shape == (D, D)
    x = np.zeros(D)
    work = np.zeros(3 * D)
    _load().gka_oracle_cheb_solve(_ptr(A), _ptr(q), D, float(mu), float(L), int(r),
                                  _ptr(x), _ptr(work))
    return x


def _gate(gate, shape):
    if gate is None:
        return None
    g = _f64(gate)
    assert g.shape == shape, (g.shape, shape)
    return g


def forward(q, k, v, beta, a: float, r: int, *, gate=None, init_state=None,
            solve_from: int = 0, want_norms: bool = False, want_final_state: bool = False,
            chunk: int = 0, want_chunk_states: bool = False, nthreads: int = 0):
    """Token-by-token forward.  q, k, v: [B, H, T, D]; beta: [B, H, T];
    gate: optional write gate [B, H, T] (None: 1 for every token).

    Returns a dict with ``o`` [B,H,T,D] and, on request, ``norms`` [B,H,T],
    ``final_state`` [B,H,2,D,D] and ``chunk_states`` [B,H,T/chunk,2,D,D]
    (the state in force before each chunk's first token).
    """
    q, k, v, beta = _f64(q), _f64(k), _f64(v), _f64(beta)
    B, H, T, D = q.shape
    assert k.shape == q.shape and v.shape == q.shape and beta.shape == (B, H, T)
    o = np.zeros((B, H, T, D))
    norms = np.zeros((B, H, T)) if want_norms else None
    fs = np.zeros((B, H, 2, D, D)) if want_final_state else None
    cs = None
    if want_chunk_states:
        assert chunk > 0 and T % chunk == 0
        cs = np.zeros((B, H, T // chunk, 2, D, D))
    g = _gate(gate, (B, H, T))
    init = None if init_state is None else _f64(init_state)
    if init is not None:
        assert init.shape == (B, H, 2, D, D)
    rc = _load().gka_oracle_forward(_ptr(q), _ptr(k), _ptr(v), _ptr(beta), _ptr(g), B, H, T, D,
                                    float(a), int(r), _ptr(init), int(solve_from),
                                    _ptr(o), _ptr(norms), _ptr(fs), int(chunk), _ptr(cs),
                                    int(nthreads))
    if rc != 0:
        raise ValueError("gka_oracle_forward: bad arguments")
    out = {"o": o}
    if want_norms:
        out["norms"] = norms
    if want_final_state:
        out["final_state"] = fs
    if want_chunk_states:
        out["chunk_states"] = cs
    return out


def decode_step(state, q, k, v, beta, a: float, r: int, nthreads: int = 0, gate=None):
    """One recurrent step.  state [B,H,2,D,D] (returned updated, new array);
    q, k, v: [B,H,D]; beta [B,H]; gate: optional write gate [B,H].
    Returns (o [B,H,D], state)."""
    st = _f64(state).copy()
    q, k, v, beta = _f64(q), _f64(k), _f64(v), _f64(beta)
    B, H, D = q.shape
    assert st.shape == (B, H, 2, D, D) and beta.shape == (B, H)
    o = np.zeros((B, H, D))
    g = _gate(gate, (B, H))
    rc = _load().gka_oracle_decode_step(_ptr(st), _ptr(q), _ptr(k), _ptr(v), _ptr(beta),
                                        _ptr(g), B, H, D, float(a), int(r), _ptr(o), int(nthreads))
    if rc != 0:
        raise ValueError("gka_oracle_decode_step: bad arguments")
    return o, st


def chunked_norms(k, beta, chunk: int, nthreads: int = 0, gate=None) -> np.ndarray:
    """||H_t||_F by the chunk-wise closed form.  k [B,H,T,D], beta [B,H,T],
    gate: optional write gate [B,H,T]."""
    k, beta = _f64(k), _f64(beta)
    B, H, T, D = k.shape
    g = _gate(gate, (B, H, T))
    out = np.zeros((B, H, T))
    rc = _load().gka_oracle_chunked_norms(_ptr(k), _ptr(beta), _ptr(g), B, H, T, D, int(chunk),
                                          _ptr(out), int(nthreads))
    if rc != 0:
        raise ValueError("gka_oracle_chunked_norms: bad arguments")
    return out


def backward(q, k, v, beta, dout, a: float, r: int, *, gate=None, nthreads: int = 0):
    """Implicit-differentiation backward of the layer (see the C file).  q, k, v,
    dout: [B, H, T, D]; beta (and the optional gate): [B, H, T].  Returns a dict
    with dq, dk, dv [B, H, T, D], dbeta [B, H, T] and, with a gate, dgate [B, H, T]."""
    q, k, v, beta, dout = _f64(q), _f64(k), _f64(v), _f64(beta), _f64(dout)
    B, H, T, D = q.shape
    assert k.shape == q.shape and v.shape == q.shape and dout.shape == q.shape
    assert beta.shape == (B, H, T)
    g = _gate(gate, (B, H, T))
    out = {n: np.zeros((B, H, T, D)) for n in ("dq", "dk", "dv")}
    out["dbeta"] = np.zeros((B, H, T))
    dg = np.zeros((B, H, T)) if g is not None else None
    rc = _load().gka_oracle_backward(_ptr(q), _ptr(k), _ptr(v), _ptr(beta), _ptr(g), _ptr(dout),
                                     B, H, T, D, float(a), int(r), _ptr(out["dq"]),
                                     _ptr(out["dk"]), _ptr(out["dv"]), _ptr(out["dbeta"]),
                                     _ptr(dg), int(nthreads))
    if rc != 0:
        raise ValueError(f"gka_oracle_backward failed ({rc})")
    if dg is not None:
        out["dgate"] = dg
    return out


SOLVERS = ("chebyshev", "gd", "agd", "cg")


def solver_study(q, k, beta, a: float, r: int, solver: str, *, gate=None, nthreads: int = 0):
    """Relative residual ||q_t - A_t x_i|| / ||q_t||, i = 0..r, of ``solver`` (one of
    SOLVERS) on every token's system A_t x = q_t.  Returns [B, H, T, r + 1]."""
    q, k, beta = _f64(q), _f64(k), _f64(beta)
    B, H, T, D = q.shape
    g = _gate(gate, (B, H, T))
    out = np.zeros((B, H, T, r + 1))
    rc = _load().gka_oracle_solver_study(_ptr(q), _ptr(k), _ptr(beta), _ptr(g), B, H, T, D,
                                         float(a), int(r), SOLVERS.index(solver), _ptr(out),
                                         int(nthreads))
    if rc != 0:
        raise ValueError("gka_oracle_solver_study: bad arguments")
    return out


def solver_residuals(A, q, mu: float, L: float, r: int, solver: str) -> np.ndarray:
    """Residual history ||q - A x_i|| / ||q||, i = 0..r, of ``solver`` on A x = q."""
    A, q = _f64(A), _f64(q)
    D = q.shape[0]
    assert A.shape == (D, D)
    out = np.zeros(r + 1)
    _load().gka_oracle_solver_residuals(_ptr(A), _ptr(q), D, float(mu), float(L), int(r),
                                        SOLVERS.index(solver), _ptr(out))
    return out
