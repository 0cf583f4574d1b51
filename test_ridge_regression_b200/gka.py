"""Python binding of libgka.so: argument marshalling only.

Every step of the layer runs in the library's CUDA kernels; this module checks
tensor shapes, dtypes and devices, hands raw device pointers and the current
CUDA stream to the C ABI (include/gka.h) and raises on a non-zero status.
There is no fallback: if the library is missing or a call fails, it raises.
"""
from __future__ import annotations

import ctypes
from pathlib import Path

import torch

_PKG = Path(__file__).resolve().parent
LIB_PATH = _PKG / "libgka.so"

GKA_F32, GKA_BF16 = 0, 1
_DT = {torch.float32: GKA_F32, torch.bfloat16: GKA_BF16}


class GkaError(RuntimeError):
    def __init__(self, fn: str, status: int):
        self.status = status
        msg = _lib().gka_status_string(status).decode()
        if status == -5:
            msg += f" (cudaError {_lib().gka_last_cuda_error()})"
        super().__init__(f"{fn}: {msg} [{status}]")


KERNEL_NAMES = ["chunk_delta", "state_scan", "chunk_norm", "chunk_solve", "decode_step",
                "chunk_solve_tc", "state_pass_tc", "bwd_solve", "bwd_delta", "adjoint_scan",
                "bwd_rows", "bwd_grads", "solver_study"]
_KERNEL_COUNT = 16


class KernelTimes(ctypes.Structure):
    _fields_ = [("ms", ctypes.c_double * _KERNEL_COUNT), ("launches", ctypes.c_int * _KERNEL_COUNT)]


class WorkspaceLayout(ctypes.Structure):
    _fields_ = [("states_offset", ctypes.c_size_t), ("decay_offset", ctypes.c_size_t),
                ("norms_offset", ctypes.c_size_t), ("states_lp_offset", ctypes.c_size_t),
                ("total_bytes", ctypes.c_size_t)]


_L = None


def _lib():
    global _L
    if _L is None:
        if not LIB_PATH.exists():
            raise ImportError(f"{LIB_PATH} is missing: build it with "
                              "`python -m test_ridge_regression_b200.build`")
        lib = ctypes.CDLL(str(LIB_PATH))
        vp, i, f, sz = ctypes.c_void_p, ctypes.c_int, ctypes.c_float, ctypes.c_size_t
        lib.gka_forward_workspace_bytes.argtypes = [i, i, i, i, i, i]
        lib.gka_forward_workspace_bytes.restype = sz
        lib.gka_forward_workspace_layout.argtypes = [i, i, i, i, i, i, ctypes.POINTER(WorkspaceLayout)]
        lib.gka_forward_workspace_layout.restype = i
        lib.gka_forward.argtypes = [vp, vp, vp, vp, vp, i, i, i, i, i, f, i, i, vp, vp, sz, vp]
        lib.gka_forward.restype = i
        lib.gka_forward_gated.argtypes = [vp, vp, vp, vp, vp, vp, i, i, i, i, i, f, i, i, vp, vp,
                                          sz, vp]
        lib.gka_forward_gated.restype = i
        lib.gka_forward_static_scratch.argtypes = [vp, vp, vp, vp, vp, i, i, i, i, i, f, i, i,
                                                   vp, vp]
        lib.gka_forward_host_workspace_bytes.argtypes = [i, i, i, i, i, i, i]
        lib.gka_forward_host_workspace_bytes.restype = sz
        lib.gka_forward_host.argtypes = [vp, vp, vp, vp, vp, i, i, i, i, i, f, i, i, vp, i, vp,
                                         sz, vp]
        lib.gka_forward_host.restype = i
        lib.gka_forward_static_scratch.restype = i
        lib.gka_decode_step.argtypes = [vp, vp, vp, vp, vp, vp, i, i, i, i, f, i, vp]
        lib.gka_decode_step.restype = i
        lib.gka_decode_step_gated.argtypes = [vp, vp, vp, vp, vp, vp, vp, i, i, i, i, f, i, vp]
        lib.gka_decode_step_gated.restype = i
        lib.gka_backward_workspace_bytes.argtypes = [i, i, i, i, i, i]
        lib.gka_backward_workspace_bytes.restype = sz
        lib.gka_backward.argtypes = [vp] * 11 + [i, i, i, i, i, f, i, i, vp, sz, vp]
        lib.gka_backward.restype = i
        lib.gka_solver_study_workspace_bytes.argtypes = [i, i, i, i, i, i]
        lib.gka_solver_study_workspace_bytes.restype = sz
        lib.gka_solver_study.argtypes = [vp, vp, vp, vp, i, i, i, i, i, f, i, i, i, vp, vp, sz, vp]
        lib.gka_solver_study.restype = i
        lib.gka_selftest_timeout.argtypes = [vp]
        lib.gka_selftest_timeout.restype = i
        lib.gka_device_status.argtypes = [vp]
        lib.gka_device_status.restype = i
        lib.gka_last_cuda_error.argtypes = []
        lib.gka_last_cuda_error.restype = i
        lib.gka_status_string.argtypes = [i]
        lib.gka_status_string.restype = ctypes.c_char_p
        lib.gka_version.argtypes = []
        lib.gka_version.restype = i
        lib.gka_profiler_enable.argtypes = [i]
        lib.gka_profiler_enable.restype = i
        lib.gka_profiler_read.argtypes = [ctypes.POINTER(KernelTimes)]
        lib.gka_profiler_read.restype = i
        _L = lib
    return _L


def lib():
    """The loaded ctypes library (raises ImportError if it was not built)."""
    return _lib()


def _ptr(t):
    return None if t is None else ctypes.c_void_p(t.data_ptr())


def _stream(stream):
    if stream is None:
        stream = torch.cuda.current_stream()
    return ctypes.c_void_p(stream.cuda_stream)


def _check(fn, rc):
    if rc != 0:
        raise GkaError(fn, rc)


def _dtype(t: torch.Tensor) -> int:
    if t.dtype not in _DT:
        raise TypeError(f"unsupported dtype {t.dtype}; use float32 or bfloat16")
    return _DT[t.dtype]


def _dev(*ts):
    for t in ts:
        if t is not None and (not t.is_cuda or not t.is_contiguous()):
            raise ValueError("tensors must be contiguous CUDA tensors")


def workspace_bytes(B, H, T, D, chunk, dtype=torch.bfloat16) -> int:
    return int(_lib().gka_forward_workspace_bytes(B, H, T, D, chunk, _DT[dtype]))


def workspace_layout(B, H, T, D, chunk, dtype=torch.bfloat16) -> WorkspaceLayout:
    out = WorkspaceLayout()
    _check("gka_forward_workspace_layout",
           _lib().gka_forward_workspace_layout(B, H, T, D, chunk, _DT[dtype], ctypes.byref(out)))
    return out


def alloc_workspace(B, H, T, D, chunk, dtype=torch.bfloat16, device=None) -> torch.Tensor:
    n = workspace_bytes(B, H, T, D, chunk, dtype)
    return torch.empty(max(n, 256), dtype=torch.uint8, device=device or "cuda")


def gka_forward(q, k, v, beta, a: float, r: int, chunk: int, *, o=None, final_state=None,
                workspace=None, stream=None):
    """Chunk-wise GKA forward (see include/gka.h).  q, k, v: [B, H, T, D] fp32 or
    bf16 CUDA tensors; beta: [B, H, T] fp32.  Returns o (same shape/dtype as v)."""
    _dev(q, k, v, beta, o, final_state, workspace)
    B, H, T, D = q.shape
    if k.shape != q.shape or v.shape != q.shape or beta.shape != (B, H, T):
        raise ValueError("shape mismatch")
    dt = _dtype(q)
    if k.dtype != q.dtype or v.dtype != q.dtype or beta.dtype != torch.float32:
        raise TypeError("q, k, v must share a dtype; beta must be float32")
    if o is None:
        o = torch.empty_like(v)
    if final_state is not None and (final_state.dtype != torch.float32 or
                                    final_state.shape != (B, H, 2, D, D)):
        raise ValueError("final_state must be float32 [B, H, 2, D, D]")
    if workspace is None:
        workspace = alloc_workspace(B, H, T, D, chunk, q.dtype, q.device)
    rc = _lib().gka_forward(_ptr(q), _ptr(k), _ptr(v), _ptr(beta), _ptr(o), B, H, T, D, dt,
                            float(a), int(r), int(chunk), _ptr(final_state), _ptr(workspace),
                            workspace.numel() * workspace.element_size(), _stream(stream))
    _check("gka_forward", rc)
    return o


def gka_forward_gated(q, k, v, beta, gate, a: float, r: int, chunk: int, *, o=None,
                      final_state=None, workspace=None, stream=None):
    """Write-gated forward (see include/gka.h): as gka_forward, with gate [B, H, T]
    fp32 in [0, 1] scaling each token's write into H and M (None: no gate)."""
    _dev(q, k, v, beta, gate, o, final_state, workspace)
    B, H, T, D = q.shape
    if k.shape != q.shape or v.shape != q.shape or beta.shape != (B, H, T):
        raise ValueError("shape mismatch")
    if gate is not None and (gate.shape != (B, H, T) or gate.dtype != torch.float32):
        raise ValueError("gate must be float32 [B, H, T]")
    dt = _dtype(q)
    if k.dtype != q.dtype or v.dtype != q.dtype or beta.dtype != torch.float32:
        raise TypeError("q, k, v must share a dtype; beta must be float32")
    if o is None:
        o = torch.empty_like(v)
    if final_state is not None and (final_state.dtype != torch.float32 or
                                    final_state.shape != (B, H, 2, D, D)):
        raise ValueError("final_state must be float32 [B, H, 2, D, D]")
    if workspace is None:
        workspace = alloc_workspace(B, H, T, D, chunk, q.dtype, q.device)
    rc = _lib().gka_forward_gated(_ptr(q), _ptr(k), _ptr(v), _ptr(beta), _ptr(gate), _ptr(o),
                                  B, H, T, D, dt, float(a), int(r), int(chunk), _ptr(final_state),
                                  _ptr(workspace), workspace.numel() * workspace.element_size(),
                                  _stream(stream))
    _check("gka_forward_gated", rc)
    return o


def host_workspace_bytes(B, H, T, D, chunk, dtype=torch.bfloat16, slice_pairs=0) -> int:
    return int(_lib().gka_forward_host_workspace_bytes(B, H, T, D, chunk, _DT[dtype], slice_pairs))


def alloc_host_workspace(B, H, T, D, chunk, dtype=torch.bfloat16, slice_pairs=0,
                         device=None) -> torch.Tensor:
    n = host_workspace_bytes(B, H, T, D, chunk, dtype, slice_pairs)
    return torch.empty(max(n, 256), dtype=torch.uint8, device=device or "cuda")


def gka_forward_host(q, k, v, beta, a: float, r: int, chunk: int, *, o=None, final_state=None,
                     slice_pairs=0, workspace=None, stream=None):
    """gka_forward from HOST tensors with the copies overlapped with the compute
    (see include/gka.h).  q, k, v: [B, H, T, D] fp32 or bf16 CPU tensors (pinned
    for overlap), beta: [B, H, T] fp32.  Returns o on the host; it is complete
    once `stream` (default: the current CUDA stream) has completed."""
    for t in (q, k, v, beta, o, final_state):
        if t is not None and (t.is_cuda or not t.is_contiguous()):
            raise ValueError("tensors must be contiguous host tensors")
    B, H, T, D = q.shape
    if k.shape != q.shape or v.shape != q.shape or beta.shape != (B, H, T):
        raise ValueError("shape mismatch")
    dt = _dtype(q)
    if k.dtype != q.dtype or v.dtype != q.dtype or beta.dtype != torch.float32:
        raise TypeError("q, k, v must share a dtype; beta must be float32")
    if o is None:
        o = torch.empty(q.shape, dtype=q.dtype, pin_memory=q.is_pinned())
    if final_state is not None and (final_state.dtype != torch.float32 or
                                    final_state.shape != (B, H, 2, D, D)):
        raise ValueError("final_state must be float32 [B, H, 2, D, D]")
    if workspace is None:
        workspace = alloc_host_workspace(B, H, T, D, chunk, q.dtype, slice_pairs)
    rc = _lib().gka_forward_host(_ptr(q), _ptr(k), _ptr(v), _ptr(beta), _ptr(o), B, H, T, D, dt,
                                 float(a), int(r), int(chunk), _ptr(final_state), int(slice_pairs),
                                 _ptr(workspace), workspace.numel() * workspace.element_size(),
                                 _stream(stream))
    _check("gka_forward_host", rc)
    return o


def gka_forward_static_scratch(q, k, v, beta, a: float, r: int, chunk: int, *, o=None,
                               final_state=None, stream=None):
    """gka_forward whose scratch is the library's own static device array
    (for callers that cannot allocate device memory; see include/gka.h).
    Calls that overlap on the GPU race on that array."""
    _dev(q, k, v, beta, o, final_state)
    B, H, T, D = q.shape
    if k.shape != q.shape or v.shape != q.shape or beta.shape != (B, H, T):
        raise ValueError("shape mismatch")
    dt = _dtype(q)
    if k.dtype != q.dtype or v.dtype != q.dtype or beta.dtype != torch.float32:
        raise TypeError("q, k, v must share a dtype; beta must be float32")
    if o is None:
        o = torch.empty_like(v)
    rc = _lib().gka_forward_static_scratch(_ptr(q), _ptr(k), _ptr(v), _ptr(beta), _ptr(o), B, H,
                                           T, D, dt, float(a), int(r), int(chunk),
                                           _ptr(final_state), _stream(stream))
    _check("gka_forward_static_scratch", rc)
    return o


def gka_decode_step(state, q, k, v, beta, a: float, r: int, *, o=None, stream=None):
    """One recurrent step in place on state [B, H, 2, D, D] fp32; q, k, v: [B, H, D];
    beta: [B, H] fp32.  Returns o [B, H, D]."""
    _dev(state, q, k, v, beta, o)
    B, H, D = q.shape
    if state.dtype != torch.float32 or state.shape != (B, H, 2, D, D):
        raise ValueError("state must be float32 [B, H, 2, D, D]")
    if k.shape != q.shape or v.shape != q.shape or beta.shape != (B, H):
        raise ValueError("shape mismatch")
    dt = _dtype(q)
    if o is None:
        o = torch.empty_like(v)
    rc = _lib().gka_decode_step(_ptr(state), _ptr(q), _ptr(k), _ptr(v), _ptr(beta), _ptr(o),
                                B, H, D, dt, float(a), int(r), _stream(stream))
    _check("gka_decode_step", rc)
    return o


def gka_decode_step_gated(state, q, k, v, beta, gate, a: float, r: int, *, o=None,
                          stream=None):
    """Write-gated decode step in place on state [B, H, 2, D, D] fp32; gate [B, H]
    fp32 in [0, 1] (None: no gate).  Returns o [B, H, D]."""
    _dev(state, q, k, v, beta, gate, o)
    B, H, D = q.shape
    if state.dtype != torch.float32 or state.shape != (B, H, 2, D, D):
        raise ValueError("state must be float32 [B, H, 2, D, D]")
    if k.shape != q.shape or v.shape != q.shape or beta.shape != (B, H):
        raise ValueError("shape mismatch")
    if gate is not None and (gate.shape != (B, H) or gate.dtype != torch.float32):
        raise ValueError("gate must be float32 [B, H]")
    dt = _dtype(q)
    if o is None:
        o = torch.empty_like(v)
    rc = _lib().gka_decode_step_gated(_ptr(state), _ptr(q), _ptr(k), _ptr(v), _ptr(beta),
                                      _ptr(gate), _ptr(o), B, H, D, dt, float(a), int(r),
                                      _stream(stream))
    _check("gka_decode_step_gated", rc)
    return o


def backward_workspace_bytes(B, H, T, D, chunk, dtype=torch.bfloat16) -> int:
    return int(_lib().gka_backward_workspace_bytes(B, H, T, D, chunk, _DT[dtype]))


def gka_backward(q, k, v, beta, dout, a: float, r: int, chunk: int = 32, *, gate=None,
                 workspace=None, stream=None):
    """Implicit-differentiation backward (see include/gka.h).  q, k, v, dout:
    [B, H, T, D] fp32 or bf16 CUDA tensors; beta (and the optional gate):
    [B, H, T] fp32.  Returns a dict with dq, dk, dv (dtype of q), dbeta and, with a
    gate, dgate (fp32)."""
    _dev(q, k, v, beta, gate, dout, workspace)
    B, H, T, D = q.shape
    if any(t.shape != q.shape for t in (k, v, dout)) or beta.shape != (B, H, T):
        raise ValueError("shape mismatch")
    if gate is not None and (gate.shape != (B, H, T) or gate.dtype != torch.float32):
        raise ValueError("gate must be float32 [B, H, T]")
    dt = _dtype(q)
    if any(t.dtype != q.dtype for t in (k, v, dout)) or beta.dtype != torch.float32:
        raise TypeError("q, k, v, dout must share a dtype; beta must be float32")
    out = {n: torch.empty_like(q) for n in ("dq", "dk", "dv")}
    out["dbeta"] = torch.empty_like(beta)
    if gate is not None:
        out["dgate"] = torch.empty_like(gate)
    if workspace is None:
        n = backward_workspace_bytes(B, H, T, D, chunk, q.dtype)
        workspace = torch.empty(max(n, 256), dtype=torch.uint8, device=q.device)
    rc = _lib().gka_backward(_ptr(q), _ptr(k), _ptr(v), _ptr(beta), _ptr(gate), _ptr(dout),
                             _ptr(out["dq"]), _ptr(out["dk"]), _ptr(out["dv"]), _ptr(out["dbeta"]),
                             _ptr(out.get("dgate")), B, H, T, D, dt, float(a), int(r), int(chunk),
                             _ptr(workspace), workspace.numel() * workspace.element_size(),
                             _stream(stream))
    _check("gka_backward", rc)
    return out


SOLVERS = ("chebyshev", "gd", "agd", "cg")


def gka_solver_study(q, k, beta, a: float, r: int, solver: str, chunk: int = 64, *, gate=None,
                     workspace=None, stream=None):
    """Residual history ||q_t - A_t x_i|| / ||q_t||, i = 0..r, of ``solver`` (one of
    SOLVERS) on every token's system (see include/gka.h).  Returns [B, H, T, r + 1] fp32."""
    _dev(q, k, beta, gate, workspace)
    B, H, T, D = q.shape
    if k.shape != q.shape or beta.shape != (B, H, T):
        raise ValueError("shape mismatch")
    if gate is not None and (gate.shape != (B, H, T) or gate.dtype != torch.float32):
        raise ValueError("gate must be float32 [B, H, T]")
    dt = _dtype(q)
    if k.dtype != q.dtype or beta.dtype != torch.float32:
        raise TypeError("q, k must share a dtype; beta must be float32")
    resid = torch.empty(B, H, T, r + 1, dtype=torch.float32, device=q.device)
    if workspace is None:
        n = int(_lib().gka_solver_study_workspace_bytes(B, H, T, D, chunk, dt))
        workspace = torch.empty(max(n, 256), dtype=torch.uint8, device=q.device)
    rc = _lib().gka_solver_study(_ptr(q), _ptr(k), _ptr(beta), _ptr(gate), B, H, T, D, dt,
                                 float(a), int(r), int(chunk), SOLVERS.index(solver), _ptr(resid),
                                 _ptr(workspace), workspace.numel() * workspace.element_size(),
                                 _stream(stream))
    _check("gka_solver_study", rc)
    return resid


def selftest_timeout(stream=None) -> None:
    """Launch the bounded-wait self-test (see include/gka.h)."""
    _check("gka_selftest_timeout", _lib().gka_selftest_timeout(_stream(stream)))


def device_status(stream=None) -> int:
    """Synchronises the stream and returns the library's device status code."""
    return int(_lib().gka_device_status(_stream(stream)))


def profiler_enable(on: bool = True) -> None:
    """Bracket every library kernel launch with CUDA events on its stream."""
    _check("gka_profiler_enable", _lib().gka_profiler_enable(1 if on else 0))


def profiler_read() -> dict:
    """Per-kernel {name: (total_ms, launches)} since the last read (waits on the events)."""
    out = KernelTimes()
    _check("gka_profiler_read", _lib().gka_profiler_read(ctypes.byref(out)))
    return {name: (out.ms[i], out.launches[i]) for i, name in enumerate(KERNEL_NAMES)
            if out.launches[i]}
