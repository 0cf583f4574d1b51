"""gka_forward_static_scratch: the forward for callers that cannot allocate
device memory (a plugin inside a host application that owns all device
allocations, or a latency-critical caller that cannot take cudaMalloc's
implicit synchronisation).  Its scratch is the library's own static device
array, so the tests check, through the C ABI, that calls in a row (each one
finding the previous call's leftovers in that array, at the same or at other
offsets) give bit for bit the results of gka_forward with a caller workspace:
both run the same deterministic kernels (no atomics, no reduction order that
depends on the launch), so any difference is a scratch fault.  A problem too
large for the array is refused before anything runs.

This file is collected last on purpose (its name sorts last)."""
import ctypes

import pytest
import torch

from helpers import TOL, head_rel_err
from test_ridge_regression_b200 import build, gka
from test_ridge_regression_b200.inputs import make_inputs

pytestmark = pytest.mark.gpu


def _call(lib, q, k, v, beta, o, a, r, chunk, fs):
    B, H, T, D = q.shape
    dt = 1 if q.dtype == torch.bfloat16 else 0
    p = lambda t: ctypes.c_void_p(t.data_ptr())
    stream = ctypes.c_void_p(torch.cuda.current_stream().cuda_stream)
    return lib.gka_forward_static_scratch(p(q), p(k), p(v), p(beta), p(o), B, H, T, D, dt,
                                          float(a), int(r), int(chunk), p(fs), stream)


def _check_against_gka_forward(lib, B, H, T, D, dtype, chunk, r, a, seed):
    q, k, v, beta = (x.cuda() for x in make_inputs(B, H, T, D, dtype, 3.0, 1.0, seed))
    fs_ref = torch.empty(B, H, 2, D, D, device="cuda")
    ref = gka.gka_forward(q, k, v, beta, a, r, chunk, final_state=fs_ref)
    o = torch.full_like(ref, float("nan"))
    fs = torch.full_like(fs_ref, float("nan"))
    rc = _call(lib, q, k, v, beta, o, a, r, chunk, fs)
    assert rc == 0, lib.gka_status_string(rc)
    assert gka.device_status() == 0
    # same kernels, same inputs: identical bits (a tolerance would hide a scratch fault)
    assert torch.equal(o, ref), f"max |diff| {(o.float() - ref.float()).abs().max().item():.3e}"
    assert torch.equal(fs, fs_ref)
    # and both still agree with the layer within the bf16 / fp32 parity bar
    assert head_rel_err(o, ref) <= TOL[dtype]


@pytest.mark.parametrize("dtype,D,chunk,r", [(torch.bfloat16, 128, 64, 20),
                                             (torch.float32, 64, 32, 10)])
def test_static_scratch_matches_gka_forward_twice(dtype, D, chunk, r):
    build.build()
    lib = gka.lib()
    B, H, T, a = 1, 4, 512, 0.5
    assert gka.workspace_bytes(B, H, T, D, chunk, dtype) <= 64 << 20
    for seed in (21, 22):
        _check_against_gka_forward(lib, B, H, T, D, dtype, chunk, r, a, seed)


def test_static_scratch_both_state_paths_after_other_shapes():
    """40 heads take the one-pass state kernel over whole sequences, 24 heads and
    8 heads the segmented states, which also use the fp32 state region of the
    workspace; each call follows one of another shape or chunk, so that the
    leftovers sit at other offsets of the array."""
    build.build()
    lib = gka.lib()
    for shape in [(2, 4, 1024, 128, 128), (1, 40, 256, 128, 64), (1, 24, 512, 128, 64)]:
        assert gka.workspace_bytes(*shape, torch.bfloat16) <= 64 << 20
    _check_against_gka_forward(lib, 2, 4, 1024, 128, torch.bfloat16, 128, 20, 0.5, 31)
    _check_against_gka_forward(lib, 1, 40, 256, 128, torch.bfloat16, 64, 20, 0.5, 32)
    _check_against_gka_forward(lib, 1, 24, 512, 128, torch.bfloat16, 64, 20, 0.1, 33)
    _check_against_gka_forward(lib, 1, 40, 256, 128, torch.bfloat16, 64, 20, 0.5, 34)


def test_static_scratch_refuses_oversized_problem():
    build.build()
    lib = gka.lib()
    B, H, T, D, chunk = 8, 8, 2048, 128, 64          # needs ~280 MB of scratch
    assert gka.workspace_bytes(B, H, T, D, chunk) > 64 << 20
    q = torch.zeros(B, H, T, D, dtype=torch.bfloat16, device="cuda")
    beta = torch.ones(B, H, T, device="cuda")
    o = torch.zeros_like(q)
    fs = torch.zeros(B, H, 2, D, D, device="cuda")
    assert _call(lib, q, q, q, beta, o, 0.5, 20, chunk, fs) == -8
    assert torch.all(o == 0)
