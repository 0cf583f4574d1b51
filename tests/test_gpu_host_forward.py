"""gka_forward_host (host buffers, copies overlapped with the compute) against
gka_forward on device copies of the same inputs.  A head's result does not
depend on how many heads share a launch, so slicings that keep the chunk-state
path (one pass from 24 heads, else two passes) give identical bits; mixed
paths agree to the fp16 state copies."""
import pytest
import torch

from helpers import head_rel_err
from test_ridge_regression_b200 import build, gka
from test_ridge_regression_b200.inputs import make_inputs

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def _built():
    build.build()


def device_reference(q, k, v, beta, a, r, C):
    B, H, T, D = q.shape
    fs = torch.empty(B, H, 2, D, D, device="cuda")
    o = gka.gka_forward(q.cuda(), k.cuda(), v.cuda(), beta.cuda(), a, r, C, final_state=fs)
    torch.cuda.synchronize()
    return o.cpu(), fs.cpu()


def host_run(q, k, v, beta, a, r, C, slice_pairs, pinned=True):
    B, H, T, D = q.shape
    if pinned:
        q, k, v, beta = (t.pin_memory() for t in (q, k, v, beta))
    fs = torch.empty(B, H, 2, D, D, pin_memory=pinned)
    o = gka.gka_forward_host(q, k, v, beta, a, r, C, final_state=fs, slice_pairs=slice_pairs)
    torch.cuda.current_stream().synchronize()
    assert gka.device_status() == 0
    return o, fs


@pytest.mark.parametrize("dtype,D,C,slice_pairs", [
    (torch.bfloat16, 128, 64, 0), (torch.bfloat16, 128, 64, 5), (torch.bfloat16, 128, 128, 3),
    (torch.float32, 64, 32, 7), (torch.float32, 32, 64, 1)])
def test_host_forward_identical_to_device(dtype, D, C, slice_pairs):
    q, k, v, beta = make_inputs(2, 8, 2 * C, D, dtype, 2.0, 1.0, seed=1100 + D + C)
    o_ref, fs_ref = device_reference(q, k, v, beta, 0.5, 8, C)
    o, fs = host_run(q, k, v, beta, 0.5, 8, C, slice_pairs)
    assert torch.equal(o, o_ref)
    assert torch.equal(fs, fs_ref)


def test_host_forward_one_pass_slices_identical():
    # 80 heads: the whole call and slices of 40 both take the one-pass state kernel
    q, k, v, beta = make_inputs(2, 40, 192, 128, torch.bfloat16, 3.0, 1.0, seed=1201)
    o_ref, fs_ref = device_reference(q, k, v, beta, 0.5, 10, 64)
    o, fs = host_run(q, k, v, beta, 0.5, 10, 64, 40)
    assert torch.equal(o, o_ref) and torch.equal(fs, fs_ref)


def test_host_forward_mixed_state_paths_and_pageable_memory():
    # 48 heads in one device call (one pass) vs slices of 10 (segmented), pageable host memory
    q, k, v, beta = make_inputs(2, 24, 192, 128, torch.bfloat16, 3.0, 1.0, seed=1202)
    o_ref, fs_ref = device_reference(q, k, v, beta, 0.5, 10, 64)
    o, fs = host_run(q, k, v, beta, 0.5, 10, 64, 10, pinned=False)
    assert head_rel_err(o.float(), o_ref.float()) <= 5e-3
    assert head_rel_err(fs, fs_ref) <= 1e-5


def test_host_forward_twice_with_one_workspace():
    # 20 heads: the whole call and the slices of 8 both cut the two chunks into two segments
    q, k, v, beta = make_inputs(1, 20, 128, 128, torch.bfloat16, 2.0, 1.0, seed=1203)
    q, k, v, beta = (t.pin_memory() for t in (q, k, v, beta))
    ws = gka.alloc_host_workspace(1, 20, 128, 128, 64, torch.bfloat16, 8)
    o1 = gka.gka_forward_host(q, k, v, beta, 0.5, 6, 64, slice_pairs=8, workspace=ws)
    o2 = gka.gka_forward_host(q, k, v, beta, 0.5, 6, 64, slice_pairs=8, workspace=ws)
    torch.cuda.current_stream().synchronize()
    assert torch.equal(o1, o2)
    o_ref, _ = device_reference(q, k, v, beta, 0.5, 6, 64)
    assert torch.equal(o1, o_ref)


def test_host_forward_default_schedule_64_pairs():
    # the default schedule at 64 pairs is 24, 24, 16: every slice takes segmented states,
    # against one device call (one pass)
    q, k, v, beta = make_inputs(8, 8, 128, 128, torch.bfloat16, 3.0, 1.0, seed=1204)
    o_ref, fs_ref = device_reference(q, k, v, beta, 0.5, 10, 64)
    o, fs = host_run(q, k, v, beta, 0.5, 10, 64, 0)
    assert head_rel_err(o.float(), o_ref.float()) <= 5e-3
    assert head_rel_err(fs, fs_ref) <= 1e-5
