"""GPU parity of the one-pass chunk-state kernel (tensor-core path with at
least 24 heads) against the float64 oracle, and against the chunk-parallel
two-pass path (fewer heads) on the same heads."""
import pytest
import torch

from helpers import cuda, head_rel_err
from test_gpu_forward import check_against_oracle
from test_ridge_regression_b200 import gka
from test_ridge_regression_b200.inputs import make_inputs

pytestmark = pytest.mark.gpu

ONE_PASS_MIN_HEADS = 24   # B*H from which gka_forward takes the one-pass state kernel


@pytest.mark.parametrize("C", [64, 128])
@pytest.mark.parametrize("nchunks", [1, 3])
def test_one_pass_states_match_oracle(C, nchunks):
    q, k, v, beta = make_inputs(3, 8, nchunks * C, 128, torch.bfloat16, 2.0, 1.0,
                                seed=700 + C + nchunks)
    check_against_oracle(q, k, v, beta, 0.5, 8, C)


@pytest.mark.parametrize("C", [64, 128])
def test_one_pass_resets_and_strong_forgetting(C):
    q, k, v, beta = make_inputs(4, 6, 4 * C, 128, torch.bfloat16, 0.0, 2.0, seed=800 + C)
    beta[0, 0, C] = 0.0             # reset at a chunk boundary
    beta[1, 2, C + 5:C + 9] = 0.0   # inside a chunk
    beta[3, 3, 0] = 0.0             # first token
    check_against_oracle(q, k, v, beta, 0.1, 12, C)


@pytest.mark.parametrize("C", [64, 128])
def test_one_pass_agrees_with_two_pass(C):
    # 24 heads run in one call (one-pass states) and as three calls of 8 heads
    # (two-pass states); outputs and final states agree to the fp16 state copies
    q, k, v, beta = make_inputs(3, 8, 5 * C, 128, torch.bfloat16, 3.0, 1.0, seed=900 + C)
    qd, kd, vd, bd = cuda(q, k, v, beta)
    assert 3 * 8 >= ONE_PASS_MIN_HEADS > 8
    fs = torch.empty(3, 8, 2, 128, 128, device="cuda")
    o = gka.gka_forward(qd, kd, vd, bd, 0.5, 10, C, final_state=fs)
    for b in range(3):
        fsb = torch.empty(1, 8, 2, 128, 128, device="cuda")
        ob = gka.gka_forward(qd[b:b + 1].contiguous(), kd[b:b + 1].contiguous(),
                             vd[b:b + 1].contiguous(), bd[b:b + 1].contiguous(), 0.5, 10, C,
                             final_state=fsb)
        assert head_rel_err(ob.float().cpu(), o[b:b + 1].float().cpu()) <= 5e-3
        assert head_rel_err(fsb.cpu(), fs[b:b + 1].cpu()) <= 1e-5
    assert gka.device_status() == 0
