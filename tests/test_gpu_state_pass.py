"""GPU parity of the tensor-core chunk-state kernels against the float64 oracle:
the one-pass kernel over whole sequences (many heads), and the segmented path
(few heads: segment aggregates on the tensor cores, a scan of the segment
starts, then the one-pass kernel from every segment start), and the two
against each other on the same heads.

gka_forward cuts every sequence into S = min(N, SMs // (2 * B*H)) segments of
whole chunks (S = 1: the plain one-pass kernel), so the head count picks the
path."""
import pytest
import torch

from helpers import cuda, head_rel_err
from test_gpu_forward import check_against_oracle
from test_ridge_regression_b200 import gka
from test_ridge_regression_b200.inputs import make_gate, make_inputs

pytestmark = pytest.mark.gpu


def segments(BH, N):
    sms = torch.cuda.get_device_properties(0).multi_processor_count
    return max(1, min(N, sms // (2 * BH)))


@pytest.mark.parametrize("C", [64, 128])
@pytest.mark.parametrize("nchunks", [1, 3])
def test_one_pass_states_match_oracle(C, nchunks):
    B, H = 5, 8
    assert segments(B * H, nchunks) == 1
    q, k, v, beta = make_inputs(B, H, nchunks * C, 128, torch.bfloat16, 2.0, 1.0,
                                seed=700 + C + nchunks)
    check_against_oracle(q, k, v, beta, 0.5, 8, C)


@pytest.mark.parametrize("C", [64, 128])
def test_one_pass_resets_and_strong_forgetting(C):
    B, H = 5, 8
    assert segments(B * H, 4) == 1
    q, k, v, beta = make_inputs(B, H, 4 * C, 128, torch.bfloat16, 0.0, 2.0, seed=800 + C)
    beta[0, 0, C] = 0.0             # reset at a chunk boundary
    beta[1, 2, C + 5:C + 9] = 0.0   # inside a chunk
    beta[3, 3, 0] = 0.0             # first token
    check_against_oracle(q, k, v, beta, 0.1, 12, C)


@pytest.mark.parametrize("C,H,nchunks", [(64, 8, 20), (128, 8, 11), (64, 2, 12), (128, 1, 3)])
def test_segmented_states_match_oracle(C, H, nchunks):
    # uneven segments of several chunks (8 heads), one chunk each (2 heads), and
    # fewer chunks than the SMs would allow segments for (1 head)
    S = segments(H, nchunks)
    assert S > 1
    q, k, v, beta = make_inputs(1, H, nchunks * C, 128, torch.bfloat16, 3.0, 1.0,
                                seed=1700 + C + H + nchunks)
    check_against_oracle(q, k, v, beta, 0.5, 10, C)


@pytest.mark.parametrize("C", [64, 128])
def test_segmented_resets_gate_and_strong_forgetting(C):
    H, N = 8, 18
    S = segments(H, N)
    assert 1 < S < N
    q, k, v, beta = make_inputs(1, H, N * C, 128, torch.bfloat16, 0.0, 2.0, seed=1800 + C)
    first = [(s * N) // S for s in range(S)]
    beta[0, 0, first[1] * C] = 0.0               # reset at a segment start
    beta[0, 1, first[2] * C - 1] = 0.0           # last token of a segment
    beta[0, 2, first[1] * C + C + 3:first[1] * C + C + 40] = 0.0   # a run inside a segment
    beta[0, 3, :C] = 0.0                          # the whole first chunk
    check_against_oracle(q, k, v, beta, 0.1, 12, C)
    # with a write gate, zero on half a chunk of one head (a longer run without writes
    # under this forgetting decays the state below the fp32 range, which the kernels
    # treat as a zero state)
    import oracle
    from helpers import TOL
    g = make_gate((1, H, N * C), seed=1801 + C)
    g[0, 4, 2 * C:2 * C + C // 2] = 0.0
    qd, kd, vd, bd, gd = cuda(q, k, v, beta, g)
    fs = torch.empty(1, H, 2, 128, 128, device="cuda")
    o = gka.gka_forward_gated(qd, kd, vd, bd, gd, 0.1, 12, C, final_state=fs)
    ref = oracle.forward(q, k, v, beta, 0.1, 12, gate=g, want_final_state=True)
    assert gka.device_status() == 0
    assert head_rel_err(o, ref["o"]) <= TOL[torch.bfloat16]
    assert head_rel_err(fs, ref["final_state"]) <= 1e-5


@pytest.mark.parametrize("C", [64, 128])
def test_one_pass_agrees_with_segmented(C):
    # 40 heads run in one call (one pass over every sequence) and as five calls of
    # 8 heads (segmented); outputs agree to the fp16 state copies, final states to fp32
    B, H, N = 5, 8, 14
    assert segments(B * H, N) == 1 and segments(H, N) > 1
    q, k, v, beta = make_inputs(B, H, N * C, 128, torch.bfloat16, 3.0, 1.0, seed=900 + C)
    qd, kd, vd, bd = cuda(q, k, v, beta)
    fs = torch.empty(B, H, 2, 128, 128, device="cuda")
    o = gka.gka_forward(qd, kd, vd, bd, 0.5, 10, C, final_state=fs)
    for b in range(B):
        fsb = torch.empty(1, H, 2, 128, 128, device="cuda")
        ob = gka.gka_forward(qd[b:b + 1].contiguous(), kd[b:b + 1].contiguous(),
                             vd[b:b + 1].contiguous(), bd[b:b + 1].contiguous(), 0.5, 10, C,
                             final_state=fsb)
        assert head_rel_err(ob.float().cpu(), o[b:b + 1].float().cpu()) <= 5e-3
        assert head_rel_err(fsb.cpu(), fs[b:b + 1].cpu()) <= 1e-5
    assert gka.device_status() == 0
