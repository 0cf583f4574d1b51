"""GPU parity of the write-gated forward and decode step (gka_forward_gated,
gka_decode_step_gated, through the C ABI) against the float64 oracle with the
same gate: the paper's beta_t-augmented variant (ai.info page, Main Findings),
H_t = beta_t H_{t-1} + g_t k_t k_t^T and M_t = beta_t M_{t-1} + g_t v_t k_t^T.

Every kernel family is covered: the CUDA-core path (fp32, any D; bf16 with
chunks 16/32), the tensor-core path with segmented chunk states (few heads:
segment aggregates, a scan of the segment starts, one pass per segment) and
with the one-pass state kernel over whole sequences (38 heads or more on 148
SMs), and both decode kernels.  Bars as for the ungated layer: 1e-4 (fp32 inputs),
2e-2 (bf16 inputs); a gate of ones reproduces the ungated kernels bit for bit.
"""
import numpy as np
import pytest
import torch

import oracle
from helpers import TOL, cuda, f64, head_rel_err
from test_gpu_forward import tensor_core_path, ws_views
from test_ridge_regression_b200 import build, gka
from test_ridge_regression_b200.inputs import WORKLOADS, make_gate, make_inputs, workload_inputs

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def _built():
    build.build()


def gated_inputs(B, H, T, D, dtype, seed, beta_mu=2.0):
    q, k, v, beta = make_inputs(B, H, T, D, dtype, beta_mu, 1.0, seed)
    gate = make_gate((B, H, T), seed)
    gate[0, 0, 0] = 0.0                   # the very first token writes nothing
    gate[0, -1, T // 2] = 0.0             # a token inside the sequence writes nothing
    gate[-1, 0, min(63, T - 1)] = 1.0     # last token of a 64-token chunk, full write
    return q, k, v, beta, gate


def run_gated(q, k, v, beta, gate, a, r, C):
    B, H, T, D = q.shape
    qd, kd, vd, bd, gd = cuda(q, k, v, beta, gate)
    ws = gka.alloc_workspace(B, H, T, D, C, q.dtype)
    fs = torch.full((B, H, 2, D, D), float("nan"), device="cuda")
    o = gka.gka_forward_gated(qd, kd, vd, bd, gd, a, r, C, final_state=fs, workspace=ws)
    assert gka.device_status() == 0
    return o, fs, ws


def check_gated(q, k, v, beta, gate, a, r, C):
    B, H, T, D = q.shape
    o, fs, ws = run_gated(q, k, v, beta, gate, a, r, C)
    ref = oracle.forward(q, k, v, beta, a, r, gate=gate, want_norms=True, want_final_state=True)
    err = head_rel_err(o, ref["o"])
    ferr = head_rel_err(fs, ref["final_state"])
    tc = tensor_core_path(q.dtype, D, C)
    _, norms = ws_views(ws, B, H, T, D, C, q.dtype)
    nerr = head_rel_err(norms, ref["norms"])
    print(f"gated B{B} H{H} T{T} D{D} C{C} {q.dtype}: o {err:.3e}, final state {ferr:.3e}, "
          f"norms {nerr:.3e}")
    assert err <= TOL[q.dtype]
    assert ferr <= 1e-5
    assert nerr <= (1e-3 if tc else 1e-5)
    return err


@pytest.mark.parametrize("D", [32, 64, 128])
def test_gated_cuda_core_fp32(D):
    check_gated(*gated_inputs(1, 2, 256, D, torch.float32, 500 + D), 0.5, 10, 64)


@pytest.mark.parametrize("C", [16, 32])
def test_gated_cuda_core_bf16(C):
    check_gated(*gated_inputs(1, 2, 256, 128, torch.bfloat16, 520 + C, 3.0), 0.5, 20, C)


@pytest.mark.parametrize("C", [64, 128])
def test_gated_tensor_core_segmented_states(C):
    # 4 heads, 4 chunks: the sequences cut into one-chunk segments
    check_gated(*gated_inputs(2, 2, 4 * C, 128, torch.bfloat16, 540 + C, 3.0), 0.5, 20, C)


@pytest.mark.parametrize("C", [64, 128])
def test_gated_tensor_core_state_pass(C):
    # 40 heads: the one-pass state kernel over whole sequences
    check_gated(*gated_inputs(1, 40, 2 * C, 128, torch.bfloat16, 560 + C, 3.0), 0.5, 20, C)


def test_gated_tensor_core_small_a_resets():
    q, k, v, beta, gate = gated_inputs(2, 2, 384, 128, torch.bfloat16, 580, 1.0)
    beta[0, 1, 70:75] = 0.0
    gate[1, 1, 64:128] = 0.0              # a whole chunk that writes nothing
    check_gated(q, k, v, beta, gate, 0.1, 30, 64)


@pytest.mark.parametrize("dtype,D,C,H", [(torch.float32, 64, 64, 2),
                                         (torch.bfloat16, 128, 32, 2),
                                         (torch.bfloat16, 128, 64, 2),
                                         (torch.bfloat16, 128, 128, 2),
                                         (torch.bfloat16, 128, 64, 40)])
def test_unit_gate_and_null_gate_match_ungated_bit_for_bit(dtype, D, C, H):
    q, k, v, beta = make_inputs(1, H, 2 * C, D, dtype, 3.0, 1.0, seed=600 + C + H)
    qd, kd, vd, bd = cuda(q, k, v, beta)
    ones = torch.ones_like(bd)
    ws = gka.alloc_workspace(1, H, 2 * C, D, C, dtype)
    outs = []
    for call in (lambda fs: gka.gka_forward(qd, kd, vd, bd, 0.5, 20, C, final_state=fs,
                                            workspace=ws),
                 lambda fs: gka.gka_forward_gated(qd, kd, vd, bd, None, 0.5, 20, C,
                                                  final_state=fs, workspace=ws),
                 lambda fs: gka.gka_forward_gated(qd, kd, vd, bd, ones, 0.5, 20, C,
                                                  final_state=fs, workspace=ws)):
        fs = torch.empty(1, H, 2, D, D, device="cuda")
        outs.append((call(fs).clone(), fs))
    assert gka.device_status() == 0
    for o, fs in outs[1:]:
        assert torch.equal(o, outs[0][0]) and torch.equal(fs, outs[0][1])


def test_gated_full_b8h8t2048_sampled():
    """The default benchmark workload with a gate, in its launch configuration;
    the oracle checks a sample of heads over the whole sequence."""
    w = WORKLOADS["bf16_b8h8t2048d128"]
    q, k, v, beta = workload_inputs(w)
    gate = make_gate((w.B, w.H, w.T), w.seed)
    o, fs, _ = run_gated(q, k, v, beta, gate, w.a, w.r, w.chunk)
    o = o.cpu()
    worst = 0.0
    for (b, h) in [(0, 0), (7, 7), (3, 5)]:
        sl = (slice(b, b + 1), slice(h, h + 1))
        ref = oracle.forward(q[sl], k[sl], v[sl], beta[sl], w.a, w.r, gate=gate[sl],
                             want_final_state=True)
        worst = max(worst, head_rel_err(o[sl], ref["o"]))
        assert head_rel_err(fs[sl], ref["final_state"]) <= 1e-4
    print(f"gated full size: sampled o rel err {worst:.3e}")
    assert worst <= TOL[torch.bfloat16]


@pytest.mark.parametrize("D,dtype", [(32, torch.float32), (64, torch.float32),
                                     (128, torch.float32), (128, torch.bfloat16)])
def test_gated_decode_steps(D, dtype):
    batch, H, a, r = 3, 4, 0.5, 20
    q, k, v, beta, gate = gated_inputs(batch, H, 64, D, dtype, 700 + D)
    st0 = oracle.forward(q, k, v, beta, a, 1, gate=gate, solve_from=64,
                         want_final_state=True)["final_state"]
    st_gpu = torch.from_numpy(st0).float().cuda()
    st_ref = f64(st_gpu.cpu())
    outs_gpu, outs_ref = [], []
    for s in range(5):
        qs, ks, vs, bs = (t[:, :, 0] for t in make_inputs(batch, H, 1, D, dtype, 3.0, 1.0,
                                                           seed=710 + 13 * s + D))
        gs = make_gate((batch, H), 720 + s)
        if s == 2:
            gs[0, 0] = 0.0
        o = gka.gka_decode_step_gated(st_gpu, qs.cuda(), ks.cuda(), vs.cuda(), bs.cuda(),
                                      gs.cuda(), a, r)
        o_ref, st_ref = oracle.decode_step(st_ref, qs, ks, vs, bs, a, r, gate=gs)
        outs_gpu.append(o.cpu())
        outs_ref.append(o_ref)
    assert gka.device_status() == 0
    err = head_rel_err(torch.stack(outs_gpu, dim=2), np.stack(outs_ref, axis=2))
    print(f"gated decode D={D} {dtype}: o rel err {err:.3e}")
    assert err <= TOL[dtype]
    assert head_rel_err(st_gpu, st_ref) <= 1e-5


def test_gated_prefill_feeds_gated_decode():
    B, H, T, D, a, r = 1, 2, 128, 128, 0.5, 20
    q, k, v, beta, gate = gated_inputs(B, H, T + 2, D, torch.bfloat16, 730)
    ws = gka.alloc_workspace(B, H, T, D, 64, torch.bfloat16)
    st = torch.empty(B, H, 2, D, D, device="cuda")
    pre = [t[:, :, :T].contiguous().cuda() for t in (q, k, v, beta, gate)]
    gka.gka_forward_gated(*pre, a, r, 64, final_state=st, workspace=ws)
    outs = []
    for t in (T, T + 1):
        step = [x[:, :, t].contiguous().cuda() for x in (q, k, v, beta, gate)]
        outs.append(gka.gka_decode_step_gated(st, *step, a, r).cpu())
    ref = oracle.forward(q, k, v, beta, a, r, gate=gate, solve_from=T)["o"][:, :, T:]
    assert head_rel_err(torch.stack(outs, dim=2), ref) <= TOL[torch.bfloat16]
