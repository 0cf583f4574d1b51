"""GPU parity of gka_forward (through the C ABI) against the float64 oracle on
the same seeded inputs.

Metric: max over (batch, head) of the relative Frobenius error of o over the
head's [T, D] slab; bars 1e-4 (fp32 inputs) and 2e-2 (bf16 inputs, fp32
accumulation).  Intermediate results (chunk-start states, per-token norms) are
read back from the workspace and compared too.
"""
import numpy as np
import pytest
import torch

import oracle
from helpers import TOL, cuda, f64, head_rel_err
from test_ridge_regression_b200 import build, gka
from test_ridge_regression_b200.inputs import WORKLOADS, make_inputs, workload_inputs

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def _built():
    build.build()


def run_forward(q, k, v, beta, a, r, C):
    B, H, T, D = q.shape
    qd, kd, vd, bd = cuda(q, k, v, beta)
    ws = gka.alloc_workspace(B, H, T, D, C, q.dtype)
    fs = torch.full((B, H, 2, D, D), float("nan"), device="cuda")
    o = gka.gka_forward(qd, kd, vd, bd, a, r, C, final_state=fs, workspace=ws)
    assert gka.device_status() == 0
    return o, fs, ws


def tensor_core_path(dtype, D, C):
    """The rule include/gka.h states for the tensor-core solve."""
    return dtype == torch.bfloat16 and D == 128 and C in (64, 128)


def ws_views(ws, B, H, T, D, C, dtype):
    """Chunk-start states [B,H,N,2,D,D] (fp32; on the tensor-core path the fp16
    copies with their power-of-two scales undone) and norms [B,H,T]."""
    L = gka.workspace_layout(B, H, T, D, C, dtype)
    N = T // C
    norms = ws[L.norms_offset:L.norms_offset + 4 * B * H * T].view(torch.float32).view(B, H, T)
    if tensor_core_path(dtype, D, C):
        n16 = B * H * N * 2 * D * D
        lp = ws[L.states_lp_offset:L.states_lp_offset + 2 * n16].view(torch.float16)
        lp = lp.view(B, H, N, 2, D, D).double()
        off = L.states_lp_offset + ((2 * n16 + 255) // 256) * 256
        off += ((4 * B * H * N * 2 + 255) // 256) * 256
        ex = ws[off:off + 4 * B * H * N * 2].view(torch.int32).view(B, H, N, 2).double()
        return lp * torch.pow(2.0, -ex)[..., None, None], norms
    states = ws[L.states_offset:L.states_offset + 4 * B * H * (N + 1) * 2 * D * D]
    states = states.view(torch.float32).view(B, H, N + 1, 2, D, D)
    return states[:, :, :N], norms


def check_against_oracle(q, k, v, beta, a, r, C, *, check_ws=True):
    B, H, T, D = q.shape
    o, fs, ws = run_forward(q, k, v, beta, a, r, C)
    ref = oracle.forward(q, k, v, beta, a, r, want_norms=True, want_final_state=True,
                         chunk=C, want_chunk_states=True)
    tol = TOL[q.dtype]
    err = head_rel_err(o, ref["o"])
    print(f"o rel err {err:.3e} (bar {tol:g})")
    assert err <= tol
    ferr = head_rel_err(fs, ref["final_state"])
    print(f"final state rel err {ferr:.3e} (bar 1e-05)")
    assert ferr <= 1e-5, ferr
    if check_ws:
        # intermediate results: fp32 on the CUDA-core path; on the tensor-core path
        # the states are fp16 copies (relative rounding 2^-11) and the norms use them
        tc = tensor_core_path(q.dtype, D, C)
        states, norms = ws_views(ws, B, H, T, D, C, q.dtype)
        assert head_rel_err(norms, ref["norms"]) <= (1e-3 if tc else 1e-5)
        cs = f64(states)
        assert np.all(cs[:, :, 0] == 0)
        if T // C > 1:
            assert head_rel_err(cs[:, :, 1:], ref["chunk_states"][:, :, 1:],
                                head_dims=3) <= (1e-3 if tc else 1e-5)
    return err


def test_tiny_fp32_workload():
    w = WORKLOADS["tiny_fp32_b1h2t256d32"]
    q, k, v, beta = workload_inputs(w)
    check_against_oracle(q, k, v, beta, w.a, w.r, w.chunk)


@pytest.mark.parametrize("D", [32, 64, 128])
@pytest.mark.parametrize("C", [16, 32, 64, 128])
def test_fp32_dims_and_chunks(D, C):
    q, k, v, beta = make_inputs(1, 2, 256, D, torch.float32, 2.0, 1.0, seed=100 + D + C)
    check_against_oracle(q, k, v, beta, 0.5, 8, C)


@pytest.mark.parametrize("name", ["bf16_b8h8t2048d128", "bf16_b4h16t8192d128_a0.1",
                                  "bf16_b1h8t131072d128"])
def test_bf16_workload_distributions_small(name):
    # the workload's dtype, a, r, chunk and beta distribution at B=1, H=2, T=4 chunks + more
    w = WORKLOADS[name]
    q, k, v, beta = workload_inputs(w, B=1, H=2, T=6 * w.chunk)
    check_against_oracle(q, k, v, beta, w.a, w.r, w.chunk)


@pytest.mark.parametrize("C", [16, 32])
def test_bf16_cuda_core_chunks(C):
    # bf16 with chunks outside {64, 128} runs the CUDA-core solve
    q, k, v, beta = make_inputs(1, 2, 256, 128, torch.bfloat16, 3.0, 1.0, seed=300 + C)
    check_against_oracle(q, k, v, beta, 0.5, 20, C)


@pytest.mark.parametrize("C", [64, 128])
@pytest.mark.parametrize("r", [1, 2, 3])
def test_tensor_core_short_iterations(C, r):
    # r = 1 (no matrix-vector product), 2 and 3 on the tensor-core path
    q, k, v, beta = make_inputs(1, 2, 2 * C, 128, torch.bfloat16, 2.0, 1.0, seed=400 + r + C)
    check_against_oracle(q, k, v, beta, 0.5, r, C)


def test_tensor_core_resets_and_strong_forgetting():
    q, k, v, beta = make_inputs(2, 2, 384, 128, torch.bfloat16, 0.0, 2.0, seed=17)
    beta[0, 0, 64] = 0.0
    beta[0, 1, 70:75] = 0.0
    beta[1, 0, 0] = 0.0
    check_against_oracle(q, k, v, beta, 0.1, 30, 64)
    check_against_oracle(q, k, v, beta, 0.1, 30, 128)


def test_beta_zero_resets():
    q, k, v, beta = make_inputs(1, 2, 256, 64, torch.float32, 1.0, 1.0, seed=7)
    beta[0, 0, 64] = 0.0      # first token of a chunk
    beta[0, 0, 100] = 0.0     # inside a chunk
    beta[0, 1, 0] = 0.0       # very first token
    beta[0, 1, 130:140] = 0.0 # a run of resets
    check_against_oracle(q, k, v, beta, 0.5, 10, 64)


def test_unnormalised_keys_and_strong_forgetting():
    g = torch.Generator().manual_seed(3)
    q = torch.randn(1, 2, 256, 128, generator=g)
    k = 3.0 * torch.randn(1, 2, 256, 128, generator=g)
    v = torch.randn(1, 2, 256, 128, generator=g)
    beta = torch.sigmoid(-1.0 + torch.randn(1, 2, 256, generator=g))
    check_against_oracle(q, k, v, beta, 0.1, 30, 64)


def test_tensor_core_zero_keys_and_queries():
    # zero keys at the start of a sequence and after a reset leave ||H_t|| = 0 (output 0
    # by definition), zero queries give x = 0; the other tokens of the same chunks share
    # the chunk's iterate scale and decay weights with them
    q, k, v, beta = make_inputs(1, 2, 256, 128, torch.bfloat16, 2.0, 1.0, seed=21)
    k[0, 0, :5] = 0.0
    beta[0, 1, 100] = 0.0
    k[0, 1, 100:103] = 0.0
    q[0, 0, 70:74] = 0.0
    q[0, 1, 130] = 0.0
    for C in (64, 128):
        check_against_oracle(q, k, v, beta, 0.5, 20, C)


def test_tensor_core_query_scale_spread():
    # the iterate scale is one power of two per chunk, set by the largest query: token
    # queries spanning 2^-10 .. 2^10 within a chunk keep their relative accuracy, token
    # by token (not only in the head's Frobenius norm, which the large tokens dominate)
    q, k, v, beta = make_inputs(1, 2, 256, 128, torch.bfloat16, 2.0, 1.0, seed=22)
    g = torch.Generator().manual_seed(5)
    scale = torch.pow(2.0, torch.randint(-10, 11, (1, 2, 256, 1), generator=g).float())
    q = (q.float() * scale).to(torch.bfloat16)
    ref = oracle.forward(q, k, v, beta, 0.5, 20)["o"]
    for C in (64, 128):
        o, _, _ = run_forward(q, k, v, beta, 0.5, 20, C)
        got, want = f64(o), f64(ref)
        per_tok = np.linalg.norm(got - want, axis=-1) / np.linalg.norm(want, axis=-1)
        print(f"chunk {C}: worst per-token rel err {per_tok.max():.3e}")
        assert per_tok.max() <= TOL[torch.bfloat16]


def test_chunk_size_does_not_change_result():
    q, k, v, beta = make_inputs(2, 2, 512, 128, torch.bfloat16, 3.0, 1.0, seed=11)
    o64, fs64, _ = run_forward(q, k, v, beta, 0.5, 20, 64)
    o128, fs128, _ = run_forward(q, k, v, beta, 0.5, 20, 128)
    assert head_rel_err(o64, o128) <= 1e-2
    assert head_rel_err(fs64, fs128) <= 1e-5


def test_empty_sequence_and_no_heads():
    D = 64
    q = torch.zeros(1, 2, 0, D, device="cuda")
    beta = torch.zeros(1, 2, 0, device="cuda")
    fs = torch.full((1, 2, 2, D, D), 7.0, device="cuda")
    ws = torch.empty(256, dtype=torch.uint8, device="cuda")
    o = gka.gka_forward(q, q, q, beta, 0.5, 4, 64, final_state=fs, workspace=ws)
    torch.cuda.synchronize()
    assert o.numel() == 0 and torch.all(fs == 0)
    q0 = torch.zeros(0, 2, 64, D, device="cuda")
    gka.gka_forward(q0, q0, q0, torch.zeros(0, 2, 64, device="cuda"), 0.5, 4, 64, workspace=ws)
    assert gka.device_status() == 0


def test_error_codes_on_device_tensors():
    q = torch.zeros(1, 1, 100, 64, device="cuda")
    beta = torch.ones(1, 1, 100, device="cuda")
    with pytest.raises(gka.GkaError) as e:
        gka.gka_forward(q, q, q, beta, 0.5, 4, 64, workspace=torch.empty(1 << 20, dtype=torch.uint8,
                                                                             device="cuda"))
    assert e.value.status == -3
    q = torch.zeros(1, 1, 128, 64, device="cuda")
    beta = torch.ones(1, 1, 128, device="cuda")
    with pytest.raises(gka.GkaError) as e:
        gka.gka_forward(q, q, q, beta, 0.5, 4, 64, workspace=torch.empty(256, dtype=torch.uint8,
                                                                             device="cuda"))
    assert e.value.status == -4


# ---------------------------------------------------------------------------
# Full-size workloads in the launch configuration the benchmark times; the
# oracle checks a sample of heads (heads are independent), over the whole
# sequence or, for the longest ones, over a window of outputs after running
# the state recurrence through the whole prefix.
# ---------------------------------------------------------------------------

def _sampled(name, heads, window):
    w = WORKLOADS[name]
    q, k, v, beta = workload_inputs(w)
    o, fs, _ = run_forward(q, k, v, beta, w.a, w.r, w.chunk)
    o = o.cpu()
    worst = 0.0
    for (b, h) in heads:
        sl = (slice(b, b + 1), slice(h, h + 1))
        start = w.T - window if window else 0
        ref = oracle.forward(q[sl], k[sl], v[sl], beta[sl], w.a, w.r, solve_from=start,
                             want_final_state=True)
        err = head_rel_err(o[sl][:, :, start:], ref["o"][:, :, start:])
        worst = max(worst, err)
        assert head_rel_err(fs[sl], ref["final_state"]) <= 1e-4
    print(f"{name}: sampled o rel err {worst:.3e}")
    assert worst <= TOL[w.dtype]


def test_full_b8h8t2048_sampled():
    _sampled("bf16_b8h8t2048d128", [(0, 0), (7, 7), (3, 5)], window=0)


def _sampled_windows(name, heads, window, fractions=(0.25, 0.5, 0.75)):
    """Outputs at several windows spread along the sequence (at the given fractions
    of T and at its end), for a sample of heads, with the oracle's state recurrence
    carried through every prefix in segments (init_state), and the final state."""
    w = WORKLOADS[name]
    q, k, v, beta = workload_inputs(w)
    o, fs, _ = run_forward(q, k, v, beta, w.a, w.r, w.chunk)
    o, fs = o.cpu(), fs.cpu()
    pick = lambda x: torch.stack([x[b, h] for b, h in heads])[None]
    qs, ks, vs, bs, os_, fss = (pick(x) for x in (q, k, v, beta, o, fs))
    starts = sorted({int(f * w.T) // w.chunk * w.chunk for f in fractions} | {w.T - window})
    state, pos, worst = None, 0, 0.0
    for s0 in starts:
        seg = slice(pos, s0 + window)
        ref = oracle.forward(qs[:, :, seg], ks[:, :, seg], vs[:, :, seg], bs[:, :, seg], w.a, w.r,
                             init_state=state, solve_from=s0 - pos, want_final_state=True,
                             nthreads=len(heads))
        err = head_rel_err(os_[:, :, s0:s0 + window], ref["o"][:, :, s0 - pos:])
        print(f"{name}: window [{s0}, {s0 + window}) o rel err {err:.3e}")
        worst = max(worst, err)
        state, pos = ref["final_state"], s0 + window
    assert pos == w.T
    assert head_rel_err(fss, state) <= 1e-4
    assert worst <= TOL[w.dtype]


def test_full_b4h16t8192_sampled():
    _sampled_windows("bf16_b4h16t8192d128_a0.1", [(0, 0), (1, 5), (2, 10), (3, 15)], window=512)


def test_full_b1h8t131072_sampled():
    _sampled_windows("bf16_b1h8t131072d128", [(0, 0), (0, 3), (0, 7)], window=512)
