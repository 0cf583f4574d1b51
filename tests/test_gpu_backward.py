"""GPU parity of gka_backward (implicit-differentiation backward, through the C
ABI) against the float64 oracle's backward on the same seeded inputs.

Metric: max over (batch, head) of the relative Frobenius error over the head's
slab, for dq, dk, dv ([T, D]) and dbeta, dgate ([T]).  With bf16 inputs, D = 128,
chunk 32 and T a multiple of 64 every product of the backward runs on the tensor
cores (fp16 operands with power-of-two scales, fp32 accumulation); otherwise it
computes in fp32 on CUDA cores.  Bars: 1e-4 with fp32 inputs, 2e-2 with bf16 inputs
(dq, dk, dv are also rounded to bf16).
"""
import numpy as np
import pytest
import torch

import oracle
from helpers import cuda, head_rel_err
from test_ridge_regression_b200 import build, gka
from test_ridge_regression_b200.inputs import make_gate, make_inputs

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def _built():
    build.build()


def _dout(shape, dtype, seed):
    g = torch.Generator().manual_seed(seed)
    return torch.randn(*shape, generator=g).to(dtype)


def check_backward(q, k, v, beta, a, r, C, gate=None, seed=0, dout=None):
    if dout is None:
        dout = _dout(q.shape, q.dtype, 9000 + seed)
    dev = cuda(q, k, v, beta, dout)
    gd = gate.cuda() if gate is not None else None
    got = gka.gka_backward(dev[0], dev[1], dev[2], dev[3], dev[4], a, r, C, gate=gd)
    assert gka.device_status() == 0
    ref = oracle.backward(q, k, v, beta, dout, a, r, gate=gate)
    fp32 = q.dtype == torch.float32
    errs = {}
    for name in ref:
        bar = 1e-4 if fp32 else 2e-2
        errs[name] = head_rel_err(got[name], ref[name])
        assert np.all(np.isfinite(got[name].float().cpu().numpy())), name
        assert errs[name] <= bar, (name, errs[name], bar)
    print(" ".join(f"{n} {e:.2e}" for n, e in errs.items()))
    return got, ref


@pytest.mark.parametrize("D", [32, 64, 128])
@pytest.mark.parametrize("C", [16, 32])
def test_backward_fp32(D, C):
    q, k, v, beta = make_inputs(1, 2, 128, D, torch.float32, 2.0, 1.0, seed=800 + D + C)
    check_backward(q, k, v, beta, 0.5, 10, C, seed=D + C)


def test_backward_bf16_d128():
    # T = 128: the tensor-core forward supplies the iterates (4 heads: chunk increments)
    q, k, v, beta = make_inputs(1, 2, 128, 128, torch.bfloat16, 3.0, 1.0, seed=820)
    check_backward(q, k, v, beta, 0.5, 20, 32, seed=1)


def test_backward_bf16_d128_cuda_core_recompute():
    # T = 96 (not a multiple of 64): the CUDA-core forward supplies the iterates
    q, k, v, beta = make_inputs(1, 2, 96, 128, torch.bfloat16, 3.0, 1.0, seed=821)
    check_backward(q, k, v, beta, 0.5, 20, 32, seed=7)


def test_backward_bf16_state_pass_gate_resets():
    # 24 heads: the tensor-core forward's segmented states; a write gate, resets
    q, k, v, beta = make_inputs(1, 24, 128, 128, torch.bfloat16, 2.0, 1.0, seed=822)
    gate = make_gate((1, 24, 128), 822)
    gate[0, 3, 10:20] = 0.0
    beta[0, 5, 64] = 0.0
    check_backward(q, k, v, beta, 0.5, 20, 32, gate=gate, seed=8)


def test_backward_bf16_zero_upstream_gradient():
    # dL/do = 0: u, y, every adjoint (and its fp16 copy) and every intra-chunk product
    # vanish, so every gradient is exactly zero (all-zero tiles take the scale 1)
    q, k, v, beta = make_inputs(1, 4, 128, 128, torch.bfloat16, 3.0, 1.0, seed=823)
    gate = make_gate((1, 4, 128), 823)
    dev = cuda(q, k, v, beta)
    dout = torch.zeros_like(dev[0])
    got = gka.gka_backward(dev[0], dev[1], dev[2], dev[3], dout, 0.5, 20, 32, gate=gate.cuda())
    assert gka.device_status() == 0
    for name, t in got.items():
        assert torch.count_nonzero(t) == 0, name


def test_backward_bf16_gradient_in_last_chunk_only():
    # dL/do only on the last 32 tokens: the adjoints of every earlier chunk are what reaches
    # them from the last one, their own increments zero
    q, k, v, beta = make_inputs(1, 2, 256, 128, torch.bfloat16, 3.0, 1.0, seed=824)
    dout = _dout(q.shape, q.dtype, 9100)
    dout[:, :, :-32] = 0
    check_backward(q, k, v, beta, 0.5, 20, 32, dout=dout)


@pytest.mark.parametrize("D,C", [(64, 32), (128, 16), (32, 16)])
def test_backward_bf16_cuda_core_shapes(D, C):
    # bf16 inputs with D != 128 (all on CUDA cores), or D = 128 with chunk 16 (tensor-core
    # iterates and adjoint solve, the row products and increments on CUDA cores)
    q, k, v, beta = make_inputs(1, 2, 128, D, torch.bfloat16, 2.0, 1.0, seed=880 + D + C)
    check_backward(q, k, v, beta, 0.5, 12, C, seed=9 + D)


def test_backward_write_gate_and_resets():
    q, k, v, beta = make_inputs(1, 2, 128, 64, torch.float32, 1.0, 1.0, seed=830)
    gate = make_gate((1, 2, 128), 830)
    gate[0, 0, 0] = 0.0
    gate[0, 1, 40:48] = 0.0
    beta[0, 0, 32] = 0.0      # first token of a chunk
    beta[0, 1, 50] = 0.0      # inside a chunk
    check_backward(q, k, v, beta, 0.5, 10, 32, gate=gate, seed=2)


def test_backward_small_a_strong_forgetting():
    q, k, v, beta = make_inputs(1, 2, 96, 128, torch.float32, 0.0, 2.0, seed=840)
    check_backward(q, k, v, beta, 0.1, 30, 16, seed=3)


def test_backward_zero_keys_at_start():
    q, k, v, beta = make_inputs(1, 2, 64, 32, torch.float32, 2.0, 1.0, seed=850)
    k[0, 0, :3] = 0.0
    got, _ = check_backward(q, k, v, beta, 0.5, 8, 16, seed=4)
    assert torch.all(got["dq"][0, 0, :3] == 0)


def test_backward_chunk_size_invariance():
    q, k, v, beta = make_inputs(1, 2, 128, 64, torch.float32, 2.0, 1.0, seed=860)
    dout = _dout(q.shape, q.dtype, 5)
    dev = cuda(q, k, v, beta, dout)
    g16 = gka.gka_backward(*dev, 0.5, 10, 16)
    g32 = gka.gka_backward(*dev, 0.5, 10, 32)
    for n in g16:
        assert head_rel_err(g16[n], g32[n]) <= 1e-5, n


def test_backward_larger_bf16():
    q, k, v, beta = make_inputs(2, 4, 512, 128, torch.bfloat16, 3.0, 1.0, seed=870)
    check_backward(q, k, v, beta, 0.5, 20, 32, seed=6)


def test_backward_error_codes():
    q = torch.zeros(1, 1, 64, 64, device="cuda")
    beta = torch.ones(1, 1, 64, device="cuda")
    with pytest.raises(gka.GkaError) as e:
        gka.gka_backward(q, q, q, beta, q, 0.5, 4, 64)
    assert e.value.status == -2
    with pytest.raises(gka.GkaError) as e:
        gka.gka_backward(q[:, :, :48], q[:, :, :48], q[:, :, :48], beta[:, :, :48], q[:, :, :48],
                         0.5, 4, 32)
    assert e.value.status == -3


def test_backward_full_b8h8t2048_sampled():
    """The default forward workload (B8 H8 T2048 D128 bf16, a 0.5, r 20) through the
    backward in the benchmark's launch configuration (chunk 32); the oracle checks a
    sample of heads (heads are independent)."""
    from test_ridge_regression_b200.inputs import WORKLOADS, workload_inputs
    w = WORKLOADS["bf16_b8h8t2048d128"]
    q, k, v, beta = workload_inputs(w)
    dout = _dout(q.shape, q.dtype, 77)
    got = gka.gka_backward(*cuda(q, k, v, beta, dout), w.a, w.r, 32)
    assert gka.device_status() == 0
    got = {n: t.cpu() for n, t in got.items()}
    worst = {}
    for (b, h) in [(0, 0), (7, 7)]:
        sl = (slice(b, b + 1), slice(h, h + 1))
        ref = oracle.backward(q[sl], k[sl], v[sl], beta[sl], dout[sl], w.a, w.r, nthreads=1)
        for name in ref:
            e = head_rel_err(got[name][sl], ref[name])
            bar = 2e-2
            worst[name] = max(worst.get(name, 0.0), e)
            assert e <= bar, (name, b, h, e)
    print("full size sampled:", " ".join(f"{n} {e:.2e}" for n, e in worst.items()))
