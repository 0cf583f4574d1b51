"""GPU parity of gka_decode_step (through the C ABI) against the float64
oracle.  Both sides start from the same fp32 state (the oracle's prefill state
rounded to fp32) and see the same seeded single-token inputs."""
import numpy as np
import pytest
import torch

import oracle
from helpers import TOL, f64, head_rel_err
from test_ridge_regression_b200 import build, gka
from test_ridge_regression_b200.inputs import DECODE, decode_prefill_inputs, decode_step_inputs, make_inputs

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def _built():
    build.build()


def oracle_prefill_state(batch, H, D, dtype, prefill, seed):
    q, k, v, beta = make_inputs(batch, H, prefill, D, dtype, 3.0, 1.0, seed)
    st = oracle.forward(q, k, v, beta, 0.5, 1, solve_from=prefill, want_final_state=True)
    return torch.from_numpy(st["final_state"]).float()   # fp32 start state for both sides


@pytest.mark.parametrize("D,dtype", [(32, torch.float32), (64, torch.float32),
                                     (128, torch.float32), (128, torch.bfloat16)])
def test_decode_steps_small(D, dtype):
    batch, H, steps, a, r = 3, 4, 6, 0.5, 20
    st0 = oracle_prefill_state(batch, H, D, dtype, 64, seed=D)
    st_gpu = st0.cuda()
    st_ref = f64(st0)
    outs_gpu, outs_ref = [], []
    for s in range(steps):
        q, k, v, beta = make_inputs(batch, H, 1, D, dtype, 3.0, 1.0, seed=1000 + 17 * s + D)
        q, k, v, beta = q[:, :, 0], k[:, :, 0], v[:, :, 0], beta[:, :, 0]
        o = gka.gka_decode_step(st_gpu, q.cuda(), k.cuda(), v.cuda(), beta.cuda(), a, r)
        o_ref, st_ref = oracle.decode_step(st_ref, q, k, v, beta, a, r)
        outs_gpu.append(o.cpu())
        outs_ref.append(o_ref)
    assert gka.device_status() == 0
    og = torch.stack(outs_gpu, dim=2)
    orf = np.stack(outs_ref, axis=2)
    err = head_rel_err(og, orf)
    print(f"decode D={D} {dtype}: o rel err {err:.3e}")
    assert err <= TOL[dtype]
    assert head_rel_err(st_gpu, st_ref) <= 1e-5


def test_decode_zero_state_first_token():
    # from a zero state the first step is the first-token closed form of the oracle
    batch, H, D = 2, 2, 128
    st = torch.zeros(batch, H, 2, D, D, device="cuda")
    q, k, v, beta = make_inputs(batch, H, 1, D, torch.float32, 3.0, 1.0, seed=5)
    q, k, v, beta = q[:, :, 0], k[:, :, 0], v[:, :, 0], beta[:, :, 0]
    o = gka.gka_decode_step(st, q.cuda(), k.cuda(), v.cuda(), beta.cuda(), 0.5, 20)
    o_ref, _ = oracle.decode_step(np.zeros((batch, H, 2, D, D)), q, k, v, beta, 0.5, 20)
    assert head_rel_err(o, o_ref) <= 1e-4


def test_decode_zero_key_gives_zero_output():
    batch, H, D = 1, 2, 64
    st = torch.zeros(batch, H, 2, D, D, device="cuda")
    z = torch.zeros(batch, H, D, device="cuda")
    v = torch.ones(batch, H, D, device="cuda")
    o = gka.gka_decode_step(st, z + 1, z, v, torch.ones(batch, H, device="cuda"), 0.5, 5)
    assert gka.device_status() == 0
    assert torch.all(o == 0) and torch.all(torch.isfinite(st))


def test_decode_full_size_sampled():
    """All 256 x 32 heads in the benchmark's launch configuration.  The start
    state of every head is an oracle prefill state (8 x 32 distinct heads,
    tiled along the batch); the oracle checks a sample of heads over 3 steps."""
    w = DECODE
    base_b = 8
    base = oracle_prefill_state(base_b, w.H, w.D, torch.bfloat16, w.prefill, seed=w.seed)
    st_gpu = base.repeat(w.batch // base_b, 1, 1, 1, 1).contiguous().cuda()
    sample = [(0, 0), (255, 31), (100, 7), (17, 20)]
    st_ref = {bh: f64(base[bh[0] % base_b, bh[1]])[None, None] for bh in sample}
    worst = 0.0
    for s in range(3):
        q, k, v, beta = decode_step_inputs(w, s)
        o = gka.gka_decode_step(st_gpu, q.cuda(), k.cuda(), v.cuda(), beta.cuda(), w.a, w.r).cpu()
        for (b, h) in sample:
            o_ref, st_ref[(b, h)] = oracle.decode_step(
                st_ref[(b, h)], q[b:b + 1, h:h + 1], k[b:b + 1, h:h + 1], v[b:b + 1, h:h + 1],
                beta[b:b + 1, h:h + 1], w.a, w.r)
            worst = max(worst, head_rel_err(o[b:b + 1, h:h + 1], o_ref))
    assert gka.device_status() == 0
    for (b, h) in sample:
        assert head_rel_err(st_gpu[b:b + 1, h:h + 1], st_ref[(b, h)]) <= 1e-5
    print(f"decode full size: sampled o rel err {worst:.3e}")
    assert worst <= TOL[torch.bfloat16]


def test_forward_final_state_feeds_decode():
    """Prefill through gka_forward, continue with gka_decode_step; the oracle runs
    the same token stream in one recurrence."""
    B, H, T, D, a, r = 1, 2, 128, 128, 0.5, 20
    q, k, v, beta = make_inputs(B, H, T + 2, D, torch.bfloat16, 3.0, 1.0, seed=9)
    ws = gka.alloc_workspace(B, H, T, D, 64, torch.bfloat16)
    st = torch.empty(B, H, 2, D, D, device="cuda")
    gka.gka_forward(q[:, :, :T].contiguous().cuda(), k[:, :, :T].contiguous().cuda(),
                    v[:, :, :T].contiguous().cuda(), beta[:, :, :T].contiguous().cuda(), a, r, 64,
                    final_state=st, workspace=ws)
    outs = []
    for t in (T, T + 1):
        outs.append(gka.gka_decode_step(st, q[:, :, t].contiguous().cuda(),
                                        k[:, :, t].contiguous().cuda(),
                                        v[:, :, t].contiguous().cuda(),
                                        beta[:, :, t].contiguous().cuda(), a, r).cpu())
    ref = oracle.forward(q, k, v, beta, a, r, solve_from=T)["o"][:, :, T:]
    assert head_rel_err(torch.stack(outs, dim=2), ref) <= TOL[torch.bfloat16]
