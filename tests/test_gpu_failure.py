"""Failure reporting on the GPU without a fault: a bounded device wait that
gives up raises the library's device flag, gka_device_status() reports
GKA_ERR_DEVICE_TIMEOUT once, and the context keeps working."""
import pytest
import torch

from helpers import TOL, head_rel_err
from test_ridge_regression_b200 import build, gka
from test_ridge_regression_b200.inputs import make_inputs

pytestmark = pytest.mark.gpu


def test_bounded_wait_reports_timeout_and_context_survives():
    build.build()
    assert gka.device_status() == 0
    gka.selftest_timeout()
    assert gka.device_status() == -6          # GKA_ERR_DEVICE_TIMEOUT
    assert gka.device_status() == 0           # the flag was cleared
    # the context still runs the real path
    q, k, v, beta = (t.cuda() for t in make_inputs(1, 2, 128, 128, torch.bfloat16, 3.0, 1.0, 3))
    o1 = gka.gka_forward(q, k, v, beta, 0.5, 20, 64)
    o2 = gka.gka_forward(q, k, v, beta, 0.5, 20, 64)
    assert gka.device_status() == 0
    assert torch.equal(o1, o2)                # deterministic


def test_forward_is_deterministic_and_linear():
    # invariances of the method on the GPU path: linear in q and in v, k -> s k gives o / s
    q1, k, v1, beta = make_inputs(1, 2, 256, 128, torch.float32, 2.0, 1.0, 5)
    q2, _, v2, _ = make_inputs(1, 2, 256, 128, torch.float32, 2.0, 1.0, 6)
    f = lambda q, k, v: gka.gka_forward(q.cuda(), k.cuda(), v.cuda(), beta.cuda(), 0.5, 10,
                                        64).cpu()
    base = f(q1, k, v1)
    assert head_rel_err(f(2 * q1 + q2, k, v1), 2 * base + f(q2, k, v1)) <= TOL[torch.float32]
    assert head_rel_err(f(q1, k, -v1 + 3 * v2), -base + 3 * f(q1, k, v2)) <= TOL[torch.float32]
    assert head_rel_err(f(q1, 2 * k, v1), base / 2) <= TOL[torch.float32]
    # the same on the tensor-core path, at the bf16 bar
    qb, kb, vb, bb = make_inputs(1, 2, 256, 128, torch.bfloat16, 2.0, 1.0, 7)
    g = lambda q, k, v: gka.gka_forward(q.cuda(), k.cuda(), v.cuda(), bb.cuda(), 0.5, 20,
                                        64).float().cpu()
    gb = g(qb, kb, vb)
    assert head_rel_err(g(qb, (2 * kb.float()).to(torch.bfloat16), vb), gb / 2) <= TOL[torch.bfloat16]
    assert head_rel_err(g(qb, kb, (-vb.float()).to(torch.bfloat16)), -gb) <= TOL[torch.bfloat16]
