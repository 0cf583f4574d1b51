"""Shared helpers of the GPU parity tests (comparison metric and tolerances).

Error metric: for every (batch, head), ||o_gpu - o_ref||_F / ||o_ref||_F over
that head's [T, D] slab, in float64; the test takes the maximum over heads.
Tolerances: 1e-4 for fp32 inputs; 2e-2 for bf16 inputs with fp32 accumulation.
"""
import numpy as np
import torch

TOL = {torch.float32: 1e-4, torch.bfloat16: 2e-2}


def f64(t):
    if isinstance(t, torch.Tensor):
        return t.detach().to("cpu").double().numpy()
    return np.asarray(t, dtype=np.float64)


def head_rel_err(got, ref, head_dims=2):
    """Max over leading `head_dims` axes of the relative Frobenius error."""
    g, r = f64(got), f64(ref)
    assert g.shape == r.shape, (g.shape, r.shape)
    lead = g.shape[:head_dims]
    g = g.reshape(int(np.prod(lead)), -1)
    r = r.reshape(int(np.prod(lead)), -1)
    num = np.linalg.norm(g - r, axis=1)
    den = np.linalg.norm(r, axis=1)
    den = np.where(den == 0, 1.0, den)
    return float((num / den).max())


def cuda(*ts):
    return [t.cuda() for t in ts]
