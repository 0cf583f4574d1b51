"""Seeded synthetic inputs shared by the CUDA path's tests, the oracle's tests
and the benchmark.  This module holds no arithmetic of the layer itself: it
only draws random numbers and shapes them like the workloads of the Gated
KalmaNet paper (random regression with B=8, T=2048, 8 heads, head dim 128 in
the solver study of Fig. 1; 8 heads, head dim 128 in the runtime study of
Fig. 3b; contexts up to 128k tokens in Fig. 4).

Recipe: q, k ~ N(0, 1), l2-normalised per token in fp32 (the block applies an
l2 norm before the layer, Fig. 2 of the paper), then cast to the compute
dtype; v ~ N(0, 1) cast to the dtype; beta = sigmoid(N(mu, sigma)) in fp32.
All draws come from one torch CPU generator seeded per workload, in the order
q, k, v, beta.

Write gate (the paper's beta_t-augmented variant; ai.info page, Main Findings):
g = sigmoid(N(mu, sigma)) in fp32, mu = 0 and sigma = 1.5 by default (the pages
give no distribution for the learned gate; this spreads it over (0, 1) around
1/2), from its own generator seeded with the workload seed + 1_000_000, so the
other inputs do not change when a gate is drawn.
"""
from __future__ import annotations

from dataclasses import dataclass

import torch


@dataclass(frozen=True)
class Workload:
    name: str
    B: int
    H: int
    T: int
    D: int
    chunk: int
    a: float
    r: int
    dtype: torch.dtype
    beta_mu: float
    beta_sigma: float
    seed: int


# The forward workloads, named by their shapes.
WORKLOADS = {
    w.name: w
    for w in [
        Workload("tiny_fp32_b1h2t256d32", 1, 2, 256, 32, 64, 0.5, 10, torch.float32, 2.0, 0.5, 1),
        Workload("bf16_b8h8t2048d128", 8, 8, 2048, 128, 64, 0.5, 20, torch.bfloat16, 3.0, 1.0, 2),
        Workload("bf16_b4h16t8192d128_a0.1", 4, 16, 8192, 128, 64, 0.1, 30, torch.bfloat16, 1.0, 1.0, 3),
        Workload("bf16_b1h8t131072d128", 1, 8, 131072, 128, 128, 0.5, 20, torch.bfloat16, 4.0, 1.0, 4),
    ]
}


@dataclass(frozen=True)
class DecodeWorkload:
    name: str
    batch: int
    H: int
    D: int
    a: float
    r: int
    prefill: int
    steps: int
    beta_mu: float
    beta_sigma: float
    seed: int


DECODE = DecodeWorkload("decode_bf16_b256h32d128", 256, 32, 128, 0.5, 20, 512, 1024, 3.0, 1.0, 5)


def _gen(seed: int) -> torch.Generator:
    g = torch.Generator(device="cpu")
    g.manual_seed(seed)
    return g


def _unit_rows(x: torch.Tensor) -> torch.Tensor:
    # per-token l2 normalisation in fp32 (input preparation, not the layer)
    return x / x.norm(dim=-1, keepdim=True).clamp_min(1e-30)


def make_inputs(B: int, H: int, T: int, D: int, dtype: torch.dtype, beta_mu: float,
                beta_sigma: float, seed: int):
    """q, k, v: [B, H, T, D] in ``dtype``; beta: [B, H, T] fp32.  CPU tensors."""
    g = _gen(seed)
    q = _unit_rows(torch.randn(B, H, T, D, generator=g, dtype=torch.float32)).to(dtype)
    k = _unit_rows(torch.randn(B, H, T, D, generator=g, dtype=torch.float32)).to(dtype)
    v = torch.randn(B, H, T, D, generator=g, dtype=torch.float32).to(dtype)
    beta = torch.sigmoid(beta_mu + beta_sigma * torch.randn(B, H, T, generator=g,
                                                            dtype=torch.float32))
    return q.contiguous(), k.contiguous(), v.contiguous(), beta.contiguous()


def make_gate(shape, seed: int, mu: float = 0.0, sigma: float = 1.5) -> torch.Tensor:
    """Write gate in (0, 1), fp32 CPU tensor of ``shape`` ([B, H, T] or [B, H])."""
    g = _gen(seed + 1_000_000)
    return torch.sigmoid(mu + sigma * torch.randn(*shape, generator=g,
                                                  dtype=torch.float32)).contiguous()


def workload_inputs(w: Workload, *, B: int | None = None, H: int | None = None,
                    T: int | None = None):
    """Inputs of a named workload, optionally with a smaller B, H or T (the same
    distributions and seed)."""
    return make_inputs(B or w.B, H or w.H, T or w.T, w.D, w.dtype, w.beta_mu,
                       w.beta_sigma, w.seed)


def decode_prefill_inputs(w: DecodeWorkload, batch: int | None = None, H: int | None = None,
                          dtype: torch.dtype = torch.bfloat16):
    """The prefill sequence that builds the decode state: [b, H, prefill, D]."""
    return make_inputs(batch or w.batch, H or w.H, w.prefill, w.D, dtype, w.beta_mu,
                       w.beta_sigma, w.seed)


def decode_step_inputs(w: DecodeWorkload, step: int, batch: int | None = None,
                       H: int | None = None, dtype: torch.dtype = torch.bfloat16):
    """Fresh single-token inputs of decode step ``step``: q, k, v [b, H, D], beta [b, H]."""
    q, k, v, beta = make_inputs(batch or w.batch, H or w.H, 1, w.D, dtype, w.beta_mu,
                                w.beta_sigma, w.seed * 1_000_003 + 7919 * (step + 1))
    return q[:, :, 0].contiguous(), k[:, :, 0].contiguous(), v[:, :, 0].contiguous(), \
        beta[:, :, 0].contiguous()
