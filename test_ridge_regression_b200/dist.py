"""Multi-process plumbing for running the layer on several GPUs of one node.

The (batch, head) recurrences are independent, so the path shards by batch
with no exchange step: every rank runs its own batch on its own GPU (weak
scaling).  The only collective is the end-of-run reduction of timings (the
slowest rank defines the job's time).  torch.distributed is used as plumbing
(NCCL between GPUs, gloo on CPU).
"""
from __future__ import annotations

import os
from datetime import timedelta


def rank_env():
    """(rank, world_size, local_rank) from the torchrun environment (defaults 0, 1, 0)."""
    return (int(os.environ.get("RANK", "0")), int(os.environ.get("WORLD_SIZE", "1")),
            int(os.environ.get("LOCAL_RANK", "0")))


def shard_seed(seed: int, rank: int) -> int:
    """Seed of rank `rank`'s batch: distinct, reproducible data per rank."""
    return seed + 1_000_003 * rank


def init(backend: str, timeout_s: float = 120.0, device=None):
    """Initialise the default process group (rendezvous on 127.0.0.1 unless set)."""
    import torch.distributed as dist
    os.environ.setdefault("MASTER_ADDR", "127.0.0.1")
    kw = {"timeout": timedelta(seconds=timeout_s)}
    if device is not None:
        kw["device_id"] = device
    dist.init_process_group(backend, **kw)


def max_over_ranks(value: float, device=None) -> float:
    """Maximum of `value` over all ranks (identity without a process group)."""
    import torch
    import torch.distributed as dist
    if not (dist.is_available() and dist.is_initialized()) or dist.get_world_size() == 1:
        return float(value)
    t = torch.tensor([float(value)], dtype=torch.float64, device=device or "cpu")
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())
