"""The multi-GPU path's host logic on CPU: two gloo ranks, each with its own
batch seed, agree on the job time as the maximum over ranks."""
import os
import socket

import pytest
import torch.multiprocessing as mp


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _worker(rank, world, port, out):
    os.environ.update({"RANK": str(rank), "WORLD_SIZE": str(world), "LOCAL_RANK": str(rank),
                       "MASTER_ADDR": "127.0.0.1", "MASTER_PORT": str(port)})
    import torch.distributed as dist
    from test_ridge_regression_b200 import dist as gdist
    r, w, lr = gdist.rank_env()
    gdist.init("gloo", timeout_s=60)
    t = gdist.max_over_ranks(10.0 * (r + 1))
    out.put((r, w, lr, gdist.shard_seed(2, r), t))
    dist.barrier()
    dist.destroy_process_group()


def test_two_gloo_ranks_reduce_max_and_shard_seeds():
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_worker, args=(r, 2, port, q)) for r in range(2)]
    for p in procs:
        p.start()
    res = sorted(q.get(timeout=120) for _ in procs)
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    assert [x[0] for x in res] == [0, 1]
    assert all(x[1] == 2 for x in res)
    assert all(x[4] == 20.0 for x in res)          # max over ranks
    assert res[0][3] != res[1][3]                  # distinct batches per rank


def test_single_process_defaults():
    from test_ridge_regression_b200 import dist as gdist
    assert gdist.max_over_ranks(3.5) == 3.5
    assert gdist.shard_seed(7, 0) == 7
