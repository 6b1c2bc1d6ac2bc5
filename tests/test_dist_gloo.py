"""Host logic of the multi-GPU benchmark path on CPU: world-size-2 gloo process
groups stand in for the NCCL ranks.  Each rank runs an independent replica
(the layer's EP ranks are logical, inside one GPU), so the only cross-rank step
is the max-over-ranks reduction of the timed region, plus the rank environment
and the whole-job token count."""
import os
import socket

import pytest
import torch.multiprocessing as mp


def _free_port():
    s = socket.socket()
    s.bind(("127.0.0.1", 0))
    p = s.getsockname()[1]
    s.close()
    return p


def _worker(rank, world, port, q):
    import torch.distributed as dist
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), RANK=str(rank),
                      WORLD_SIZE=str(world), LOCAL_RANK=str(rank))
    import sys
    sys.path.insert(0, os.path.dirname(os.path.dirname(os.path.abspath(__file__))))
    import bench
    from datetime import timedelta
    dist.init_process_group("gloo", rank=rank, world_size=world, timeout=timedelta(seconds=60))
    try:
        r, w, lr = bench.dist_env()
        got = bench.max_over_ranks(10.0 + 5.0 * rank)   # rank 1 is the slow one
        tokens = w * 4096 * 30                           # whole-job tokens of 30 steps
        q.put((r, w, lr, got, tokens / (got / 1e3)))
        dist.barrier()
    finally:
        dist.destroy_process_group()


def test_max_over_ranks_and_whole_job_value_gloo_world2():
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
    assert [r[:3] for r in res] == [(0, 2, 0), (1, 2, 1)]
    # both ranks see the slowest rank's time, and the value counts all ranks' tokens
    assert all(r[3] == 15.0 for r in res)
    assert all(abs(r[4] - 2 * 4096 * 30 / 0.015) < 1e-6 for r in res)


def test_max_over_ranks_without_process_group_is_identity():
    import bench
    assert bench.max_over_ranks(3.25) == 3.25
