"""Host logic of the replicas-only multi-GPU bench, on two gloo ranks (CPU):
the barrier, the max-over-ranks timing and the whole-job aggregate."""

import os
import socket

import pytest
import torch.multiprocessing as mp

import bench


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _worker(rank, world, port, q):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), WORLD_SIZE=str(world),
                      RANK=str(rank), LOCAL_RANK=str(rank))
    ctx = bench.DistCtx()
    ctx.init("gloo")
    ctx.barrier()
    t = [1.5, 2.5][rank]  # rank 1 is the slower replica
    m = ctx.max(t)
    v = bench.aggregate_value(5120, ctx.world, m)
    ctx.barrier()
    ctx.close()
    q.put((rank, m, v))


def test_two_rank_max_and_aggregate():
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_worker, args=(r, 2, port, q)) for r in range(2)]
    for p in procs:
        p.start()
    out = sorted(q.get(timeout=120) for _ in procs)
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    for rank, m, v in out:
        assert m == 2.5
        assert v == pytest.approx(5120 * 2 / 2.5)


def test_single_process_context_is_inert():
    ctx = bench.DistCtx()
    assert ctx.world == int(os.environ.get("WORLD_SIZE", "1"))
    if ctx.world == 1:
        ctx.barrier()
        assert ctx.max(3.0) == 3.0
