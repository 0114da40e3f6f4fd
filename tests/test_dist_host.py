"""The multi-process plumbing of bench.py on CPU: two gloo ranks (the path
the benchmark takes under torchrun, with NCCL, on N GPUs).  The forward has
no exchange step (replicas only), so what is checked is the timing
reduction: the max over ranks, the barrier, and the whole-job value."""

import os
import socket
import sys

import pytest
import torch.multiprocessing as mp

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _free_port():
    s = socket.socket()
    s.bind(("127.0.0.1", 0))
    p = s.getsockname()[1]
    s.close()
    return p


def _rank_main(rank, world, port, out):
    os.environ.update({"RANK": str(rank), "WORLD_SIZE": str(world), "LOCAL_RANK": str(rank),
                       "MASTER_ADDR": "127.0.0.1", "MASTER_PORT": str(port)})
    sys.path.insert(0, ROOT)
    import bench
    ctx = bench.DistCtx(world, backend="gloo")
    ctx.barrier()
    ms = ctx.max(10.0 + 5.0 * rank)          # rank r "took" 10 + 5r ms
    out[rank] = (ms, bench.replica_value(100.0, ctx.world, ms))
    ctx.close()


def test_two_gloo_ranks_time_as_the_slowest():
    world = 2
    port = _free_port()
    ctx = mp.get_context("spawn")
    with ctx.Manager() as m:
        out = m.dict()
        procs = [ctx.Process(target=_rank_main, args=(r, world, port, out)) for r in range(world)]
        for p in procs:
            p.start()
        for p in procs:
            p.join(120)
            assert p.exitcode == 0
        res = dict(out)
    for r in range(world):
        ms, value = res[r]
        assert ms == 15.0                      # the max over ranks, on every rank
        assert value == pytest.approx(2 * 100.0 / 0.015)


def test_single_process_needs_no_process_group():
    sys.path.insert(0, ROOT)
    import bench
    os.environ.pop("WORLD_SIZE", None)
    ctx = bench.DistCtx(1, backend="gloo")
    assert ctx.max(3.5) == 3.5 and ctx.dist is None
    ctx.barrier()
    ctx.close()
