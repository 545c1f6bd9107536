"""The multi-process plumbing of bench.py on CPU: two gloo ranks, the
timed region reduced as max over ranks and the work as a sum (replicas,
weak scaling).  No GPU involved."""
import os
import socket

import pytest
import torch.distributed as dist
import torch.multiprocessing as mp


def _free_port() -> int:
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _worker(rank, world, port, out):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port),
                      RANK=str(rank), WORLD_SIZE=str(world), LOCAL_RANK=str(rank))
    import bench
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        assert bench.dist_env() == (world, rank, rank)
        elapsed = 0.5 + rank            # rank 1 is the slow one
        units = 1000.0 * (rank + 1)
        t, u = bench.reduce_timing(elapsed, units)
        bench.barrier()
        out[rank] = (t, u)
    finally:
        dist.destroy_process_group()


def test_reduce_timing_two_ranks():
    world = 2
    port = _free_port()
    ctx = mp.get_context("spawn")
    with ctx.Manager() as mgr:
        out = mgr.dict()
        procs = [ctx.Process(target=_worker, args=(r, world, port, out)) for r in range(world)]
        for p in procs:
            p.start()
        for p in procs:
            p.join(timeout=120)
            assert p.exitcode == 0
        for r in range(world):
            t, u = out[r]
            assert t == pytest.approx(1.5)      # max over ranks
            assert u == pytest.approx(3000.0)   # sum over ranks


def test_reduce_timing_single_process_is_identity():
    import bench
    assert bench.reduce_timing(0.25, 7.0) == (0.25, 7.0)
