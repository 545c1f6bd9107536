"""The tensor-parallel row split of the decode GEMV (w4_quant_matmul_b200.tp)
on the CPU with two gloo ranks: each rank's slice comes from the oracle's GEMV
on that rank's rows only, and the all-gather must assemble exactly the full
oracle product, in row order, on every rank.  No GPU involved: this checks
the partitioning, the padding of the last shard and the gather order."""
import os
import socket

import numpy as np
import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp

from w4_quant_matmul_b200.tp import shard_rows


def _free_port() -> int:
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


@pytest.mark.parametrize("N,world", [(1, 2), (300, 2), (151936, 4), (17, 3), (8, 8), (9, 8)])
def test_shards_cover_the_rows_once(N, world):
    seen = np.zeros(N, np.int64)
    chunks = set()
    for r in range(world):
        n0, n1, chunk = shard_rows(N, world, r)
        assert 0 <= n0 <= n1 <= N and n1 - n0 <= chunk and chunk % 8 == 0
        seen[n0:n1] += 1
        chunks.add(chunk)
        if r > 0:
            assert n0 == min(N, shard_rows(N, world, r - 1)[1])  # contiguous, rank order
    assert np.all(seen == 1) and len(chunks) == 1


def _oracle_gemv(codes, d, m, x, out_dtype=None):
    import oracle
    y = oracle.get().gemv(codes.numpy(), d.numpy().view(np.uint16), m.numpy().view(np.uint16),
                          x.numpy().view(np.uint16))
    return torch.from_numpy(np.ascontiguousarray(y))


def _worker(rank, world, port, N, K, M, out):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    import synth
    from w4_quant_matmul_b200.tp import ShardedW4Linear
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        codes, d, m = synth.quantized_weights_direct(N, K, seed=21)
        x = synth.activations(M, K, seed=22)
        lin = ShardedW4Linear(torch.from_numpy(codes), torch.from_numpy(d.view(np.int16)),
                              torch.from_numpy(m.view(np.int16)), device="cpu",
                              gemv=_oracle_gemv)
        y = lin(torch.from_numpy(x.view(np.int16)))
        out[rank] = y.numpy().tobytes(), y.shape
    finally:
        dist.destroy_process_group()


@pytest.mark.parametrize("N,K,M", [(300, 512, 3), (37, 256, 1)])
def test_row_split_gathers_the_full_product(N, K, M):
    import oracle
    import synth
    world = 2
    port = _free_port()
    ctx = mp.get_context("spawn")
    with ctx.Manager() as mgr:
        out = mgr.dict()
        procs = [ctx.Process(target=_worker, args=(r, world, port, N, K, M, out))
                 for r in range(world)]
        for p in procs:
            p.start()
        for p in procs:
            p.join(timeout=120)
            assert p.exitcode == 0
        codes, d, m = synth.quantized_weights_direct(N, K, seed=21)
        x = synth.activations(M, K, seed=22)
        want = oracle.get().gemv(codes, d, m, x)
        for r in range(world):
            buf, shape = out[r]
            got = np.frombuffer(buf, dtype=np.float64).reshape(shape)
            assert got.shape == (M, N)
            assert np.array_equal(got, want), r
