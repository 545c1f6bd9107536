"""Tensor-parallel split of the decode GEMV over output rows.

The ROCM_OCTAVE page (vLLM PR #59774, tensor-parallel serving on four GPUs)
reports that at long context the GEMMs and the collective after them
dominate.  Split by output rows (N), the collective is an all-gather of y
rather than a sum: rank r of P holds a contiguous range of W's rows with
their d and m, computes its slice of y with the library's own GEMV on its
own GPU, and one all-gather over the process group assembles y [M][N] on
every rank.  No rank reads another rank's memory; NCCL (or gloo on the CPU)
moves the y slices.

Every rank holds the same number of rows, ``chunk`` (a multiple of 8, so that
each slice of a bf16 y starts on a 16-byte boundary); the last rank's range
is padded with zero rows (codes 0, d = m = 0, which give y = 0), so every
slice has the same shape and the gather needs no per-rank sizes.
"""
from __future__ import annotations

from typing import Callable, Optional

__all__ = ["shard_rows", "ShardedW4Linear"]

ALIGN = 8


def shard_rows(N: int, world: int, rank: int, align: int = ALIGN):
    """(n0, n1, chunk): this rank's rows [n0, n1) of N and the padded width
    every rank's slice has.  Ranges are contiguous, in rank order, and cover
    [0, N) exactly once."""
    if world < 1 or not 0 <= rank < world:
        raise ValueError("need 0 <= rank < world")
    chunk = -(-N // world)
    chunk = -(-chunk // align) * align
    n0 = min(N, rank * chunk)
    n1 = min(N, n0 + chunk)
    return n0, n1, chunk


class ShardedW4Linear:
    """One W4-G256 weight matrix split over the ranks of ``group`` by rows.

    codes [N][K/2], d and m [N][K/256]: the full planes (any device); each
    rank keeps its own rows, padded to ``chunk``, on ``device``.
    ``gemv(codes, d, m, x, out_dtype)`` computes the local slice (default: the
    library's w4_gemv on the current CUDA device); a CPU test passes its own.
    """

    def __init__(self, codes, d, m, group=None, device=None,
                 gemv: Optional[Callable] = None):
        import torch
        import torch.distributed as dist
        self.group = group
        self.world = dist.get_world_size(group) if dist.is_initialized() else 1
        self.rank = dist.get_rank(group) if dist.is_initialized() else 0
        self.N = int(codes.shape[0])
        self.K = int(codes.shape[1]) * 2
        n0, n1, chunk = shard_rows(self.N, self.world, self.rank)
        self.n0, self.n1, self.chunk = n0, n1, chunk
        device = device if device is not None else codes.device

        def rows(plane):
            out = torch.zeros((chunk,) + tuple(plane.shape[1:]), dtype=plane.dtype,
                              device=device)
            out[: n1 - n0] = plane[n0:n1].to(device)
            return out

        self.codes, self.d, self.m = rows(codes), rows(d), rows(m)
        if gemv is None:
            from . import w4_gemv as gemv
        self._gemv = gemv

    def forward(self, x, out_dtype=None):
        """y [M][N] on every rank: the local slice, then one all-gather."""
        import torch
        import torch.distributed as dist
        y_local = self._gemv(self.codes, self.d, self.m, x, out_dtype)
        M = y_local.shape[0]
        if self.world == 1:
            return y_local[:, : self.N]
        gathered = torch.empty((self.world * M, self.chunk), dtype=y_local.dtype,
                               device=y_local.device)
        dist.all_gather_into_tensor(gathered, y_local.contiguous(), group=self.group)
        # [P * M][chunk] = [P][M][chunk] -> [M][P * chunk]: rank r's slice holds
        # output rows r * chunk ... r * chunk + chunk - 1
        y = gathered.view(self.world, M, self.chunk).permute(1, 0, 2).reshape(
            M, self.world * self.chunk)
        return y[:, : self.N]

    __call__ = forward
