"""A matrix split by output rows over the ranks of a process group.

The path itself needs no exchange: each GPU decodes and multiplies its own
rows.  When a caller wants the whole y on every rank (a row-parallel layer
followed by a replicated one), one all-gather of y moves 4·batch·rows bytes,
tiny next to the weights.  Each rank compresses its own rows, so every shard
has its own code table (the decoder never looks outside its matrix).  Shards
are whole 8-row tile blocks, as equal as that allows.

Every rank runs the library's kernels on its shard; the gather is
torch.distributed's (NCCL on GPUs, gloo in the CPU tests).
"""
from __future__ import annotations

from typing import Callable

import numpy as np

TILE_ROWS = 8


def row_ranges(rows: int, world: int) -> list[tuple[int, int]]:
    """[start, end) of each rank's rows: whole 8-row blocks, as equal as
    possible, earlier ranks taking the extra block; a rank may get none."""
    if rows < 1 or world < 1:
        raise ValueError("rows and world must be positive")
    blocks = -(-rows // TILE_ROWS)
    out, b0 = [], 0
    for r in range(world):
        nb = blocks // world + (1 if r < blocks % world else 0)
        start, end = min(b0 * TILE_ROWS, rows), min((b0 + nb) * TILE_ROWS, rows)
        out.append((start, end))
        b0 += nb
    return out


class ShardedMatrix:
    """This rank's rows of W, compressed; gemv returns the whole y on every rank.

    `local` is this rank's CompressedMatrix (None when it has no rows).
    `group` is a torch.distributed process group, or None for a single
    process (world 1, no collective)."""

    def __init__(self, local, ranges: list[tuple[int, int]], rank: int, group=None,
                 gather: Callable | None = None):
        self.local = local
        self.ranges = ranges
        self.rank = rank
        self.group = group
        self.rows = ranges[-1][1]
        self.world = len(ranges)
        self._gather = gather

    @classmethod
    def compress(cls, w_host: np.ndarray, group=None, device="cuda", compress=None, **kw):
        """Every rank calls this with the whole W (or at least its rows); rank r
        keeps rows ranges[r].  kw goes to CompressedMatrix.compress."""
        rank, world = _rank_world(group)
        w_host = np.ascontiguousarray(w_host, dtype=np.uint16)
        ranges = row_ranges(w_host.shape[0], world)
        start, end = ranges[rank]
        if compress is None:
            from ._lib import CompressedMatrix
            compress = CompressedMatrix.compress
        local = compress(np.ascontiguousarray(w_host[start:end]), device=device, **kw) \
            if end > start else None
        return cls(local, ranges, rank, group)

    def gemv(self, x, local_gemv: Callable | None = None):
        """y = x @ W^T as FP32 [batch, rows] on every rank: the local rows, then
        one all-gather (padded to the largest shard, then trimmed)."""
        import torch
        batch = x.reshape(-1, x.shape[-1]).shape[0]
        width = max(e - s for s, e in self.ranges)
        mine = self.ranges[self.rank][1] - self.ranges[self.rank][0]
        part = torch.zeros((batch, width), dtype=torch.float32, device=x.device)
        if mine:
            y_local = local_gemv(x) if local_gemv is not None else self.local.gemv(x)
            part[:, :mine] = y_local
        if self.world == 1:
            return part[:, :self.rows].contiguous()
        gathered = torch.empty((self.world, batch, width), dtype=torch.float32, device=x.device)
        gather = self._gather or _all_gather
        gather(gathered, part, self.group)
        if batch == 1 and all(e - s == width for s, e in self.ranges):
            # One row of x and equal shards: the gathered rows are y, in order.
            return gathered.view(1, self.world * width)
        return torch.cat([gathered[r, :, :e - s] for r, (s, e) in enumerate(self.ranges)], dim=1)

    def close(self) -> None:
        if self.local is not None:
            self.local.close()


def _rank_world(group) -> tuple[int, int]:
    import torch.distributed as dist
    if group is None and not (dist.is_available() and dist.is_initialized()):
        return 0, 1
    return dist.get_rank(group), dist.get_world_size(group)


def _all_gather(out, part, group) -> None:
    import torch.distributed as dist
    dist.all_gather_into_tensor(out.view(-1), part.contiguous().view(-1), group=group)
