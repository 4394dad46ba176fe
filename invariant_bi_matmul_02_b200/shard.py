"""Row sharding for running the path on several GPUs, one process per GPU.

Rows are independent units of the path: a row's bits do not depend on which
other rows share its batch, so a global batch can be split across GPUs by rows
with no collective on the data path.  Every rank holds a replica of the weights.
The only collective is the timing reduction (the maximum over ranks).
"""
from __future__ import annotations


def shard_rows(total_rows: int, world: int, rank: int) -> tuple[int, int]:
    """Contiguous, balanced [start, stop) of `total_rows` rows for `rank` of `world`.

    The first (total_rows % world) ranks take one extra row; every row belongs to
    exactly one rank and ranks keep the global row order.
    """
    if world < 1 or not 0 <= rank < world or total_rows < 0:
        raise ValueError("bad shard arguments")
    base, extra = divmod(total_rows, world)
    start = rank * base + min(rank, extra)
    return start, start + base + (1 if rank < extra else 0)


def weak_rows(rows_per_rank: int, rank: int) -> tuple[int, int]:
    """Rows of `rank` when every rank processes the same number of rows (weak scaling)."""
    if rows_per_rank < 0 or rank < 0:
        raise ValueError("bad shard arguments")
    return rank * rows_per_rank, (rank + 1) * rows_per_rank


def max_over_ranks(value: float, device=None) -> float:
    """Maximum of a per-rank scalar over the default process group (value itself if none)."""
    import torch
    import torch.distributed as dist
    if not (dist.is_available() and dist.is_initialized()) or dist.get_world_size() == 1:
        return float(value)
    t = torch.tensor([float(value)], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())
