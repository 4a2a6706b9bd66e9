"""Process-group helpers for running the path on several GPUs.

Rows (and whole matrices) are independent -- the scale is per row and the
Hadamard transform stays inside a row -- so work is split by rows with no
data-path collective.  The only collective is the timing reduction.
"""
from __future__ import annotations

import os


def rank_info():
    """(rank, world_size, local_rank) from the launcher's environment."""
    return (int(os.environ.get("RANK", "0")), int(os.environ.get("WORLD_SIZE", "1")),
            int(os.environ.get("LOCAL_RANK", "0")))


def shard_rows(rows: int, world: int, rank: int):
    """Contiguous row range [start, stop) of this rank; sizes differ by at most one."""
    base, extra = divmod(rows, world)
    start = rank * base + min(rank, extra)
    return start, start + base + (1 if rank < extra else 0)


def max_over_ranks(value: float, device=None) -> float:
    """Maximum of a per-rank float over the default process group."""
    import torch
    import torch.distributed as dist

    if not dist.is_available() or not dist.is_initialized() or dist.get_world_size() == 1:
        return float(value)
    t = torch.tensor([float(value)], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())
