"""Multi-GPU plumbing for the W4A4 layer: token sharding and device timing.

The layer shards by tokens with no exchange: every token's activation scale
is computed from its own row, and the quantized weights are replicated, so
rank r can run rows [start, start + count) of the batch on its own GPU and
the concatenation of the ranks' outputs is the single-GPU output, bit for
bit.  Nothing here moves tensor data between GPUs; torch.distributed is used
only for the timing reduction (max over ranks) and barriers.
"""
from __future__ import annotations

import os


def token_shard(m_total: int, world: int, rank: int) -> tuple[int, int]:
    """Contiguous, balanced split of m_total tokens: (start, count) of `rank`."""
    if world < 1 or not 0 <= rank < world or m_total < 0:
        raise ValueError("bad shard request")
    base, extra = divmod(m_total, world)
    start = rank * base + min(rank, extra)
    return start, base + (1 if rank < extra else 0)


def dist_env() -> tuple[int, int, int]:
    """(rank, world_size, local_rank) from the torchrun environment (1 process by default)."""
    return (int(os.environ.get("RANK", "0")), int(os.environ.get("WORLD_SIZE", "1")),
            int(os.environ.get("LOCAL_RANK", "0")))


def max_over_ranks(value: float, device=None) -> float:
    """Largest value over all ranks (identity without an initialised process group)."""
    import torch
    import torch.distributed as dist
    if not (dist.is_available() and dist.is_initialized()) or dist.get_world_size() == 1:
        return float(value)
    t = torch.tensor([float(value)], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())
