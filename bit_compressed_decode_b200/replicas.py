"""Independent replicas over GPUs: one process per GPU, each decoding its own shard of
the block's sequences.

Decode rows are independent ("FlexGen Guide", section 2: a GPU batch of sequences goes
through the loaded layer on its own), so the block splits across GPUs with no
collective on the data path: each rank holds a replica of the (4-bit) weights and the
KV cache of its own sequences.  torch.distributed only carries the timing reduction.
"""
from __future__ import annotations

import datetime
import os


def shard(total: int, world: int, rank: int) -> tuple[int, int]:
    """(first sequence, count) of `rank`'s contiguous, balanced share of `total` sequences."""
    if world < 1 or not 0 <= rank < world or total < 0:
        raise ValueError("bad shard arguments")
    base, extra = divmod(total, world)
    start = rank * base + min(rank, extra)
    return start, base + (1 if rank < extra else 0)


def env_ranks() -> tuple[int, int, int]:
    """(rank, world size, local rank) from the torch.distributed.run environment."""
    return (int(os.environ.get("RANK", "0")), int(os.environ.get("WORLD_SIZE", "1")),
            int(os.environ.get("LOCAL_RANK", "0")))


def init(backend: str, timeout_s: float = 300.0, device=None) -> None:
    import torch.distributed as dist
    kw = {"timeout": datetime.timedelta(seconds=timeout_s)}
    if device is not None:
        kw["device_id"] = device
    dist.init_process_group(backend, **kw)


def max_over_ranks(value: float, device=None) -> float:
    """The largest of every rank's `value` (the job time is the slowest rank's)."""
    import torch
    import torch.distributed as dist
    if not dist.is_initialized() or dist.get_world_size() == 1:
        return float(value)
    t = torch.tensor([float(value)], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())
