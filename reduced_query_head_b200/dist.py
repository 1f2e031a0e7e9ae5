"""Host-side helpers for running the attention path on several GPUs.

Decoupled-head attention over (batch, KV group) units needs no data exchange:
every unit reads only its own Q heads and its own K/V group. So N GPUs run
N disjoint shards of the units, one process per GPU, and the only collective
is the timing reduction (max over ranks) around the measured region.
"""
from __future__ import annotations

import os


def shard_range(n_units: int, rank: int, world: int):
    """Contiguous, balanced [start, stop) of n_units for this rank."""
    if world < 1 or not 0 <= rank < world or n_units < 0:
        raise ValueError("bad shard request")
    base, extra = divmod(n_units, world)
    start = rank * base + min(rank, extra)
    return start, start + base + (1 if rank < extra else 0)


def shard_batch_groups(B: int, H_kv: int, rank: int, world: int):
    """(batch, group) units of one rank, in row-major order of (b, g)."""
    start, stop = shard_range(B * H_kv, rank, world)
    return [divmod(u, H_kv) for u in range(start, stop)]


def env_rank_world():
    return int(os.environ.get("RANK", "0")), int(os.environ.get("WORLD_SIZE", "1")), \
        int(os.environ.get("LOCAL_RANK", "0"))


def max_over_ranks(values, device=None):
    """Element-wise maximum of a list of floats across all ranks (identity when not initialised)."""
    import torch
    import torch.distributed as dist
    t = torch.tensor(list(values), dtype=torch.float64, device=device)
    if dist.is_available() and dist.is_initialized() and dist.get_world_size() > 1:
        dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return [float(x) for x in t.cpu()]
