"""Host-side helpers for running the attention path on several GPUs.

Decoupled-head attention over (batch, KV group) units needs no data exchange:
every unit reads only its own Q heads and its own K/V group. So N GPUs run
N disjoint shards of the units, one process per GPU, and the only collective
is the timing reduction (max over ranks) around the measured region.

A single sequence too long for one GPU is sharded by query position instead
(sequence_blocks); there the K/V all-gather is a real exchange step.
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


# ---------------------------------------------------------------------------
# Sequence sharding: one long sequence over several GPUs. Each rank owns blocks
# of query positions (and the K/V rows it computed for them); the exchange step
# gathers every rank's K and V, then each rank runs attention for its own
# query rows against all keys (sqa_attn_fwd_rows).
# ---------------------------------------------------------------------------

def sequence_blocks(N: int, rank: int, world: int, causal: bool):
    """Query-position blocks [(start, stop), ...] of this rank.

    Non-causal: one contiguous block. Causal: the sequence is cut into
    2 * world near-equal chunks and rank r takes chunks r and 2*world-1-r, so
    every rank pairs a cheap early chunk with an expensive late one and the
    causal work is balanced.
    """
    if world < 1 or not 0 <= rank < world or N < 1:
        raise ValueError("bad shard request")
    if not causal:
        return [shard_range(N, rank, world)]
    a = shard_range(N, rank, 2 * world)
    b = shard_range(N, 2 * world - 1 - rank, 2 * world)
    return [blk for blk in (a, b) if blk[1] > blk[0]]


def gather_sequence(local, N: int, world: int, causal: bool, group=None):
    """All-gather every rank's token rows into global order.

    `local` is [B, n_local, H, d]: this rank's rows of its sequence_blocks,
    concatenated in block order. Returns [B, N, H, d] on every rank.

    One sequence (B = 1) in equal shards, the sequence-sharding case, is
    gathered straight into the global buffer: non-causal blocks arrive in rank
    order, which is global order; causal ranks' first chunks (0 .. world-1)
    arrive in place, and only their second chunks (2*world-1-r, in reverse)
    are moved once more. Other shapes go through a padded gather and a copy
    of each block into place.
    """
    import torch
    import torch.distributed as dist
    blocks = [sequence_blocks(N, r, world, causal) for r in range(world)]
    sizes = [sum(b - a for a, b in blk) for blk in blocks]
    B, n_local = local.shape[0], local.shape[1]
    rest = tuple(local.shape[2:])
    full = torch.empty((B, N) + rest, dtype=local.dtype, device=local.device)
    if B == 1 and len(set(sizes)) == 1 and hasattr(dist, "all_gather_into_tensor"):
        if not causal:
            dist.all_gather_into_tensor(full[0], local[0].contiguous(), group=group)
            return full
        chunk = N // (2 * world)
        if N == 2 * world * chunk:
            dist.all_gather_into_tensor(full[0, :world * chunk], local[0, :chunk].contiguous(), group=group)
            late = torch.empty((world * chunk,) + rest, dtype=local.dtype, device=local.device)
            dist.all_gather_into_tensor(late, local[0, chunk:2 * chunk].contiguous(), group=group)
            for r in range(world):
                c = 2 * world - 1 - r
                full[0, c * chunk:(c + 1) * chunk] = late[r * chunk:(r + 1) * chunk]
            return full
    top = max(sizes)
    pad = torch.zeros((B, top) + rest, dtype=local.dtype, device=local.device)
    pad[:, :n_local] = local
    parts = [torch.empty_like(pad) for _ in range(world)]
    dist.all_gather(parts, pad.contiguous(), group=group)
    for r in range(world):
        off = 0
        for a, b in blocks[r]:
            full[:, a:b] = parts[r][:, off:off + (b - a)]
            off += b - a
    return full


def sequence_parallel_attention(q_local, k_local, v_local, N: int, rank: int, world: int, causal: bool,
                                attn_rows, group=None):
    """This rank's attention output rows for a sequence sharded by sequence_blocks.

    q_local, k_local, v_local: this rank's rows ([B, n_local, H, d]) of its
    blocks in block order. K and V are gathered (the one exchange step), then
    attn_rows(q_block, k_full, v_full, q_offset) computes each block's rows.
    Returns [B, n_local, H_q, d] in the same block order.
    """
    k_full = gather_sequence(k_local, N, world, causal, group)
    v_full = gather_sequence(v_local, N, world, causal, group)
    outs, off = [], 0
    for a, b in sequence_blocks(N, rank, world, causal):
        outs.append(attn_rows(q_local[:, off:off + (b - a)].contiguous(), k_full, v_full, a))
        off += b - a
    import torch
    return torch.cat(outs, dim=1)
