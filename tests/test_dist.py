"""Multi-rank host logic on CPU: shards are disjoint and complete, and the
max-over-ranks timing reduction works across a world of two gloo ranks."""
import os
import socket

import pytest
import torch.multiprocessing as mp

from reduced_query_head_b200.dist import max_over_ranks, shard_batch_groups, shard_range


@pytest.mark.parametrize("n,world", [(0, 1), (1, 2), (7, 2), (16, 4), (44, 8), (5, 8)])
def test_shards_partition_the_units(n, world):
    seen = []
    for r in range(world):
        a, b = shard_range(n, r, world)
        assert 0 <= a <= b <= n
        seen.extend(range(a, b))
    assert seen == list(range(n))
    sizes = [shard_range(n, r, world)[1] - shard_range(n, r, world)[0] for r in range(world)]
    assert max(sizes) - min(sizes) <= 1


def test_batch_group_units_cover_once():
    units = [u for r in range(3) for u in shard_batch_groups(4, 5, r, 3)]
    assert sorted(units) == [(b, g) for b in range(4) for g in range(5)]


def test_bad_requests_rejected():
    with pytest.raises(ValueError):
        shard_range(4, 2, 2)
    with pytest.raises(ValueError):
        shard_range(4, 0, 0)


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _worker(rank, world, port, q):
    import torch.distributed as dist
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        got = max_over_ranks([float(rank), 10.0 - rank])
        units = shard_batch_groups(2, 3, rank, world)
        q.put((rank, got, units))
    finally:
        dist.destroy_process_group()


def test_two_gloo_ranks_reduce_and_shard():
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_worker, args=(r, 2, port, q)) for r in range(2)]
    for p in procs:
        p.start()
    res = {}
    for _ in procs:
        r, got, units = q.get(timeout=120)
        res[r] = (got, units)
    for p in procs:
        p.join(60)
        assert p.exitcode == 0
    assert res[0][0] == [1.0, 10.0] and res[1][0] == [1.0, 10.0]
    assert sorted(res[0][1] + res[1][1]) == [(b, g) for b in range(2) for g in range(3)]


# ---------------------------------------------------------------- sequence sharding
from reduced_query_head_b200.dist import sequence_blocks  # noqa: E402


@pytest.mark.parametrize("causal", [False, True])
@pytest.mark.parametrize("N,world", [(1, 1), (37, 2), (100, 4), (7, 4), (1000, 8)])
def test_sequence_blocks_partition_and_balance(N, world, causal):
    seen = []
    for r in range(world):
        seen.extend(t for a, b in sequence_blocks(N, r, world, causal) for t in range(a, b))
    assert sorted(seen) == list(range(N)) and len(seen) == N
    if causal and N >= 4 * world:
        # Causal work of a row t is t + 1 keys. With equal chunks of c rows, rank r's pair
        # (chunks r and 2W-1-r) costs c^2 (2W - 1) + c (c + 1) whatever r is; uneven chunks
        # (sizes differ by one) add at most two rows of at most N keys.
        work = [sum(t + 1 for a, b in sequence_blocks(N, r, world, True) for t in range(a, b)) for r in range(world)]
        assert max(work) - min(work) <= 2 * N
        contiguous = [sum(t + 1 for t in range(*shard_range(N, r, world))) for r in range(world)]
        assert max(contiguous) - min(contiguous) > 2 * N   # what the pairing avoids


def _attn_rows_cpu(q_block, k_full, v_full, q_offset, causal, scale):
    """float64 reference for one block of query rows at global positions q_offset.."""
    import torch
    n, N = q_block.shape[1], k_full.shape[1]
    R = q_block.shape[2] // k_full.shape[2]
    q = q_block.permute(0, 2, 1, 3)
    k = k_full.permute(0, 2, 1, 3).repeat_interleave(R, dim=1)
    v = v_full.permute(0, 2, 1, 3).repeat_interleave(R, dim=1)
    s = scale * q @ k.transpose(-1, -2)
    if causal:
        t = torch.arange(n)[:, None] + q_offset
        s = s.masked_fill(torch.arange(N)[None, :] > t, float("-inf"))
    return (torch.softmax(s, dim=-1) @ v).permute(0, 2, 1, 3)


def _seq_worker(rank, world, port, causal, q, B=2, N=37):
    import torch
    import torch.distributed as dist
    from reduced_query_head_b200.dist import sequence_parallel_attention
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        g = torch.Generator().manual_seed(7)
        H_q, H_kv, d, scale = 4, 2, 8, 0.35
        qf = torch.randn(B, N, H_q, d, generator=g, dtype=torch.float64)
        kf = torch.randn(B, N, H_kv, d, generator=g, dtype=torch.float64)
        vf = torch.randn(B, N, H_kv, d, generator=g, dtype=torch.float64)
        blocks = sequence_blocks(N, rank, world, causal)
        take = lambda x: torch.cat([x[:, a:b] for a, b in blocks], dim=1)
        out = sequence_parallel_attention(take(qf), take(kf), take(vf), N, rank, world, causal,
                                          lambda qb, kk, vv, off: _attn_rows_cpu(qb, kk, vv, off, causal, scale))
        want = take(_attn_rows_cpu(qf, kf, vf, 0, causal, scale))
        q.put((rank, float((out - want).abs().max())))
    finally:
        dist.destroy_process_group()


@pytest.mark.parametrize("B,N", [(2, 37), (1, 64)])
@pytest.mark.parametrize("causal", [False, True])
def test_sequence_parallel_attention_two_gloo_ranks(causal, B, N):
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_seq_worker, args=(r, 2, port, causal, q, B, N)) for r in range(2)]
    for p in procs:
        p.start()
    res = [q.get(timeout=120) for _ in procs]
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    assert sorted(r for r, _ in res) == [0, 1]
    assert max(e for _, e in res) <= 1e-12, res


def _gather_worker(rank, world, port, cases, q):
    import torch
    import torch.distributed as dist
    from reduced_query_head_b200.dist import gather_sequence
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        errs = []
        for B, N, causal in cases:
            full = torch.arange(B * N * 3 * 2, dtype=torch.float32).reshape(B, N, 3, 2)
            blocks = sequence_blocks(N, rank, world, causal)
            local = torch.cat([full[:, a:b] for a, b in blocks], dim=1)
            got = gather_sequence(local, N, world, causal)
            errs.append(((B, N, causal), bool(torch.equal(got, full))))
        q.put((rank, errs))
    finally:
        dist.destroy_process_group()


@pytest.mark.parametrize("world", [2, 4])
def test_gather_sequence_restores_global_order(world):
    """The K/V exchange of sequence sharding: one sequence in equal shards (gathered straight into
    place, causal chunks pairs included) and shapes that take the padded path (B > 1, uneven shards)."""
    cases = [(1, 64, False), (1, 64, True), (1, 40, True), (1, 37, False), (1, 37, True), (2, 64, False),
             (2, 37, True)]
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_gather_worker, args=(r, world, port, cases, q)) for r in range(world)]
    for p in procs:
        p.start()
    res = [q.get(timeout=120) for _ in procs]
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    for _, errs in res:
        assert all(ok for _, ok in errs), errs
