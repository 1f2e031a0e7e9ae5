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
