"""Multi-rank host logic on CPU: two gloo ranks shard a batch by rows and
reduce their timings with a max; the shards cover every row exactly once."""

import os
import socket

import pytest
import torch
import torch.multiprocessing as mp

from rwkv_delta_rule_b200.dist import max_over_ranks, rank_seed, shard_rows


@pytest.mark.parametrize("B,world", [(8, 2), (7, 2), (5, 3), (1, 4), (0, 2)])
def test_shards_cover_rows_once(B, world):
    rows = []
    for r in range(world):
        lo, hi = shard_rows(B, world, r)
        assert 0 <= lo <= hi <= B
        rows.extend(range(lo, hi))
    assert rows == list(range(B))
    sizes = [shard_rows(B, world, r)[1] - shard_rows(B, world, r)[0] for r in range(world)]
    assert max(sizes) - min(sizes) <= 1


def test_rank_seeds_differ():
    assert len({rank_seed(1001, r) for r in range(8)}) == 8


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _worker(rank, world, port, out):
    import torch.distributed as dist

    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        lo, hi = shard_rows(8, world, rank)
        local = float(10 * (rank + 1))
        out[rank] = max_over_ranks(local)
        # the shard sizes reach every rank the same way
        t = torch.tensor([hi - lo], dtype=torch.int64)
        dist.all_reduce(t)
        out[world + rank] = float(t.item())
    finally:
        dist.destroy_process_group()


def test_gloo_two_ranks_max_and_shards():
    world = 2
    ctx = mp.get_context("spawn")
    out = ctx.Array("d", 2 * world)
    port = _free_port()
    procs = [ctx.Process(target=_worker, args=(r, world, port, out)) for r in range(world)]
    for p in procs:
        p.start()
    for p in procs:
        p.join(timeout=120)
        assert p.exitcode == 0
    assert list(out[:world]) == [20.0, 20.0]
    assert list(out[world:]) == [8.0, 8.0]


def test_single_process_max_is_identity():
    assert max_over_ranks(3.5) == 3.5
