"""Multi-rank host logic on CPU (gloo, world size 2): unit sharding and max-over-ranks timing."""
import os
import socket

import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp

from attention_tcgen05_tma_b200.distributed import max_over_ranks, shard_range


def test_shard_range_covers_units_once():
    for n in (0, 1, 7, 8, 4096):
        for world in (1, 2, 3, 8):
            seen = []
            for r in range(world):
                a, b = shard_range(n, r, world)
                seen.extend(range(a, b))
                assert (b - a) in (n // world, n // world + 1)
            assert seen == list(range(n))


def _free_port():
    s = socket.socket()
    s.bind(("127.0.0.1", 0))
    p = s.getsockname()[1]
    s.close()
    return p


def _worker(rank, world, port, out):
    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    import datetime
    dist.init_process_group("gloo", rank=rank, world_size=world, timeout=datetime.timedelta(seconds=60))
    try:
        ms = 10.0 + 5.0 * rank
        out[rank] = max_over_ranks(ms, dist)
        a, b = shard_range(8, rank, world)
        t = torch.tensor([b - a], dtype=torch.int64)
        dist.all_reduce(t)
        out[world + rank] = float(t.item())
    finally:
        dist.destroy_process_group()


def test_two_rank_gloo_max_and_sharding():
    world = 2
    port = _free_port()
    ctx = mp.get_context("spawn")
    out = ctx.Array("d", 2 * world)
    procs = [ctx.Process(target=_worker, args=(r, world, port, out)) for r in range(world)]
    for p in procs:
        p.start()
    for p in procs:
        p.join(120)
        assert p.exitcode == 0
    assert list(out[:world]) == [15.0, 15.0]       # every rank sees the slowest rank's time
    assert list(out[world:]) == [8.0, 8.0]         # the shards cover the 8 units
