"""Ring attention's host logic on the CPU: the schedule of key/value shards
and modes, and the shard pass-along over torch.distributed (gloo, 2 and 3
ranks) -- every rank must hold shard (rank - t) mod world at step t."""
import os
import socket

import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp

from exact_tiled_attention_32_b200.ring import DIAG, FULL, SKIP, DistExchange, ring_schedule


def test_ring_schedule_modes():
    for world in (1, 2, 3, 5):
        for rank in range(world):
            s = ring_schedule(rank, world, causal=True)
            assert [src for src, _ in s] == [(rank - t) % world for t in range(world)]
            for src, mode in s:
                assert mode == (FULL if src < rank else DIAG if src == rank else SKIP)
            assert all(m == FULL for _, m in ring_schedule(rank, world, causal=False))
    # every (query shard, key shard) pair below or on the diagonal is computed exactly once
    world = 4
    seen = {(r, src) for r in range(world) for src, m in ring_schedule(r, world, True) if m != SKIP}
    assert seen == {(r, s) for r in range(world) for s in range(r + 1)}
    with pytest.raises(ValueError):
        ring_schedule(3, 3, True)


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _worker(rank, world, port, out):
    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        ex = DistExchange()
        shard = torch.full((2, 3), float(rank))
        held = [int(shard[0, 0])]
        bufs = [shard, torch.empty_like(shard)]
        cur = 0
        for t in range(world - 1):
            reqs = ex.start([bufs[cur]], [bufs[1 - cur]])
            ex.wait(reqs)
            cur = 1 - cur
            if t == 0:
                bufs[1 - cur] = torch.empty_like(shard)
            held.append(int(bufs[cur][0, 0]))
        assert shard.eq(rank).all(), "the rank's own shard was overwritten"
        out[rank] = held
    finally:
        dist.destroy_process_group()


@pytest.mark.parametrize("world", [2, 3])
def test_ring_exchange_passes_shards(world):
    ctx = mp.get_context("spawn")
    out = ctx.Manager().dict()
    mp.start_processes(_worker, args=(world, _free_port(), out), nprocs=world, join=True, start_method="spawn")
    for rank in range(world):
        assert out[rank] == [src for src, _ in ring_schedule(rank, world, True)]
