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


# ---------------------------------------------------------------- zig-zag
def test_zigzag_schedule_balance_and_coverage():
    from exact_tiled_attention_32_b200.ring import zigzag_chunks, zigzag_schedule
    for world in (1, 2, 3, 4, 7):
        seen = set()
        for rank in range(world):
            s = zigzag_schedule(rank, world, causal=True)
            assert [src for src, _ in s] == [(rank - t) % world for t in range(world)]
            for t, (src, pairs) in enumerate(s):
                modes = [m for _, _, m in pairs]
                # the same work on every rank at every step
                if t == 0:
                    assert sorted(modes) == [DIAG, DIAG, FULL, SKIP]
                else:
                    assert modes.count(FULL) == 2 and modes.count(SKIP) == 2
                for qi, ki, m in pairs:
                    a, b = zigzag_chunks(rank, world)[qi], zigzag_chunks(src, world)[ki]
                    assert m == (FULL if b < a else DIAG if b == a else SKIP)
                    if m != SKIP:
                        assert (a, b) not in seen
                        seen.add((a, b))
        # every (query chunk, key chunk) pair on or below the diagonal exactly once
        n = 2 * world
        assert seen == {(a, b) for a in range(n) for b in range(a + 1)}
        for rank in range(world):
            assert all(m == FULL for _, pairs in zigzag_schedule(rank, world, False) for _, _, m in pairs)


def test_zigzag_shard_round_trip():
    from exact_tiled_attention_32_b200.ring import zigzag_shard, zigzag_unshard
    world, C = 3, 5
    x = torch.arange(2 * 2 * 2 * world * C * 4, dtype=torch.float32).reshape(2, 2, 2 * world * C, 4)
    shards = [zigzag_shard(x, r, world) for r in range(world)]
    for r, sh in enumerate(shards):
        assert sh.shape == (2, 2, 2 * C, 4) and sh.is_contiguous()
        assert torch.equal(sh[:, :, :C], x[:, :, r * C:(r + 1) * C])
        b = 2 * world - 1 - r
        assert torch.equal(sh[:, :, C:], x[:, :, b * C:(b + 1) * C])
    assert torch.equal(zigzag_unshard(shards, world), x)
    with pytest.raises(ValueError):
        zigzag_shard(x[:, :, :-1], 0, world)


def _zigzag_worker(rank, world, port, out):
    from exact_tiled_attention_32_b200.ring import zigzag_chunks
    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        ex = DistExchange()
        # four tensors per step (K and V halves), each tagged with its chunk
        a, b = zigzag_chunks(rank, world)
        own = [torch.full((3,), float(a)), torch.full((3,), float(b)),
               torch.full((3,), 100.0 + a), torch.full((3,), 100.0 + b)]
        bufs = [tuple(x.clone() for x in own), tuple(torch.empty(3) for _ in own)]
        cur = 0
        held = [tuple(int(x[0]) for x in bufs[cur])]
        for t in range(world - 1):
            reqs = ex.start(list(bufs[cur]), list(bufs[1 - cur]))
            ex.wait(reqs)
            cur = 1 - cur
            held.append(tuple(int(x[0]) for x in bufs[cur]))
        out[rank] = held
    finally:
        dist.destroy_process_group()


@pytest.mark.parametrize("world", [2, 3])
def test_zigzag_exchange_passes_chunk_pairs(world):
    from exact_tiled_attention_32_b200.ring import zigzag_chunks, zigzag_schedule
    ctx = mp.get_context("spawn")
    out = ctx.Manager().dict()
    mp.start_processes(_zigzag_worker, args=(world, _free_port(), out), nprocs=world, join=True,
                       start_method="spawn")
    for rank in range(world):
        want = []
        for src, _ in zigzag_schedule(rank, world, True):
            a, b = zigzag_chunks(src, world)
            want.append((a, b, 100 + a, 100 + b))
        assert out[rank] == want


class _TorchKernels:
    """Stand-ins for fa_fwd_partial / fa_merge_partials in torch fp64 (the
    documented semantics of the two entry points), so that the ring drivers'
    scheduling and merging can run on the CPU."""
    FA_OK = 0

    class FAError(RuntimeError):
        def __init__(self, rc, what=""):
            super().__init__(f"{what}: {rc}")

    @staticmethod
    def fa_fwd_partial(q, k, v, o_part, lse_part, B, Hq, Hkv, Nq, Nk, d, scale, causal, stream=None):
        g = Hq // Hkv
        qq = q.double().reshape(B, Hq, Nq, d)
        kk = k.double().reshape(B, Hkv, Nk, d).repeat_interleave(g, dim=1)
        vv = v.double().reshape(B, Hkv, Nk, d).repeat_interleave(g, dim=1)
        s = scale * qq @ kk.transpose(-1, -2)
        if causal:   # query i at key position Nk - Nq + i
            i = torch.arange(Nq).unsqueeze(1) + (Nk - Nq)
            s = s.masked_fill(torch.arange(Nk).unsqueeze(0) > i, float("-inf"))
        lse = torch.logsumexp(s, dim=-1)
        p = torch.exp(s - lse.unsqueeze(-1))
        o_part.copy_((p @ vv).reshape(-1, d).float())
        lse_part.copy_(lse.reshape(-1).float())
        return 0

    @staticmethod
    def fa_merge_partials(o_parts, lse_parts, n, rows, d, o, lse, stream=None):
        # a part whose lse is -inf holds no key and is skipped (its O part is
        # never written)
        lp = lse_parts[:n].double()
        m = lp.max(dim=0).values
        live = torch.isfinite(lp)
        w = torch.where(live, torch.exp(lp - m), torch.zeros_like(lp))
        tot = w.sum(dim=0)
        op = torch.where(live.unsqueeze(-1), o_parts[:n].double(), torch.zeros(1, dtype=torch.float64))
        out = (w.unsqueeze(-1) * op).sum(dim=0) / tot.unsqueeze(-1)
        o.copy_(out.reshape(o.shape).to(o.dtype))
        lse.copy_((m + torch.log(tot)).reshape(lse.shape).float())
        return 0


@pytest.mark.parametrize("zigzag", [True, False])
@pytest.mark.parametrize("world,causal", [(1, True), (2, True), (3, True), (4, False)])
def test_ring_driver_host_logic(world, causal, zigzag, monkeypatch):
    """emulate_zigzag_forward and emulate_ring_forward with torch stand-ins
    for the two kernels give the oracle's attention of the whole sequence:
    the shard or chunk pairs, modes, part slots, merges and the final
    un-sharding are right."""
    import sys

    import numpy as np

    import oracle
    import exact_tiled_attention_32_b200 as pkg
    from exact_tiled_attention_32_b200 import ring
    from exact_tiled_attention_32_b200 import synthetic as syn
    monkeypatch.setitem(sys.modules, "exact_tiled_attention_32_b200.binding", _TorchKernels)
    monkeypatch.setattr(pkg, "binding", _TorchKernels, raising=False)
    monkeypatch.setattr(torch.cuda, "current_stream", lambda *a, **k: None)
    B, Hq, Hkv, d = 1, 4, 2, 16
    N = 2 * world * 6
    w = syn.Workload("zz", B, Hq, Hkv, N, d, causal, 1300 + N).draw()
    t = lambda a: torch.from_numpy(a.view(np.int16).astype(np.int32) << 16).view(torch.float32)
    run = ring.emulate_zigzag_forward if zigzag else ring.emulate_ring_forward
    o, lse = run(t(w.q), t(w.k), t(w.v), world, causal=causal, scale=w.scale)
    oo, lo = oracle.attention(w.q, w.k, w.v, B, Hq, Hkv, N, d, w.scale, causal)
    assert np.abs(o.double().numpy().reshape(-1, d) - oo).max() < 1e-2      # bf16 output rounding
    assert np.abs(lse.double().numpy().reshape(-1) - lo).max() < 1e-5


def _driver_worker(rank, world, port, zigzag, causal, out):
    """One rank of the distributed drivers over gloo, with the torch
    stand-ins for the kernels: returns this rank's O and lse."""
    import sys

    import numpy as np

    import exact_tiled_attention_32_b200 as pkg
    from exact_tiled_attention_32_b200 import ring
    from exact_tiled_attention_32_b200 import synthetic as syn
    sys.modules["exact_tiled_attention_32_b200.binding"] = _TorchKernels
    pkg.binding = _TorchKernels
    torch.cuda.current_stream = lambda *a, **k: None
    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        B, Hq, Hkv, d = 1, 4, 2, 16
        N = 2 * world * 6
        w = syn.Workload("zzd", B, Hq, Hkv, N, d, causal, 1400 + N).draw()
        t = lambda a: torch.from_numpy(a.view(np.int16).astype(np.int32) << 16).view(torch.float32)
        q, k, v = t(w.q), t(w.k), t(w.v)
        if zigzag:
            o, lse = ring.ring_attention_forward_zigzag(ring.zigzag_shard(q, rank, world), ring.zigzag_shard(k, rank, world),
                                                        ring.zigzag_shard(v, rank, world), causal=causal, scale=w.scale)
        else:
            L = N // world
            sl = slice(rank * L, (rank + 1) * L)
            o, lse = ring.ring_attention_forward(q[:, :, sl].contiguous(), k[:, :, sl].contiguous(),
                                                 v[:, :, sl].contiguous(), causal=causal, scale=w.scale)
        out[rank] = (o.double().numpy(), lse.double().numpy())
    finally:
        dist.destroy_process_group()


@pytest.mark.parametrize("zigzag", [False, True])
@pytest.mark.parametrize("world,causal", [(2, True), (3, True), (2, False)])
def test_distributed_ring_drivers(world, causal, zigzag):
    """ring_attention_forward and ring_attention_forward_zigzag over gloo
    ranks, the kernels replaced by torch stand-ins: every rank's rows match
    the oracle's attention of the whole sequence."""
    import numpy as np

    import oracle
    from exact_tiled_attention_32_b200 import ring
    from exact_tiled_attention_32_b200 import synthetic as syn
    ctx = mp.get_context("spawn")
    out = ctx.Manager().dict()
    mp.start_processes(_driver_worker, args=(world, _free_port(), zigzag, causal, out), nprocs=world, join=True,
                       start_method="spawn")
    B, Hq, Hkv, d = 1, 4, 2, 16
    N = 2 * world * 6
    w = syn.Workload("zzd", B, Hq, Hkv, N, d, causal, 1400 + N).draw()
    oo, lo = oracle.attention(w.q, w.k, w.v, B, Hq, Hkv, N, d, w.scale, causal)
    oo = torch.from_numpy(oo.reshape(B, Hq, N, d))
    lo = torch.from_numpy(lo.reshape(B, Hq, N))
    if zigzag:
        want = [(ring.zigzag_shard(oo, r, world), ring.zigzag_shard(lo.unsqueeze(-1), r, world).squeeze(-1))
                for r in range(world)]
    else:
        L = N // world
        want = [(oo[:, :, r * L:(r + 1) * L], lo[:, :, r * L:(r + 1) * L]) for r in range(world)]
    for r in range(world):
        o, lse = out[r]
        assert np.abs(o - want[r][0].numpy()).max() < 1e-2
        assert np.abs(lse - want[r][1].numpy()).max() < 1e-5
