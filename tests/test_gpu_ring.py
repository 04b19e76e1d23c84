"""Ring attention's kernels on one B200: fa_fwd_partial (one key range's fp32
share), fa_merge_partials (the logsumexp merge) and every rank of a ring run
one after the other (emulate_ring_forward: the ring's schedule, per-step
kernels and merge, without communication), against the fp64 oracle of the
whole sequence.  Tolerances as the forward's."""
import numpy as np
import pytest

import oracle
from exact_tiled_attention_32_b200 import synthetic as syn
from fa_util import assert_parity, to_device

pytestmark = pytest.mark.gpu


@pytest.mark.parametrize("world,B,Hq,Hkv,N,d,causal", [
    (1, 1, 2, 2, 256, 128, True),
    (2, 1, 4, 2, 512, 128, True),
    (4, 2, 2, 2, 1024, 64, True),
    (4, 1, 2, 1, 768, 128, False),
    (3, 1, 2, 2, 384, 128, True),     # shards of 128
    (2, 1, 2, 2, 300, 128, True),     # shards of 150: ragged tiles in every shard
])
def test_emulated_ring_matches_oracle(world, B, Hq, Hkv, N, d, causal):
    import torch
    from exact_tiled_attention_32_b200 import binding as fa
    from exact_tiled_attention_32_b200.ring import emulate_ring_forward
    w = syn.Workload("ring", B, Hq, Hkv, N, d, causal, 1200 + N + world).draw()
    o, lse = emulate_ring_forward(to_device(w.q), to_device(w.k), to_device(w.v), world, causal=causal,
                                  scale=w.scale)
    torch.cuda.synchronize()
    assert fa.fa_get_device_status() == 0
    oo, lo = oracle.attention(w.q, w.k, w.v, B, Hq, Hkv, N, d, w.scale, causal)
    assert_parity(o.float().cpu().numpy().astype(np.float64).reshape(-1, d),
                  lse.cpu().numpy().astype(np.float64).reshape(-1), oo, lo, f"ring {world} {N} {causal}")


def test_partial_share_and_merge():
    """Keys split in two ranges: each range's share against the oracle of that
    range alone, and their merge against the oracle of all keys."""
    import torch
    from exact_tiled_attention_32_b200 import binding as fa
    B, Hq, Hkv, Nq, Nk, d = 1, 4, 2, 200, 700, 128
    w = syn.Workload("part", B, Hq, Hkv, Nq, d, False, 1250, Nk=Nk).draw()
    q, k, v = to_device(w.q), to_device(w.k), to_device(w.v)
    rows = B * Hq * Nq
    o_parts = torch.empty((2, rows, d), dtype=torch.float32, device="cuda")
    l_parts = torch.empty((2, rows), dtype=torch.float32, device="cuda")
    cut = 300
    halves = [(0, cut), (cut, Nk)]
    for n, (a, b) in enumerate(halves):
        ks, vs = k[:, :, a:b].contiguous(), v[:, :, a:b].contiguous()
        assert fa.fa_fwd_partial(q, ks, vs, o_parts[n], l_parts[n], B, Hq, Hkv, Nq, b - a, d, w.scale, False) == 0
    o = torch.empty((B, Hq, Nq, d), dtype=torch.bfloat16, device="cuda")
    lse = torch.empty((B, Hq, Nq), dtype=torch.float32, device="cuda")
    assert fa.fa_merge_partials(o_parts, l_parts, 2, rows, d, o, lse) == 0
    torch.cuda.synchronize()
    for n, (a, b) in enumerate(halves):
        kb = np.ascontiguousarray(w.k[:, :, a:b])
        vb = np.ascontiguousarray(w.v[:, :, a:b])
        oo, lo = oracle.attention_kv(w.q, kb, vb, B, Hq, Hkv, Nq, b - a, d, w.scale, False)
        assert np.abs(o_parts[n].cpu().numpy() - oo).max() <= 1e-2       # fp32 share, bf16 P
        assert np.abs(l_parts[n].cpu().numpy() - lo).max() <= 1e-3
    oo, lo = oracle.attention_kv(w.q, w.k, w.v, B, Hq, Hkv, Nq, Nk, d, w.scale, False)
    assert_parity(o.float().cpu().numpy().astype(np.float64).reshape(-1, d),
                  lse.cpu().numpy().astype(np.float64).reshape(-1), oo, lo, "merge")


def test_merge_argument_errors():
    from exact_tiled_attention_32_b200 import binding as fa
    p = 1 << 20
    assert fa.fa_merge_partials(p, p, 0, 10, 128, p, p) == fa.FA_ERR_SHAPE
    assert fa.fa_merge_partials(p, p, 2, 10, 96, p, p) == fa.FA_ERR_HEADDIM
    assert fa.fa_merge_partials(0, p, 2, 10, 128, p, p) == fa.FA_ERR_NULL
    assert fa.fa_merge_partials(p, p, 2, 0, 128, 0, 0) == fa.FA_OK


def test_ring_forward_on_one_rank():
    """The distributed driver itself (one NCCL rank: one step, no exchange)."""
    import socket

    import torch
    import torch.distributed as dist
    from exact_tiled_attention_32_b200.ring import ring_attention_forward
    with socket.socket() as sk:
        sk.bind(("127.0.0.1", 0))
        port = sk.getsockname()[1]
    dist.init_process_group("nccl", init_method=f"tcp://127.0.0.1:{port}", rank=0, world_size=1)
    try:
        w = syn.Workload("ring1", 1, 2, 2, 384, 128, True, 1260).draw()
        o, lse = ring_attention_forward(to_device(w.q), to_device(w.k), to_device(w.v), causal=True)
        torch.cuda.synchronize()
        oo, lo = oracle.attention(w.q, w.k, w.v, 1, 2, 2, 384, 128, w.scale, True)
        assert_parity(o.float().cpu().numpy().astype(np.float64).reshape(-1, 128),
                      lse.cpu().numpy().astype(np.float64).reshape(-1), oo, lo, "ring world 1")
    finally:
        dist.destroy_process_group()


@pytest.mark.parametrize("world,B,Hq,Hkv,N,d,causal", [
    (1, 1, 2, 2, 256, 128, True),
    (2, 1, 4, 2, 512, 128, True),     # chunks of 128
    (4, 2, 2, 2, 1024, 64, True),
    (3, 1, 2, 1, 900, 128, True),     # chunks of 150: ragged tiles in every chunk
    (4, 1, 2, 2, 1024, 128, False),
])
def test_emulated_zigzag_ring_matches_oracle(world, B, Hq, Hkv, N, d, causal):
    """The zig-zag assignment (rank r holds chunks r and 2 world - 1 - r):
    every rank's four chunk pairs per step, run one after the other, merged,
    and put back in sequence order."""
    import torch
    from exact_tiled_attention_32_b200 import binding as fa
    from exact_tiled_attention_32_b200.ring import emulate_zigzag_forward
    w = syn.Workload("zigzag", B, Hq, Hkv, N, d, causal, 1270 + N + world).draw()
    o, lse = emulate_zigzag_forward(to_device(w.q), to_device(w.k), to_device(w.v), world, causal=causal,
                                    scale=w.scale)
    torch.cuda.synchronize()
    assert fa.fa_get_device_status() == 0
    oo, lo = oracle.attention(w.q, w.k, w.v, B, Hq, Hkv, N, d, w.scale, causal)
    assert_parity(o.float().cpu().numpy().astype(np.float64).reshape(-1, d),
                  lse.cpu().numpy().astype(np.float64).reshape(-1), oo, lo, f"zigzag {world} {N} {causal}")


def test_zigzag_ring_forward_on_one_rank():
    """The distributed zig-zag driver (one NCCL rank: its shard is chunks 0
    and 1, the whole sequence in order)."""
    import socket

    import torch
    import torch.distributed as dist
    from exact_tiled_attention_32_b200.ring import ring_attention_forward_zigzag
    with socket.socket() as sk:
        sk.bind(("127.0.0.1", 0))
        port = sk.getsockname()[1]
    dist.init_process_group("nccl", init_method=f"tcp://127.0.0.1:{port}", rank=0, world_size=1)
    try:
        w = syn.Workload("zz1", 1, 2, 2, 384, 128, True, 1280).draw()
        o, lse = ring_attention_forward_zigzag(to_device(w.q), to_device(w.k), to_device(w.v), causal=True)
        torch.cuda.synchronize()
        oo, lo = oracle.attention(w.q, w.k, w.v, 1, 2, 2, 384, 128, w.scale, True)
        assert_parity(o.float().cpu().numpy().astype(np.float64).reshape(-1, 128),
                      lse.cpu().numpy().astype(np.float64).reshape(-1), oo, lo, "zigzag world 1")
    finally:
        dist.destroy_process_group()
