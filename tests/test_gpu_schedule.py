"""The forward's dynamic work schedule.

Every CTA starts with its own item and then takes the next item of a global
order from a per-launch counter; consecutive launches take consecutive
counters out of a small ring, each tagged with the launch's epoch, so a
counter is reused (with a new epoch) every ring-length launches and never
reset.  Which CTA computes which item changes from launch to launch, but each
item is computed whole by one CTA, so the output must be bitwise the same on
every launch: checked here over more launches than the ring holds, for
a shape with far more items than CTAs (1,024: the dynamic schedule; causal,
uneven item sizes), one with fewer items than CTAs (the static schedule), a
packed batch (item count known only on the device), the no-allocation entry
point (its own, smaller ring) and two streams at once.
One launch per shape is also checked against the oracle.
"""
import pytest

import oracle
from exact_tiled_attention_32_b200 import synthetic as syn
from fa_util import assert_parity, gather, to_device

pytestmark = pytest.mark.gpu

RING = 64            # work counters per device in the library (fa_fwd and the entry points built on it)
NOALLOC_RING = 16    # counters of fa_fwd_noalloc


def _shape(name):
    if name == "many-causal":
        # 1,024 items (pairs of query tiles) on 148 SMs: the dynamic schedule
        return syn.Workload(name, 2, 16, 4, 8192, 64, True, 1401).draw()
    if name == "few-items":
        return syn.Workload(name, 1, 2, 2, 700, 128, False, 1402).draw()
    return syn.packed_from_lengths(name, [1500, 1, 300, 2049, 77, 640], 8, 128, True, 1403, Hkv=2).draw()


def _launch(fa, entry, w, q, k, v, cu, stream):
    import torch
    o = torch.empty_like(q)
    lse = torch.empty((w.Hq, w.N) if w.packed else (w.B, w.Hq, w.N), dtype=torch.float32, device=q.device)
    rc = entry(q, k, v, o, lse, w.B, w.Hq, w.Hkv, w.N, w.d, w.scale, w.causal, cu, stream)
    assert rc == fa.FA_OK
    return o, lse


@pytest.mark.parametrize("name", ["many-causal", "few-items", "packed"])
def test_repeated_launches_are_bitwise_identical(name):
    import torch
    from exact_tiled_attention_32_b200 import binding as fa
    w = _shape(name)
    q, k, v = to_device(w.q), to_device(w.k), to_device(w.v)
    cu = None if w.cu_seqlens is None else torch.from_numpy(w.cu_seqlens).cuda()
    stream = torch.cuda.current_stream()
    o0, l0 = _launch(fa, fa.fa_fwd, w, q, k, v, cu, stream)
    torch.cuda.synchronize()
    assert fa.fa_get_device_status(stream) == fa.FA_OK
    og, lg = gather(w, o0, l0)
    oo, lo = oracle.attention(w.q, w.k, w.v, w.B, w.Hq, w.Hkv, w.N, w.d, w.scale, w.causal, w.cu_seqlens)
    assert_parity(og, lg, oo, lo, f"{name} against the oracle")
    mismatches = 0
    for i in range(RING + 9):               # every counter reused at least once, with a new epoch
        o, lse = _launch(fa, fa.fa_fwd, w, q, k, v, cu, stream)
        mismatches += int(not (torch.equal(o, o0) and torch.equal(lse, l0)))
    torch.cuda.synchronize()
    assert fa.fa_get_device_status(stream) == fa.FA_OK
    assert mismatches == 0


def test_noalloc_ring_reuse_is_bitwise_identical():
    import torch
    from exact_tiled_attention_32_b200 import binding as fa
    w = _shape("many-causal")
    q, k, v = to_device(w.q), to_device(w.k), to_device(w.v)
    stream = torch.cuda.current_stream()
    o0, l0 = _launch(fa, fa.fa_fwd, w, q, k, v, None, stream)
    for i in range(NOALLOC_RING + 5):
        o, lse = _launch(fa, fa.fa_fwd_noalloc, w, q, k, v, None, stream)
        assert fa.fa_get_noalloc_status(stream) == fa.FA_OK
        assert torch.equal(o, o0) and torch.equal(lse, l0), i


def test_two_streams_at_once():
    """Launches in flight together on two streams take different counters."""
    import torch
    from exact_tiled_attention_32_b200 import binding as fa
    wa, wb = _shape("many-causal"), _shape("packed")
    qa, ka, va = to_device(wa.q), to_device(wa.k), to_device(wa.v)
    qb, kb, vb = to_device(wb.q), to_device(wb.k), to_device(wb.v)
    cub = torch.from_numpy(wb.cu_seqlens).cuda()
    main = torch.cuda.current_stream()
    ra = _launch(fa, fa.fa_fwd, wa, qa, ka, va, None, main)
    rb = _launch(fa, fa.fa_fwd, wb, qb, kb, vb, cub, main)
    torch.cuda.synchronize()
    s1, s2 = torch.cuda.Stream(), torch.cuda.Stream()
    outs = []
    for i in range(12):
        outs.append(_launch(fa, fa.fa_fwd, wa, qa, ka, va, None, s1))
        outs.append(_launch(fa, fa.fa_fwd, wb, qb, kb, vb, cub, s2))
    torch.cuda.synchronize()
    assert fa.fa_get_device_status() == fa.FA_OK
    for i, (o, lse) in enumerate(outs):
        ref = ra if i % 2 == 0 else rb
        assert torch.equal(o, ref[0]) and torch.equal(lse, ref[1]), i


def test_packed_long_sequences_in_head_blocks():
    """A packed bf16 batch big enough for the dynamic schedule whose long
    sequences run in blocks of fewer heads than Hq: Hq = 10 on 5 KV heads
    (GQA groups of 2), sequences of 70,000 and 40,000 tokens (K and V of one
    KV head above 16 MiB: blocks of one group, 2 heads, so five blocks),
    shorter ones (all heads in one block), a one-token sequence and an empty
    one.  Sampled rows of every sequence and head (tile boundaries included)
    against the oracle."""
    from fa_util import run_gpu, sample_rows
    w = syn.packed_from_lengths("headblocks", [70000, 3000, 0, 40000, 512, 1], 10, 128, True, 1404,
                                Hkv=5).draw()
    o, lse, st = run_gpu(w)
    assert st == 0
    rows = sample_rows(w, early=2, tile_stride=64, n_random=3, seed=11)
    oo, lo = oracle.attention(w.q, w.k, w.v, w.B, w.Hq, w.Hkv, w.N, w.d, w.scale, w.causal, w.cu_seqlens,
                              rows=rows)
    assert_parity(o[rows], lse[rows], oo, lo, "packed head blocks")


def test_cuda_graph_replays():
    """A forward captured in a CUDA graph keeps its counter and epoch on every
    replay; the launch's last take puts the counter back to zero, so each
    replay computes every item: five replays give the eager call's output
    bitwise, on a dense shape (dynamic schedule: 1024 items) and a packed
    one."""
    import torch
    from exact_tiled_attention_32_b200 import binding as fa
    cases = [syn.Workload("graph-dense", 1, 32, 8, 16384, 64, True, 1405).draw(),
             syn.packed_from_lengths("graph-packed", [40000, 3000, 20000, 512], 8, 128, True, 1406, Hkv=4).draw()]
    for w in cases:
        q, k, v = to_device(w.q), to_device(w.k), to_device(w.v)
        cu = None if w.cu_seqlens is None else torch.from_numpy(w.cu_seqlens).cuda()
        ref_o, ref_lse = fa.attention_forward(q, k, v, causal=w.causal, scale=w.scale, cu_seqlens=cu)
        torch.cuda.synchronize()
        assert fa.fa_get_device_status() == fa.FA_OK
        o = torch.empty_like(ref_o)
        lse = torch.empty_like(ref_lse)
        g = torch.cuda.CUDAGraph()
        with torch.cuda.graph(g):
            s = torch.cuda.current_stream()
            rc = fa.fa_fwd(q, k, v, o, lse, w.B, w.Hq, w.Hkv, w.N, w.d, w.scale, w.causal, cu, s)
        assert rc == fa.FA_OK
        for i in range(5):
            o.fill_(7.0)
            g.replay()
            torch.cuda.synchronize()
            assert fa.fa_get_device_status() == fa.FA_OK, (w.name, i)
            assert torch.equal(o, ref_o) and torch.equal(lse, ref_lse), (w.name, i)
        del g


def test_partials_and_merge_under_the_dynamic_schedule():
    """fa_fwd_partial on a launch big enough for the dynamic schedule (2048
    items), over two key halves of a causal problem, merged with
    fa_merge_partials: O and lse equal fa_fwd's within the forward's
    tolerances, and sampled rows match the oracle."""
    import torch
    from exact_tiled_attention_32_b200 import binding as fa
    from fa_util import compare, gather, sample_rows
    w = syn.Workload("partials", 1, 32, 8, 16384, 128, True, 1407).draw()
    q, k, v = to_device(w.q), to_device(w.k), to_device(w.v)
    o_ref, lse_ref = fa.attention_forward(q, k, v, causal=True, scale=w.scale)
    s = torch.cuda.current_stream()
    half = w.N // 2
    rows = w.B * w.Hq * w.N
    o_parts = torch.empty((2, rows, w.d), dtype=torch.float32, device="cuda")
    lse_parts = torch.empty((2, rows), dtype=torch.float32, device="cuda")
    # share 0, keys [0, half): row t sees keys 0 .. min(t, half - 1): a causal
    # call for the rows below half, a non-causal one for the rows from half on
    kk, vv = k[:, :, :half].contiguous(), v[:, :, :half].contiguous()
    o0 = o_parts[0].view(w.B, w.Hq, w.N, w.d)
    l0 = lse_parts[0].view(w.B, w.Hq, w.N)
    qa, qb = q[:, :, :half].contiguous(), q[:, :, half:].contiguous()
    oa = torch.empty((w.B, w.Hq, half, w.d), dtype=torch.float32, device="cuda")
    la = torch.empty((w.B, w.Hq, half), dtype=torch.float32, device="cuda")
    ob, lb = torch.empty_like(oa), torch.empty_like(la)
    assert fa.fa_fwd_partial(qa, kk, vv, oa, la, w.B, w.Hq, w.Hkv, half, half, w.d, w.scale, 1, s) == fa.FA_OK
    assert fa.fa_fwd_partial(qb, kk, vv, ob, lb, w.B, w.Hq, w.Hkv, half, half, w.d, w.scale, 0, s) == fa.FA_OK
    o0[:, :, :half] = oa
    o0[:, :, half:] = ob
    l0[:, :, :half] = la
    l0[:, :, half:] = lb
    # share 1: keys [half, N): rows below half see none of them (-inf), rows t >= half see
    # keys half .. t: a causal chunk of half rows against half keys
    o1 = o_parts[1].view(w.B, w.Hq, w.N, w.d)
    l1 = lse_parts[1].view(w.B, w.Hq, w.N)
    o1[:, :, :half] = 0
    l1[:, :, :half] = float("-inf")
    kc, vc = k[:, :, half:].contiguous(), v[:, :, half:].contiguous()
    assert fa.fa_fwd_partial(qb, kc, vc, ob, lb, w.B, w.Hq, w.Hkv, half, half, w.d, w.scale, 1, s) == fa.FA_OK
    o1[:, :, half:] = ob
    l1[:, :, half:] = lb
    o = torch.empty_like(o_ref)
    lse = torch.empty_like(lse_ref)
    assert fa.fa_merge_partials(o_parts, lse_parts, 2, rows, w.d, o, lse, s) == fa.FA_OK
    torch.cuda.synchronize()
    assert fa.fa_get_device_status() == fa.FA_OK
    mx, mean, lmx = compare(*gather(w, o, lse), *gather(w, o_ref, lse_ref))
    assert mx <= 1e-2 and mean <= 1e-3 and lmx <= 1e-3, (mx, mean, lmx)
    sel = sample_rows(w, early=4, tile_stride=16, n_random=4, seed=12)
    oo, lo = oracle.attention(w.q, w.k, w.v, w.B, w.Hq, w.Hkv, w.N, w.d, w.scale, True, rows=sel)
    og, lg = gather(w, o, lse)
    assert_parity(og[sel], lg[sel], oo, lo, "merged partials")
