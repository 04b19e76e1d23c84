"""fa_fwd_kvcache on B200: a chunk of Nq queries (the last Nq positions)
against Nk keys, compared with the fp64 oracle, and the chunked-prefill
identity (chunks of a sequence against all earlier keys give the rows of the
whole causal forward).  Tolerances as the other parity tests."""
import numpy as np
import pytest

import oracle
from exact_tiled_attention_32_b200 import synthetic as syn
from fa_util import assert_parity, sample_rows, to_device

pytestmark = pytest.mark.gpu


def _run(w):
    import torch
    from exact_tiled_attention_32_b200 import binding as fa
    o, lse = fa.attention_forward_kvcache(to_device(w.q), to_device(w.k), to_device(w.v),
                                          causal=w.causal, scale=w.scale)
    torch.cuda.synchronize()
    assert fa.fa_get_device_status() == 0
    return o.float().cpu().numpy().astype(np.float64).reshape(-1, w.d), lse.cpu().numpy().astype(np.float64).reshape(-1)


CASES = [
    # B, Hq, Hkv, Nq, Nk, d, causal
    (1, 4, 2, 1, 1000, 128, True),        # one decode step against a cache
    (2, 4, 4, 5, 300, 64, True),
    (1, 8, 2, 128, 4096, 128, True),
    (1, 2, 2, 200, 777, 128, True),
    (1, 4, 4, 384, 384, 64, True),        # Nq == Nk: the plain forward
    (2, 2, 1, 100, 513, 128, False),
    (1, 2, 2, 257, 1024, 64, True),
    (1, 3, 1, 300, 301, 128, True),
]


@pytest.mark.parametrize("B,Hq,Hkv,Nq,Nk,d,causal", CASES)
def test_chunk_all_rows(B, Hq, Hkv, Nq, Nk, d, causal):
    w = syn.Workload("chunk", B, Hq, Hkv, Nq, d, causal, 700 + Nq + Nk, Nk=Nk).draw()
    o, lse = _run(w)
    oo, lo = oracle.attention_kv(w.q, w.k, w.v, B, Hq, Hkv, Nq, Nk, d, w.scale, causal)
    assert_parity(o, lse, oo, lo, f"chunk {B},{Hq},{Hkv},{Nq},{Nk},{d},{causal}")


def test_chunked_prefill_matches_whole_forward():
    import torch
    from exact_tiled_attention_32_b200 import binding as fa
    B, H, N, d = 1, 4, 1000, 128
    w = syn.Workload("whole", B, H, H, N, d, True, 750).draw()
    q, k, v = to_device(w.q), to_device(w.k), to_device(w.v)
    o_full, l_full = fa.attention_forward(q, k, v, causal=True)
    parts_o, parts_l = [], []
    for a, b in ((0, 130), (130, 512), (512, 999), (999, 1000)):
        o, l = fa.attention_forward_kvcache(q[:, :, a:b], k[:, :, :b], v[:, :, :b], causal=True)
        parts_o.append(o)
        parts_l.append(l)
    torch.cuda.synchronize()
    o_chunks = torch.cat(parts_o, dim=2).float()
    l_chunks = torch.cat(parts_l, dim=2)
    assert (o_chunks - o_full.float()).abs().max().item() <= 1e-2
    assert (l_chunks - l_full).abs().max().item() <= 1e-3
    oo, lo = oracle.attention(w.q, w.k, w.v, B, H, H, N, d, w.scale, True)
    from fa_util import compare
    mx, mean, lmx = compare(o_chunks.cpu().numpy().astype(np.float64).reshape(-1, d),
                            l_chunks.cpu().numpy().astype(np.float64).reshape(-1), oo, lo)
    assert mx <= 1e-2 and mean <= 1e-3 and lmx <= 1e-3


PACKED = [
    # (Lq, Lk) per sequence, Hq, Hkv, d, causal
    ([(1, 1000), (130, 130), (0, 77), (200, 777), (257, 1024)], 4, 2, 128, True),
    ([(5, 300), (128, 4096), (1, 1)], 2, 1, 64, True),
    ([(100, 513), (7, 9), (0, 0), (300, 301)], 2, 2, 128, False),
]


@pytest.mark.parametrize("pairs,Hq,Hkv,d,causal", PACKED)
def test_packed_chunks_every_sequence(pairs, Hq, Hkv, d, causal):
    """fa_fwd_kvcache_varlen: each sequence's chunk against its own keys,
    compared with the oracle of that sequence's dense chunk problem."""
    import torch
    from exact_tiled_attention_32_b200 import binding as fa
    lq = [a for a, _ in pairs]
    lk = [b for _, b in pairs]
    Nq, Nk = sum(lq), sum(lk)
    st = syn.Stream(900 + Nq + Nk)
    qb = st.normal_bf16((Nq, Hq, d))
    kb = st.normal_bf16((Nk, Hkv, d))
    vb = st.normal_bf16((Nk, Hkv, d))
    cq = np.concatenate([[0], np.cumsum(lq)]).astype(np.int32)
    ck = np.concatenate([[0], np.cumsum(lk)]).astype(np.int32)
    scale = 1.0 / np.sqrt(d)
    o, lse = fa.attention_forward_kvcache(to_device(qb), to_device(kb), to_device(vb), causal=causal, scale=scale,
                                          cu_seqlens_q=torch.from_numpy(cq).cuda(),
                                          cu_seqlens_k=torch.from_numpy(ck).cuda())
    torch.cuda.synchronize()
    assert fa.fa_get_device_status() == 0
    o = o.float().cpu().numpy().astype(np.float64)
    lse = lse.cpu().numpy().astype(np.float64)
    for s_, (Lq, Lk) in enumerate(pairs):
        if Lq == 0:
            continue
        a, b = int(cq[s_]), int(ck[s_])
        dense = lambda x, lo, n: np.ascontiguousarray(x[lo:lo + n].transpose(1, 0, 2)[None])
        oo, lo = oracle.attention_kv(dense(qb, a, Lq), dense(kb, b, Lk), dense(vb, b, Lk), 1, Hq, Hkv, Lq, Lk, d,
                                     scale, causal)
        got_o = o[a:a + Lq].transpose(1, 0, 2).reshape(-1, d)
        got_l = lse[:, a:a + Lq].reshape(-1)
        assert_parity(got_o, got_l, oo, lo, f"packed chunk seq {s_} ({Lq} x {Lk})")


def test_packed_chunks_bad_offsets_reported_by_device():
    import torch
    from exact_tiled_attention_32_b200 import binding as fa
    H, d = 2, 64
    q = torch.zeros((20, H, d), dtype=torch.bfloat16, device="cuda")
    kv = torch.zeros((30, H, d), dtype=torch.bfloat16, device="cuda")
    o = torch.full_like(q, 3.0)
    lse = torch.zeros((H, 20), dtype=torch.float32, device="cuda")
    s = torch.cuda.current_stream()
    good_q = torch.tensor([0, 10, 20], dtype=torch.int32, device="cuda")
    for cq, ck in (([0, 10, 20], [0, 5, 30]),     # causal: 10 rows against 5 keys
                   ([0, 10, 20], [0, 15, 29]),    # keys do not total Nk
                   ([0, 10, 20], [1, 15, 30]),    # keys do not start at 0
                   ([0, 12, 20], [0, 25, 30])):   # causal: 8 rows against 5 keys
        cqt = torch.tensor(cq, dtype=torch.int32, device="cuda")
        ckt = torch.tensor(ck, dtype=torch.int32, device="cuda")
        assert fa.fa_fwd_kvcache_varlen(q, kv, kv, o, lse, 2, H, H, 20, 30, d, 0.1, 1, cqt, ckt, s) == fa.FA_OK
        assert fa.fa_get_device_status(s) == fa.FA_ERR_SEQLENS, (cq, ck)
        assert torch.all(o == 3.0)
    ok_k = torch.tensor([0, 15, 30], dtype=torch.int32, device="cuda")
    assert fa.fa_fwd_kvcache_varlen(q, kv, kv, o, lse, 2, H, H, 20, 30, d, 0.1, 1, good_q, ok_k, s) == fa.FA_OK
    assert fa.fa_get_device_status(s) == fa.FA_OK


def test_chunk_argument_errors():
    from exact_tiled_attention_32_b200 import binding as fa
    p = 1 << 20
    assert fa.fa_fwd_kvcache(p, p, p, p, p, 1, 2, 2, 10, 5, 64, 0.1, 1) == fa.FA_ERR_SHAPE   # causal, Nk < Nq
    assert fa.fa_fwd_kvcache(p, p, p, p, p, 1, 2, 2, 10, 0, 64, 0.1, 0) == fa.FA_ERR_SHAPE   # no keys
    assert fa.fa_fwd_kvcache(0, 0, 0, 0, 0, 1, 2, 2, 0, 5, 64, 0.1, 1) == fa.FA_OK          # empty chunk
    assert fa.fa_fwd_kvcache(p, p, p, p, p, 1, 2, 2, 4, 5, 96, 0.1, 1) == fa.FA_ERR_HEADDIM


def test_p3_sampled_rows():
    """The chunk workload the bench times: 2048 rows against 16384 keys."""
    w = syn.config("p3").draw()
    o, lse = _run(w)
    rng = np.random.default_rng(3)
    rows = []
    for h in range(w.Hq):
        base = h * w.N
        ts = set(range(4)) | {w.N - 1} | set(rng.integers(0, w.N, 12).tolist())
        ts |= {128 * m for m in range(0, w.N // 128, 4)}
        rows.extend(base + t for t in sorted(ts))
    rows = np.array(rows)
    oo, lo = oracle.attention_kv(w.q, w.k, w.v, w.B, w.Hq, w.Hkv, w.N, w.Nk, w.d, w.scale, True, rows=rows)
    assert_parity(o[rows], lse[rows], oo, lo, "p3")
