"""The size limits of the packed paths on B200: the forward and the backward
at the maximum of 1024 sequences (the schedule tables at capacity), a
sequence at the forward's maximum of 262,144 tokens (sampled rows), and one
token past it rejected on the device.  Tolerances as the other parity tests;
the 1024 short causal sequences have rows with one or two keys, whose O is
a V row (|O| up to ~4.5), so there the bf16-derived bound of the stress tests
applies (the rounding of O alone can reach 2^-8 |O| > 1e-2 there)."""
import numpy as np
import pytest

import oracle
from exact_tiled_attention_32_b200 import synthetic as syn
from fa_util import assert_bf16_bound, assert_parity, gather, softmax_weighted_abs_v, to_device

pytestmark = pytest.mark.gpu


def _lens(n, lo, hi, seed):
    return [int(x) for x in syn.Stream(seed).integers(lo, hi, n)]


def test_forward_1024_sequences():
    import torch
    from exact_tiled_attention_32_b200 import binding as fa
    lens = _lens(1024, 0, 40, 31)
    w = syn.packed_from_lengths("many", lens, 2, 64, True, 1300, Hkv=1).draw()
    cu = torch.from_numpy(w.cu_seqlens).cuda()
    o, lse = fa.attention_forward(to_device(w.q), to_device(w.k), to_device(w.v), causal=True, cu_seqlens=cu)
    torch.cuda.synchronize()
    assert fa.fa_get_device_status() == 0
    og, lg = gather(w, o, lse)
    oo, lo = oracle.attention(w.q, w.k, w.v, w.B, w.Hq, w.Hkv, w.N, w.d, w.scale, True, w.cu_seqlens)
    assert_bf16_bound(og, lg, oo, lo, softmax_weighted_abs_v(w, w.scale, True, lo), "1024 sequences")


def test_backward_1024_sequences():
    """dQ, dK, dV of every sequence against the oracle of that sequence, with
    the gradient bound of the backward tests."""
    import torch
    from exact_tiled_attention_32_b200 import binding as fa
    from test_gpu_bwd import _check, _d_terms
    lens = _lens(1024, 0, 24, 32)
    Hq, Hkv, d = 2, 1, 64
    w = syn.packed_from_lengths("many", lens, Hq, d, True, 1301, Hkv=Hkv).draw()
    do = syn.Stream(1302).normal_bf16(w.q_shape())
    cu = torch.from_numpy(w.cu_seqlens).cuda()
    q, k, v, dod = (to_device(a) for a in (w.q, w.k, w.v, do))
    o, lse = fa.attention_forward(q, k, v, causal=True, cu_seqlens=cu)
    dq, dk, dv = fa.attention_backward(q, k, v, o, lse, dod, causal=True, cu_seqlens=cu)
    torch.cuda.synchronize()
    assert fa.fa_get_device_status() == 0
    dq, dk, dv = (t.float().cpu().numpy().astype(np.float64) for t in (dq, dk, dv))
    for s_, L in enumerate(lens):
        if L == 0:
            continue
        a = int(w.cu_seqlens[s_])
        sl = slice(a, a + L)
        dense = lambda x: np.ascontiguousarray(x[sl].transpose(1, 0, 2)[None])
        args = (dense(w.q), dense(w.k), dense(w.v), dense(do), 1, Hq, Hkv, L, d, w.scale, True)
        rq, rk, rv = oracle.attention_bwd(*args)
        tq, tk = _d_terms(*args)
        _check(dq[sl].transpose(1, 0, 2), rq[0], f"dq seq {s_}", tq[0])
        _check(dk[sl].transpose(1, 0, 2), rk[0], f"dk seq {s_}", tk[0])
        _check(dv[sl].transpose(1, 0, 2), rv[0], f"dv seq {s_}")


def test_forward_longest_sequence():
    """A sequence of 262,144 tokens (1024 pairs of 128-row tiles, the limit of
    the packed schedule) followed by a short one: sampled rows of both."""
    import torch
    from exact_tiled_attention_32_b200 import binding as fa
    lens = [262144, 5]
    w = syn.packed_from_lengths("longest", lens, 1, 64, True, 1303).draw()
    cu = torch.from_numpy(w.cu_seqlens).cuda()
    o, lse = fa.attention_forward(to_device(w.q), to_device(w.k), to_device(w.v), causal=True, cu_seqlens=cu)
    torch.cuda.synchronize()
    assert fa.fa_get_device_status() == 0
    og, lg = gather(w, o, lse)
    rng = np.random.default_rng(4)
    rows = np.unique(np.concatenate([[0, 1, 127, 128, 255, 256, 262143, 262144, 262148],
                                     np.arange(0, 262144, 16384) + 127, rng.integers(0, w.N, 24)]))
    oo, lo = oracle.attention(w.q, w.k, w.v, w.B, w.Hq, w.Hkv, w.N, w.d, w.scale, True, w.cu_seqlens, rows=rows)
    assert_parity(og[rows], lg[rows], oo, lo, "262144-token sequence")


def test_sequence_past_the_limit_is_rejected_on_the_device():
    import torch
    from exact_tiled_attention_32_b200 import binding as fa
    N, H, d = 262145, 1, 64
    q = torch.zeros((N, H, d), dtype=torch.bfloat16, device="cuda")
    o = torch.full_like(q, 3.0)
    lse = torch.zeros((H, N), dtype=torch.float32, device="cuda")
    cu = torch.tensor([0, N], dtype=torch.int32, device="cuda")
    assert fa.fa_fwd(q, q, q, o, lse, 1, H, H, N, d, 0.125, 1, cu, torch.cuda.current_stream()) == 0
    assert fa.fa_get_device_status(torch.cuda.current_stream()) == fa.FA_ERR_SEQLENS
    assert torch.all(o == 3.0)
