"""fa_fwd_fp8 on B200: E4M3 Q, K, V with per-tensor scales, compared with the
fp64 oracle of attention on the dequantised inputs.

Tolerance (per output element, derived from the arithmetic): the forward's
1e-2, plus one bf16 rounding of O (2^-7 |O|), plus the E4M3 rounding of P for
the P V product.  The kernel computes P = 2^SHIFT exp2(x - m_ref) against a
reference m_ref that is never above the row's final maximum m and never more
than THRESHOLD (log2 units) below the scores it is applied to, with
SHIFT + THRESHOLD = 8.75, so P <= 2^8.75 < 448 (E4M3's largest value).
Every entry with exp(s - m) >= 2^-(6 + SHIFT) of the final maximum then has
P >= 2^-6, a normal E4M3 number (relative error <= 2^-4); an entry below that
is off by at most half the subnormal step, 2^-10 in P units, i.e. at most
2^-(10 + SHIFT) in units of the final maximum.  After the division by the
row sum l = sum_j exp(s_j - m):
|dO_c| <= 1e-2 + 2^-7 |O_c| + 2^-4 sum_j p_j |v_jc| + 2^-(10+SHIFT) sum_{tiny j} |v_jc| / l.
The weights p, l and the tiny set come from the exact scores of the
dequantised inputs.  The kernel's THRESHOLD is 3 (SHIFT 5.75).

Mean bound (over the compared elements): the worst case above adds every
weight's rounding error with the same sign; the mean error is checked
against the typical size instead.  Taking the E4M3 rounding errors d_j of
the weights as independent and zero-mean, each at most 2^-4 relative and
uniform within its rounding interval (E[d_j^2] <= 2^-8 / 3), the P V term
of column c has the root-mean-square size
    r_c = 2^-4 / sqrt(3) * sqrt(sum_j p_j^2 v_jc^2),
which bounds its mean absolute value.  So
    mean |dO| <= 1e-3 + mean(2^-8 |O| + 3 r + tiny term),
the benchmark spec's mean-abs 1e-3, the worst case of the bf16 rounding of O
(round to nearest: 2^-8 relative) and of the tiny weights, and three times
the typical P V rounding error as the margin for a finite sample."""
import numpy as np
import pytest

import oracle
from exact_tiled_attention_32_b200 import synthetic as syn

pytestmark = pytest.mark.gpu

S = syn.FP8_SCALE
F8_SHIFT = 5.75          # the kernel's P scaling (log2); tiny: below 2^-(6 + F8_SHIFT) of the row maximum


def _dev(codes):
    import torch
    return torch.from_numpy(np.ascontiguousarray(codes)).cuda()


def _run(w):
    import torch
    from exact_tiled_attention_32_b200 import binding as fa
    o, lse = fa.attention_forward_fp8(_dev(w.q), _dev(w.k), _dev(w.v), S, S, S, causal=w.causal, scale=w.scale)
    torch.cuda.synchronize()
    assert fa.fa_get_device_status() == 0
    return o.float().cpu().numpy().astype(np.float64).reshape(-1, w.d), lse.cpu().numpy().astype(np.float64).reshape(-1)


def _bound(w, rows, o_ref):
    """Per-element worst-case tolerance of the rows (see the module
    docstring) and the per-element terms of the mean bound."""
    qf = oracle.e4m3_decode(w.q).reshape(-1, w.d) * S
    kf = oracle.e4m3_decode(w.k).reshape(w.B, w.Hkv, w.N, w.d) * S
    vf = oracle.e4m3_decode(w.v).reshape(w.B, w.Hkv, w.N, w.d) * S
    g = w.Hq // w.Hkv
    out = np.empty((len(rows), w.d))
    rms = np.empty((len(rows), w.d))
    tiny_t = np.empty((len(rows), w.d))
    for n, rid in enumerate(rows):
        t = rid % w.N
        bh = rid // w.N
        b, h = divmod(bh, w.Hq)
        keys = t + 1 if w.causal else w.N
        K = kf[b, h // g, :keys]
        V = np.abs(vf[b, h // g, :keys])
        s = w.scale * (K @ qf[rid])
        e = np.exp(s - s.max())
        l = e.sum()
        tiny = e < 2.0 ** -(6 + F8_SHIFT)
        tiny_t[n] = 2.0 ** -(10 + F8_SHIFT) * V[tiny].sum(axis=0) / l
        out[n] = 2.0 ** -4 * (e / l) @ V + tiny_t[n]
        rms[n] = 2.0 ** -4 / np.sqrt(3.0) * np.sqrt(((e / l) ** 2) @ (V ** 2))
    worst = 1e-2 + 2.0 ** -7 * np.abs(o_ref) + out
    mean_terms = 2.0 ** -8 * np.abs(o_ref) + 3.0 * rms + tiny_t
    return worst, mean_terms


def _check(w, o, lse, rows, what):
    o_ref, l_ref = oracle.attention_fp8(w.q, w.k, w.v, S, S, S, w.B, w.Hq, w.Hkv, w.N, w.d, w.scale, w.causal,
                                        rows=rows)
    got = o[rows]
    assert not np.isnan(got).any(), f"{what}: NaN"
    err = np.abs(got - o_ref)
    worst, mean_terms = _bound(w, rows, o_ref)
    excess = err - worst
    assert excess.max() <= 0, f"{what}: O error {err.max():.3e} exceeds the E4M3 bound by {excess.max():.3e}"
    mean_bound = 1e-3 + mean_terms.mean()
    assert err.mean() <= mean_bound, f"{what}: O mean error {err.mean():.3e} > derived {mean_bound:.3e}"
    lerr = np.abs(lse[rows] - l_ref)
    assert lerr.max() <= 1e-3, f"{what}: lse error {lerr.max():.3e}"


CASES = [
    # B, Hq, Hkv, N, causal, d
    (1, 2, 2, 256, False, 128),
    (1, 2, 2, 256, True, 128),
    (1, 4, 2, 300, True, 128),      # GQA, ragged last tile
    (2, 2, 1, 1000, True, 128),
    (1, 3, 3, 129, False, 128),
    # d = 64: 64-byte rows, read into the 128-byte tiles with zero columns
    (1, 2, 2, 256, False, 64),
    (1, 4, 2, 300, True, 64),
    (2, 2, 1, 1000, True, 64),
    (1, 3, 3, 129, False, 64),
]


@pytest.mark.parametrize("B,Hq,Hkv,N,causal,d", CASES)
def test_fp8_all_rows(B, Hq, Hkv, N, causal, d):
    w = syn.Workload("fp8", B, Hq, Hkv, N, d, causal, 1100 + N + d, fp8=True).draw()
    o, lse = _run(w)
    _check(w, o, lse, np.arange(B * Hq * N), f"fp8 {B},{Hq},{Hkv},{N},{causal},d={d}")


PACKED = [
    # lengths, Hq, Hkv, causal, d
    ([300, 1, 129, 0, 513], 4, 2, True, 128),
    ([300, 1, 129, 0, 513], 4, 2, False, 128),
    ([128, 256, 77], 2, 1, True, 128),
    ([300, 1, 129, 0, 513], 4, 2, True, 64),
    ([128, 256, 77], 2, 1, False, 64),
]


@pytest.mark.parametrize("lens,Hq,Hkv,causal,d", PACKED)
def test_fp8_packed_every_sequence(lens, Hq, Hkv, causal, d):
    """fa_fwd_fp8_varlen against the oracle, sequence by sequence: each
    sequence's rows are compared with those of the dense problem of that
    sequence alone, under the same per-element and mean bounds."""
    import torch
    from exact_tiled_attention_32_b200 import binding as fa
    w = syn.packed_from_lengths("fp8p", lens, Hq, d, causal, 1200 + sum(lens) + d, Hkv=Hkv)
    w.fp8 = True
    w.draw()
    cu = torch.from_numpy(w.cu_seqlens).cuda()
    o, lse = fa.attention_forward_fp8(_dev(w.q), _dev(w.k), _dev(w.v), S, S, S, causal=causal, scale=w.scale,
                                      cu_seqlens=cu)
    torch.cuda.synchronize()
    assert fa.fa_get_device_status() == 0
    o = o.float().cpu().numpy().astype(np.float64)          # [N, Hq, d]
    lse = lse.cpu().numpy().astype(np.float64)               # [Hq, N]
    for s_, L in enumerate(lens):
        if L == 0:
            continue
        a = int(w.cu_seqlens[s_])
        ws = syn.Workload("fp8seq", 1, Hq, Hkv, L, d, causal, 0, fp8=True)
        ws.q = np.ascontiguousarray(w.q[a:a + L].transpose(1, 0, 2)[None])
        ws.k = np.ascontiguousarray(w.k[a:a + L].transpose(1, 0, 2)[None])
        ws.v = np.ascontiguousarray(w.v[a:a + L].transpose(1, 0, 2)[None])
        od = o[a:a + L].transpose(1, 0, 2).reshape(-1, d)
        ld = lse[:, a:a + L].reshape(-1)
        _check(ws, od, ld, np.arange(Hq * L), f"fp8 packed {lens} seq {s_} d={d}")


def test_fp8_varlen_argument_errors():
    from exact_tiled_attention_32_b200 import binding as fa
    p = 1 << 20
    call = lambda B=2, d=128, cu=p, ptrs=(p, p, p, p, p): fa.fa_fwd_fp8_varlen(*ptrs, B, 2, 2, 128, d, 0.1, 1,
                                                                               1, 1, 1, cu)
    assert call(d=96) == fa.FA_ERR_HEADDIM
    assert call(cu=0) == fa.FA_ERR_NULL
    assert call(cu=p + 2) == fa.FA_ERR_ALIGN
    assert call(B=1025) == fa.FA_ERR_SHAPE
    assert call(B=0, cu=0, ptrs=(0,) * 5) == fa.FA_OK


def test_fp8_argument_errors():
    from exact_tiled_attention_32_b200 import binding as fa
    p = 1 << 20
    assert fa.fa_fwd_fp8(p, p, p, p, p, 1, 2, 2, 128, 96, 0.1, 1, 1, 1, 1) == fa.FA_ERR_HEADDIM
    assert fa.fa_fwd_fp8(p, p, p, p, p, 1, 2, 2, 128, 128, 0.1, 1, 0, 1, 1) == fa.FA_ERR_SHAPE
    assert fa.fa_fwd_fp8(p, p, p, p, p, 1, 2, 2, 128, 128, 0.1, 1, 1, float("inf"), 1) == fa.FA_ERR_SHAPE
    assert fa.fa_fwd_fp8(p, p, p, p, p, 1, 4, 3, 128, 128, 0.1, 1, 1, 1, 1) == fa.FA_ERR_GQA
    assert fa.fa_fwd_fp8(0, 0, 0, 0, 0, 0, 2, 2, 128, 128, 0.1, 1, 1, 1, 1) == fa.FA_OK


def test_c3f8_sampled_rows():
    """The FP8 workload the bench times (c3's shape in E4M3): sampled rows of
    every head, tile boundaries included."""
    from fa_util import sample_rows
    w = syn.config("c3f8").draw()
    o, lse = _run(w)
    rows = sample_rows(w, early=4, tile_stride=16, n_random=4, seed=8)
    _check(w, o, lse, rows, "c3f8")


def test_c2f8_sampled_rows():
    """FP8 at d = 64 on c2's non-causal shape (the bench's c2f8): sampled rows
    of every head, tile boundaries included."""
    from fa_util import sample_rows
    w = syn.config("c2f8").draw()
    o, lse = _run(w)
    rows = sample_rows(w, early=4, tile_stride=4, n_random=8, seed=10)
    _check(w, o, lse, rows, "c2f8")


def test_c5f8_sampled_rows():
    """The packed FP8 workload the bench times (c5's 16 sequences in E4M3),
    sequence by sequence: the first rows, the first and last row of every
    eighth tile and random rows of every head, against the oracle of that
    sequence's dense problem under the same bounds."""
    import torch
    from exact_tiled_attention_32_b200 import binding as fa
    w = syn.config("c5f8").draw()
    cu = torch.from_numpy(w.cu_seqlens).cuda()
    o, lse = fa.attention_forward_fp8(_dev(w.q), _dev(w.k), _dev(w.v), S, S, S, causal=True, scale=w.scale,
                                      cu_seqlens=cu)
    torch.cuda.synchronize()
    assert fa.fa_get_device_status() == 0
    o = o.float().cpu().numpy().astype(np.float64)
    lse = lse.cpu().numpy().astype(np.float64)
    rng = np.random.default_rng(9)
    for s_, L in enumerate(w.lengths):
        a = int(w.cu_seqlens[s_])
        ws = syn.Workload("fp8seq", 1, w.Hq, w.Hkv, L, 128, True, 0, fp8=True)
        ws.q = np.ascontiguousarray(w.q[a:a + L].transpose(1, 0, 2)[None])
        ws.k = np.ascontiguousarray(w.k[a:a + L].transpose(1, 0, 2)[None])
        ws.v = np.ascontiguousarray(w.v[a:a + L].transpose(1, 0, 2)[None])
        od = o[a:a + L].transpose(1, 0, 2).reshape(-1, 128)
        ld = lse[:, a:a + L].reshape(-1)
        ts = set(range(4)) | {L - 1} | set(rng.integers(0, L, 3).tolist())
        for m in range(0, (L + 127) // 128, 8):
            ts.update((128 * m, min(128 * m + 127, L - 1)))
        rows = np.array(sorted(h * L + t for h in range(w.Hq) for t in ts))
        _check(ws, od, ld, rows, f"c5f8 seq {s_} (L={L})")
