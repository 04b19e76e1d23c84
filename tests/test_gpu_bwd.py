"""fa_bwd on B200: dQ, dK, dV compared with the fp64 oracle of the
gradients on the same bf16 inputs.  The GPU forward supplies O and the
logsumexp, as in training; the oracle differentiates the exact definition.

Tolerance: the forward's bound carried over to the gradients, plus the bf16
rounding of the result (the outputs are bf16): per element 1e-2 + 2^-7 |ref|
(one ulp), on average 1e-3 + 2^-8 mean |ref| (half an ulp), since gradients
are O(1) quantities formed from bf16-rounded P and dS, like O -- and a large
one (dV of a one-token sequence is the group's summed dO) is dominated by
its own output rounding.  dQ and dK also carry the rounding of the forward's
bf16 O inside D_i = sum_c dO_ic O_ic (the kernel, as in training, uses the O
the forward wrote): |dD_i| <= dD_i := 2^-9 sum_c |dO_ic O_ic|, which adds
scale dD_i sum_j P_ij |k_jc| to dQ_ic and scale sum_i P_ij dD_i |q_ic| to
dK_jc (P and O from the exact scores of the same inputs)."""
import numpy as np
import pytest

import oracle
from exact_tiled_attention_32_b200 import synthetic as syn
from fa_util import to_device

pytestmark = pytest.mark.gpu

MAX_ABS = 1e-2
MEAN_ABS = 1e-3


def _inputs(B, Hq, Hkv, N, d, seed):
    s = syn.Stream(seed)
    q = s.normal_bf16((B, Hq, N, d))
    k = s.normal_bf16((B, Hkv, N, d))
    v = s.normal_bf16((B, Hkv, N, d))
    do = s.normal_bf16((B, Hq, N, d))
    return q, k, v, do


def _gpu(q, k, v, do, causal, scale):
    import torch
    from exact_tiled_attention_32_b200 import binding as fa
    qd, kd, vd, dod = (to_device(a) for a in (q, k, v, do))
    o, lse = fa.attention_forward(qd, kd, vd, causal=causal, scale=scale)
    dq, dk, dv = fa.attention_backward(qd, kd, vd, o, lse, dod, causal=causal, scale=scale)
    torch.cuda.synchronize()
    assert fa.fa_get_device_status() == 0
    return tuple(t.float().cpu().numpy().astype(np.float64) for t in (dq, dk, dv))


def _d_terms(q, k, v, do, B, Hq, Hkv, N, d, scale, causal, heads=None):
    """The D-rounding terms of the module docstring: (dq_term [B, Hq, N, d],
    dk_term [B, Hkv, N, d]) in fp64, from the exact softmax of the inputs."""
    qf, kf, vf, dof = (syn.bf16_bits_to_float(a).astype(np.float64) for a in (q, k, v, do))
    g = Hq // Hkv
    tq = np.zeros((B, Hq, N, d))
    tk = np.zeros((B, Hkv, N, d))
    for b in range(B):
        for h in (range(Hq) if heads is None else heads):
            K, V = kf[b, h // g], vf[b, h // g]
            for r0 in range(0, N, 1024):
                r1 = min(N, r0 + 1024)
                s_ = scale * qf[b, h, r0:r1] @ K.T
                if causal:
                    s_ = np.where(np.arange(N)[None, :] <= np.arange(r0, r1)[:, None], s_, -np.inf)
                pm = np.exp(s_ - s_.max(axis=1, keepdims=True))
                pm /= pm.sum(axis=1, keepdims=True)
                o = pm @ V
                dd = 2.0 ** -9 * np.abs(dof[b, h, r0:r1] * o).sum(axis=1)
                tq[b, h, r0:r1] = scale * dd[:, None] * (pm @ np.abs(K))
                tk[b, h // g] += scale * pm.T @ (dd[:, None] * np.abs(qf[b, h, r0:r1]))
    return tq, tk


def _check(got, ref, what, extra=0.0):
    assert not np.isnan(got).any(), f"{what}: NaN"
    err = np.abs(got - ref)
    bound = MAX_ABS + 2.0 ** -7 * np.abs(ref) + extra
    assert (err - bound).max() <= 0, f"{what}: max error {err.max():.3e} (excess {(err - bound).max():.3e})"
    mean_bound = MEAN_ABS + 2.0 ** -8 * np.abs(ref).mean()
    assert err.mean() <= mean_bound, f"{what}: mean error {err.mean():.3e} > {mean_bound:.3e}"


CASES = [
    # B, Hq, Hkv, N, d, causal
    (1, 2, 2, 128, 128, True),
    (1, 2, 2, 128, 128, False),
    (1, 4, 2, 300, 128, True),        # GQA, ragged last block
    (2, 2, 1, 257, 64, False),
    (1, 2, 2, 1, 128, True),          # one token
    (1, 3, 3, 513, 128, False),
    (1, 8, 2, 1000, 64, True),
    (2, 2, 2, 640, 128, True),
]


@pytest.mark.parametrize("B,Hq,Hkv,N,d,causal", CASES)
def test_bwd_matches_oracle(B, Hq, Hkv, N, d, causal):
    q, k, v, do = _inputs(B, Hq, Hkv, N, d, 900 + N + d)
    scale = 1.0 / np.sqrt(d)
    dq, dk, dv = _gpu(q, k, v, do, causal, scale)
    rq, rk, rv = oracle.attention_bwd(q, k, v, do, B, Hq, Hkv, N, d, scale, causal)
    tq, tk = _d_terms(q, k, v, do, B, Hq, Hkv, N, d, scale, causal)
    tag = f"{B},{Hq},{Hkv},{N},{d},{causal}"
    _check(dq, rq, f"dq {tag}", tq)
    _check(dk, rk, f"dk {tag}", tk)
    _check(dv, rv, f"dv {tag}")


def test_bwd_dk_dv_are_deterministic_and_workspace_reusable():
    import torch
    from exact_tiled_attention_32_b200 import binding as fa
    B, Hq, Hkv, N, d = 1, 4, 2, 700, 128
    q, k, v, do = (to_device(a) for a in _inputs(B, Hq, Hkv, N, d, 950))
    o, lse = fa.attention_forward(q, k, v, causal=True)
    ws = torch.empty(fa.fa_bwd_workspace_bytes(B, Hq, N, d), dtype=torch.uint8, device="cuda")
    ws.fill_(0xFF)                  # nothing in the workspace needs initialising
    a = fa.attention_backward(q, k, v, o, lse, do, causal=True, workspace=ws)
    b = fa.attention_backward(q, k, v, o, lse, do, causal=True, workspace=ws)
    torch.cuda.synchronize()
    assert torch.equal(a[1], b[1]) and torch.equal(a[2], b[2])
    assert (a[0].float() - b[0].float()).abs().max().item() <= 2.0 ** -6


def test_bwd_argument_errors():
    from exact_tiled_attention_32_b200 import binding as fa
    p = 1 << 20
    args = dict(B=1, Hq=4, Hkv=2, N=100, d=128, scale=0.1, causal=1)

    def call(ptrs=(p,) * 9, ws=p, wb=1 << 30, **kw):
        a = dict(args)
        a.update(kw)
        return fa.fa_bwd(*ptrs, a["B"], a["Hq"], a["Hkv"], a["N"], a["d"], a["scale"], a["causal"], None, ws, wb)

    assert call(d=96) == fa.FA_ERR_HEADDIM
    assert call(Hkv=3) == fa.FA_ERR_GQA
    assert call(ws=0) == fa.FA_ERR_NULL
    assert call(ws=p + 8) == fa.FA_ERR_ALIGN
    assert call(wb=fa.fa_bwd_workspace_bytes(1, 4, 100, 128) - 1) == fa.FA_ERR_SHAPE
    assert call(ptrs=(p,) * 6 + (0, p, p)) == fa.FA_ERR_NULL
    assert call(N=0, ptrs=(0,) * 9, ws=0, wb=0) == fa.FA_OK


def test_bwd_c3_shape_one_head():
    """The backward at the bench's size (causal, H=32, N=16384, d=128): all of
    dQ, dK, dV of head 5 against the oracle, and finiteness everywhere."""
    w = syn.config("c3").draw()
    s = syn.Stream(w.seed + 77)
    do = s.normal_bf16(w.q_shape())
    dq, dk, dv = _gpu(w.q, w.k, w.v, do, True, w.scale)
    assert np.isfinite(dq).all() and np.isfinite(dk).all() and np.isfinite(dv).all()
    h = 5
    rq, rk, rv = oracle.attention_bwd(w.q, w.k, w.v, do, w.B, w.Hq, w.Hkv, w.N, w.d, w.scale, True, units=[h])
    tq, tk = _d_terms(w.q, w.k, w.v, do, w.B, w.Hq, w.Hkv, w.N, w.d, w.scale, True, heads=[h])
    _check(dq[0, h], rq[0, 0], "c3 dq head 5", tq[0, h])
    _check(dk[0, h], rk[0], "c3 dk head 5", tk[0, h])
    _check(dv[0, h], rv[0], "c3 dv head 5")


PACKED_CASES = [
    # lengths, Hq, Hkv, d, causal
    ([130, 1, 300, 128, 7], 4, 2, 128, True),
    ([256, 0, 200], 2, 2, 64, False),
    ([1000, 129], 2, 1, 128, True),
    ([64] * 9, 3, 3, 128, True),
]


@pytest.mark.parametrize("lens,Hq,Hkv,d,causal", PACKED_CASES)
def test_bwd_packed_matches_oracle(lens, Hq, Hkv, d, causal):
    """Packed variable-length batches ([N, H, d], cu_seqlens): each sequence's
    gradients against the oracle of that sequence alone."""
    import torch
    from exact_tiled_attention_32_b200 import binding as fa
    w = syn.packed_from_lengths("pk", lens, Hq, d, causal, 960 + sum(lens), Hkv=Hkv).draw()
    do = syn.Stream(961).normal_bf16(w.q_shape())
    scale = 1.0 / np.sqrt(d)
    q, k, v, dod = (to_device(a) for a in (w.q, w.k, w.v, do))
    cu = torch.from_numpy(w.cu_seqlens).cuda()
    o, lse = fa.attention_forward(q, k, v, causal=causal, scale=scale, cu_seqlens=cu)
    dq, dk, dv = fa.attention_backward(q, k, v, o, lse, dod, causal=causal, scale=scale, cu_seqlens=cu)
    torch.cuda.synchronize()
    assert fa.fa_get_device_status() == 0
    dq, dk, dv = (t.float().cpu().numpy().astype(np.float64) for t in (dq, dk, dv))
    for s_, L in enumerate(lens):
        if L == 0:
            continue
        a = int(w.cu_seqlens[s_])
        sl = slice(a, a + L)
        # this sequence as a dense B = 1 problem: [L, H, d] -> [1, H, L, d]
        dense = lambda x: np.ascontiguousarray(x[sl].transpose(1, 0, 2)[None])
        rq, rk, rv = oracle.attention_bwd(dense(w.q), dense(w.k), dense(w.v), dense(do), 1, Hq, Hkv, L, d, scale,
                                          causal)
        tq, tk = _d_terms(dense(w.q), dense(w.k), dense(w.v), dense(do), 1, Hq, Hkv, L, d, scale, causal)
        tag = f"packed {lens} seq {s_}"
        _check(dq[sl].transpose(1, 0, 2), rq[0], f"dq {tag}", tq[0])
        _check(dk[sl].transpose(1, 0, 2), rk[0], f"dk {tag}", tk[0])
        _check(dv[sl].transpose(1, 0, 2), rv[0], f"dv {tag}")


def test_bwd_packed_bad_offsets_are_reported():
    import torch
    from exact_tiled_attention_32_b200 import binding as fa
    w = syn.packed_from_lengths("pk", [100, 50], 2, 128, True, 970).draw()
    q, k, v = (to_device(a) for a in (w.q, w.k, w.v))
    cu = torch.from_numpy(w.cu_seqlens).cuda()
    o, lse = fa.attention_forward(q, k, v, causal=True, cu_seqlens=cu)
    torch.cuda.synchronize()
    bad = torch.tensor([0, 120, 100], dtype=torch.int32, device="cuda")      # decreasing offsets
    fa.attention_backward(q, k, v, o, lse, o, causal=True, cu_seqlens=bad)
    torch.cuda.synchronize()
    assert fa.fa_get_device_status() == fa.FA_ERR_SEQLENS
