"""Pins for the fp64 oracle (CPU only).

Each test checks the oracle against something other than itself: the worked
examples the pages print, closed forms, torch's fp64 scaled-dot-product
attention (an independent library routine), brute force with no max shift on
tiny shapes, and identities the pages state (tiled == untiled, any block order).
The last group plants plausible mistakes into a copy of oracle.c and checks that
the pins catch every one of them.
"""
import json
import math
import os
import shutil
import subprocess

import numpy as np
import pytest
import torch

import oracle
from exact_tiled_attention_32_b200 import synthetic as syn

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")


def _bits(shape, seed):
    return syn.Stream(seed).normal_bf16(shape)


def _f64(bits):
    return syn.bf16_bits_to_float(bits).astype(np.float64)


# --------------------------------------------------------------------------
# worked examples of the pages
# --------------------------------------------------------------------------

def test_worked_example_row_1_5_3():
    """14cs17 page, Worked Examples, Example 2: [1,5] then [3] gives the
    softmax of the whole row [1,5,3]."""
    g = json.load(open(os.path.join(GOLDEN, "worked_example_online_softmax.json")))
    row = np.array(g["row"])
    lens = [len(b) for b in g["blocks"]]
    p_whole, lse_whole = oracle.softmax(row)
    for order in (None, [1, 0]):
        p_blk, lse_blk = oracle.online_softmax(row, lens, order)
        assert np.max(np.abs(p_blk - p_whole)) < 1e-15
        assert abs(lse_blk - lse_whole) < 1e-15
    # closed form, factoring out the maximum 5 by hand:
    # p(5) = 1 / (1 + e^-4 + e^-2), p(1) = e^-4 p(5), p(3) = e^-2 p(5)
    den = 1.0 + math.exp(-4.0) + math.exp(-2.0)
    expect = np.array([math.exp(-4.0) / den, 1.0 / den, math.exp(-2.0) / den])
    assert np.max(np.abs(p_whole - expect)) < 1e-15
    assert abs(lse_whole - (5.0 + math.log(den))) < 1e-15
    # the other split of the same row
    p_blk, _ = oracle.online_softmax(row, [1, 2])
    assert np.max(np.abs(p_blk - expect)) < 1e-15


def test_xspy_verification_chunks():
    """xspy.com page, section 3: the three-chunk check, max diff < 1e-15."""
    g = json.load(open(os.path.join(GOLDEN, "xspy_online_softmax.json")))
    chunks = g["data_chunks"]
    flat = np.array([x for c in chunks for x in c])
    p_std, lse_std = oracle.softmax(flat)
    p_onl, lse_onl = oracle.online_softmax(flat, [len(c) for c in chunks])
    assert np.max(np.abs(p_std - p_onl)) < g["max_abs_diff"]
    assert abs(p_std.sum() - 1.0) < 1e-15
    # the largest entry is 4.8, the fifth element
    assert int(np.argmax(p_std)) == 4
    # closed form of the normaliser: lse = log(sum e^x)
    assert abs(lse_std - math.log(sum(math.exp(x) for x in flat))) < 1e-14


# --------------------------------------------------------------------------
# softmax invariants
# --------------------------------------------------------------------------

def test_online_softmax_any_blocking_any_order():
    rng = np.random.default_rng(7)
    for n in (1, 2, 5, 17, 40):
        x = rng.normal(0, 3, n)
        p_whole, lse_whole = oracle.softmax(x)
        assert abs(p_whole.sum() - 1.0) < 1e-12
        for bs in range(1, n + 1):
            lens = [bs] * (n // bs) + ([n % bs] if n % bs else [])
            order = rng.permutation(len(lens))
            p, lse = oracle.online_softmax(x, lens, order)
            assert np.max(np.abs(p - p_whole)) < 1e-15
            assert abs(lse - lse_whole) < 1e-13
            assert abs(p.sum() - 1.0) < 1e-12


def test_online_softmax_minus_inf_guard():
    """A leading block of -inf only (an empty prefix) contributes nothing."""
    x = np.array([-np.inf, -np.inf, 2.0, 0.0])
    p, lse = oracle.online_softmax(x, [2, 2])
    e = math.exp(-2.0)
    assert np.allclose(p, [0, 0, 1 / (1 + e), e / (1 + e)], atol=1e-15, rtol=0)
    assert abs(lse - (2.0 + math.log1p(e))) < 1e-15
    p, lse = oracle.online_softmax(np.full(3, -np.inf), [1, 2])
    assert np.all(p == 0) and lse == -np.inf
    p, lse = oracle.softmax(np.full(3, -np.inf))
    assert np.all(p == 0) and lse == -np.inf


def test_softmax_shift_invariance_and_large_values():
    x = np.array([1000.0, 1001.0, 999.0])
    p, lse = oracle.softmax(x)
    p0, lse0 = oracle.softmax(x - 1000.0)
    assert np.max(np.abs(p - p0)) < 1e-15
    assert abs(lse - (lse0 + 1000.0)) < 1e-12


# --------------------------------------------------------------------------
# attention: library routine, brute force, closed forms
# --------------------------------------------------------------------------

def _torch_reference(q, k, v, B, Hq, Hkv, N, d, scale, causal, cu=None):
    """torch's scaled_dot_product_attention in fp64 on the CPU (its math path)
    plus torch.logsumexp of the masked scaled scores; returns the oracle's row
    order."""
    def one(qs, ks, vs):      # qs [Hq, L, d], ks/vs [Hkv, L, d]
        g = Hq // Hkv
        kr = ks.repeat_interleave(g, dim=0)
        vr = vs.repeat_interleave(g, dim=0)
        o = torch.nn.functional.scaled_dot_product_attention(
            qs[None], kr[None], vr[None], is_causal=causal, scale=scale)[0]
        s = scale * qs @ kr.transpose(-1, -2)
        if causal:
            L = qs.shape[1]
            mask = torch.ones(L, L, dtype=torch.bool).tril()
            s = s.masked_fill(~mask, -math.inf)
        return o, torch.logsumexp(s, dim=-1)

    qt, kt, vt = (torch.from_numpy(_f64(a)) for a in (q, k, v))
    if cu is None:
        os_, ls_ = [], []
        for b in range(B):
            o, l = one(qt[b], kt[b], vt[b])
            os_.append(o)
            ls_.append(l)
        return torch.stack(os_).reshape(-1, d).numpy(), torch.stack(ls_).reshape(-1).numpy()
    o_all = np.zeros((Hq, N, d))
    l_all = np.zeros((Hq, N))
    for s in range(len(cu) - 1):
        a, e = int(cu[s]), int(cu[s + 1])
        if a == e:
            continue
        o, l = one(qt[a:e].transpose(0, 1), kt[a:e].transpose(0, 1), vt[a:e].transpose(0, 1))
        o_all[:, a:e] = o.numpy()
        l_all[:, a:e] = l.numpy()
    return o_all.reshape(-1, d), l_all.reshape(-1)


@pytest.mark.parametrize("B,Hq,Hkv,N,d,causal", [
    (2, 4, 4, 37, 64, False),
    (2, 4, 4, 37, 64, True),
    (1, 4, 2, 130, 128, True),
    (1, 8, 2, 129, 64, False),
    (2, 2, 1, 1, 16, True),
    (1, 3, 3, 200, 8, True),
])
def test_attention_matches_torch_fp64(B, Hq, Hkv, N, d, causal):
    s = syn.Stream(11 + N + d)
    q = s.normal_bf16((B, Hq, N, d))
    k = s.normal_bf16((B, Hkv, N, d))
    v = s.normal_bf16((B, Hkv, N, d))
    scale = 1 / math.sqrt(d)
    o, lse = oracle.attention(q, k, v, B, Hq, Hkv, N, d, scale, causal)
    o_t, lse_t = _torch_reference(q, k, v, B, Hq, Hkv, N, d, scale, causal)
    assert np.max(np.abs(o - o_t)) < 1e-12
    assert np.max(np.abs(lse - lse_t)) < 1e-12


@pytest.mark.parametrize("lens,Hq,Hkv,causal", [
    ([5, 1, 130, 64], 4, 2, True),
    ([129, 0, 7], 2, 2, False),
    ([1], 1, 1, True),
])
def test_packed_attention_matches_torch_fp64(lens, Hq, Hkv, causal):
    d = 32
    w = syn.packed_from_lengths("t", lens, Hq, d, causal, 77, Hkv=Hkv).draw()
    cu = w.cu_seqlens
    o, lse = oracle.attention(w.q, w.k, w.v, w.B, Hq, Hkv, w.N, d, w.scale, causal, cu)
    o_t, lse_t = _torch_reference(w.q, w.k, w.v, w.B, Hq, Hkv, w.N, d, w.scale, causal, cu)
    assert np.max(np.abs(o - o_t)) < 1e-12
    assert np.max(np.abs(lse - lse_t)) < 1e-12


def _brute(q, k, v, scale, causal, group):
    """Pure-Python attention with no max shift: O = sum e^s v / sum e^s."""
    Hq, L, d = len(q), len(q[0]), len(q[0][0])
    o = [[[0.0] * d for _ in range(L)] for _ in range(Hq)]
    lse = [[0.0] * L for _ in range(Hq)]
    for h in range(Hq):
        hk = h // group
        for i in range(L):
            num = [0.0] * d
            den = 0.0
            for j in range(L):
                if causal and j > i:
                    continue
                sc = scale * sum(q[h][i][c] * k[hk][j][c] for c in range(d))
                w = math.exp(sc)
                den += w
                for c in range(d):
                    num[c] += w * v[hk][j][c]
            o[h][i] = [x / den for x in num]
            lse[h][i] = math.log(den)
    return o, lse


@pytest.mark.parametrize("causal", [False, True])
@pytest.mark.parametrize("Hq,Hkv", [(2, 2), (4, 2), (3, 1)])
def test_attention_brute_force_tiny(causal, Hq, Hkv):
    B, N, d = 2, 7, 4
    s = syn.Stream(5 + Hq)
    q = s.normal_bf16((B, Hq, N, d))
    k = s.normal_bf16((B, Hkv, N, d))
    v = s.normal_bf16((B, Hkv, N, d))
    scale = 0.7
    o, lse = oracle.attention(q, k, v, B, Hq, Hkv, N, d, scale, causal)
    o = o.reshape(B, Hq, N, d)
    lse = lse.reshape(B, Hq, N)
    for b in range(B):
        ob, lb = _brute(_f64(q[b]).tolist(), _f64(k[b]).tolist(), _f64(v[b]).tolist(),
                        scale, causal, Hq // Hkv)
        assert np.max(np.abs(o[b] - np.array(ob))) < 1e-12
        assert np.max(np.abs(lse[b] - np.array(lb))) < 1e-12


def test_packed_brute_force_tiny():
    lens = [3, 1, 6]
    Hq, Hkv, d = 2, 1, 3
    w = syn.packed_from_lengths("t", lens, Hq, d, True, 9, Hkv=Hkv).draw()
    o, lse = oracle.attention(w.q, w.k, w.v, w.B, Hq, Hkv, w.N, d, 0.9, True, w.cu_seqlens)
    o = o.reshape(Hq, w.N, d)
    lse = lse.reshape(Hq, w.N)
    cu = w.cu_seqlens
    for s in range(len(lens)):
        a, e = cu[s], cu[s + 1]
        qs = _f64(w.q[a:e]).transpose(1, 0, 2).tolist()
        ks = _f64(w.k[a:e]).transpose(1, 0, 2).tolist()
        vs = _f64(w.v[a:e]).transpose(1, 0, 2).tolist()
        ob, lb = _brute(qs, ks, vs, 0.9, True, Hq // Hkv)
        assert np.max(np.abs(o[:, a:e] - np.array(ob))) < 1e-12
        assert np.max(np.abs(lse[:, a:e] - np.array(lb))) < 1e-12


def test_closed_form_causal_first_row():
    """Causal row 0 sees only key 0: O = v_0 exactly, lse = scale q_0.k_0."""
    B, H, N, d = 1, 2, 50, 64
    s = syn.Stream(3)
    q, k, v = (s.normal_bf16((B, H, N, d)) for _ in range(3))
    scale = 0.125
    o, lse = oracle.attention(q, k, v, B, H, H, N, d, scale, True)
    o = o.reshape(B, H, N, d)
    lse = lse.reshape(B, H, N)
    for h in range(H):
        assert np.array_equal(o[0, h, 0], _f64(v[0, h, 0]))
        expect = scale * float(np.dot(_f64(q[0, h, 0]), _f64(k[0, h, 0])))
        assert abs(lse[0, h, 0] - expect) < 1e-13


def test_closed_form_zero_queries():
    """All-zero Q: every allowed key has score 0, so O is the mean of the
    allowed V rows and lse = ln(count)."""
    B, H, N, d = 1, 1, 33, 16
    s = syn.Stream(4)
    q = np.zeros((B, H, N, d), dtype=np.uint16)       # +0.0 in bf16
    k, v = s.normal_bf16((B, H, N, d)), s.normal_bf16((B, H, N, d))
    vf = _f64(v[0, 0])
    for causal in (False, True):
        o, lse = oracle.attention(q, k, v, B, H, H, N, d, 1.0, causal)
        for i in range(N):
            cnt = i + 1 if causal else N
            assert np.max(np.abs(o[i] - vf[:cnt].mean(axis=0))) < 1e-14
            assert abs(lse[i] - math.log(cnt)) < 1e-14


def test_closed_form_dominant_key():
    """One key aligned with the query and a huge scale: O is that key's V."""
    N, d = 9, 8
    q = np.zeros((1, 1, N, d))
    k = np.zeros((1, 1, N, d))
    q[0, 0, :, 0] = 1.0
    k[0, 0, 4, 0] = 1.0                   # key 4 scores 1, the rest 0
    v = syn.Stream(6).normal_bf16((1, 1, N, d))
    qb, kb = syn.fp64_to_bf16_bits(q), syn.fp64_to_bf16_bits(k)
    o, lse = oracle.attention(qb, kb, v, 1, 1, 1, N, d, 1000.0, False)
    assert np.max(np.abs(o - _f64(v[0, 0, 4])[None])) < 1e-12
    assert np.max(np.abs(lse - 1000.0)) < 1e-12


def test_rows_subset_matches_full():
    w = syn.Workload("t", 2, 4, 2, 100, 32, True, 21).draw()
    o, lse = oracle.attention(w.q, w.k, w.v, w.B, w.Hq, w.Hkv, w.N, w.d, w.scale, True)
    rows = np.array([0, 99, 100, 555, 799])
    o2, lse2 = oracle.attention(w.q, w.k, w.v, w.B, w.Hq, w.Hkv, w.N, w.d, w.scale, True,
                                rows=rows)
    assert np.array_equal(o[rows], o2) and np.array_equal(lse[rows], lse2)
    with pytest.raises(ValueError):
        oracle.attention(w.q, w.k, w.v, w.B, w.Hq, w.Hkv, w.N, w.d, w.scale, True,
                         rows=np.array([w.total_rows()]))


def test_gqa_equals_mha_with_repeated_kv():
    B, Hq, Hkv, N, d = 1, 8, 2, 40, 16
    s = syn.Stream(8)
    q = s.normal_bf16((B, Hq, N, d))
    k, v = s.normal_bf16((B, Hkv, N, d)), s.normal_bf16((B, Hkv, N, d))
    o1, l1 = oracle.attention(q, k, v, B, Hq, Hkv, N, d, 0.25, True)
    kr, vr = np.repeat(k, Hq // Hkv, axis=1), np.repeat(v, Hq // Hkv, axis=1)
    o2, l2 = oracle.attention(q, kr, vr, B, Hq, Hq, N, d, 0.25, True)
    assert np.array_equal(o1, o2) and np.array_equal(l1, l2)


def test_packed_single_sequence_equals_dense():
    N, H, d = 70, 2, 16
    w = syn.packed_from_lengths("t", [N], H, d, True, 12).draw()
    o_p, l_p = oracle.attention(w.q, w.k, w.v, 1, H, H, N, d, w.scale, True, w.cu_seqlens)
    qd, kd, vd = (np.ascontiguousarray(a.transpose(1, 0, 2))[None] for a in (w.q, w.k, w.v))
    o_d, l_d = oracle.attention(qd, kd, vd, 1, H, H, N, d, w.scale, True)
    assert np.array_equal(o_p, o_d) and np.array_equal(l_p, l_d)


# --------------------------------------------------------------------------
# tiled (online) attention == materialised attention
# --------------------------------------------------------------------------

@pytest.mark.parametrize("br,bc", [(1, 1), (3, 3), (128, 128), (5, 128), (128, 7)])
def test_tiled_equals_untiled(br, bc):
    """14cs17 page, 'Flash Attention Algorithm' and Pitfall 1: the tiled
    forward is exact -- any tile sizes, any order of the key blocks."""
    B, Hq, Hkv, N, d = 1, 4, 2, 150, 32
    s = syn.Stream(31)
    q = s.normal_bf16((B, Hq, N, d))
    k, v = s.normal_bf16((B, Hkv, N, d)), s.normal_bf16((B, Hkv, N, d))
    rng = np.random.default_rng(br * 1000 + bc)
    for causal in (False, True):
        o, lse = oracle.attention(q, k, v, B, Hq, Hkv, N, d, 0.2, causal)
        nblk = (N + bc - 1) // bc
        for order in (None, rng.permutation(nblk)):
            o_t, lse_t = oracle.attention_tiled(q, k, v, B, Hq, Hkv, N, d, 0.2, causal,
                                                br=br, bc=bc, kv_order=order)
            assert np.max(np.abs(o - o_t)) < 1e-12
            assert np.max(np.abs(lse - lse_t)) < 1e-12


def test_tiled_equals_untiled_packed():
    w = syn.packed_from_lengths("t", [130, 3, 257], 2, 16, True, 41).draw()
    o, lse = oracle.attention(w.q, w.k, w.v, w.B, 2, 2, w.N, 16, w.scale, True, w.cu_seqlens)
    o_t, lse_t = oracle.attention_tiled(w.q, w.k, w.v, w.B, 2, 2, w.N, 16, w.scale, True,
                                        w.cu_seqlens, br=128, bc=64)
    assert np.max(np.abs(o - o_t)) < 1e-12
    assert np.max(np.abs(lse - lse_t)) < 1e-12


def test_sampled_p_rows_sum_to_one():
    """The P row of the oracle (O with V = identity columns) sums to 1."""
    N, d = 24, 24
    s = syn.Stream(51)
    q, k = s.normal_bf16((1, 1, N, d)), s.normal_bf16((1, 1, N, d))
    eye = syn.fp64_to_bf16_bits(np.eye(N, d)[None, None])
    for causal in (False, True):
        p, _ = oracle.attention(q, k, eye, 1, 1, 1, N, d, 0.5, causal)
        assert np.max(np.abs(p.sum(axis=1) - 1.0)) < 1e-12
        if causal:
            assert np.all(np.triu(p, 1) == 0)


# --------------------------------------------------------------------------
# planted mistakes: every one must break at least one pin
# --------------------------------------------------------------------------

MUTATIONS = {
    "dropped_scale": ("s[j] = scale * dot;", "s[j] = dot;"),
    "causal_off_by_one": ("return !a->causal || j <= r->t;", "return !a->causal || j < r->t + 1 - (r->t > 0);"),
    "gqa_interleaved": ("r->hk = r->h / group;\n        r->len = N;", "r->hk = r->h % a->Hkv;\n        r->len = N;"),
    "lse_without_max": ("lse[i] = m + log(l);", "lse[i] = log(l);"),
    "k_read_from_v": ("const uint16_t* kj = r.k0 + j * r.kv_stride;", "const uint16_t* kj = r.v0 + j * r.kv_stride;"),
    "flipped_shift": ("s[j] = exp(s[j] - m);", "s[j] = exp(m - s[j]);"),
    "transposed_row_col": ("r->qrow = a->q + ((b * a->Hq + r->h) * N + r->t) * a->d;",
                           "r->qrow = a->q + ((b * a->Hq + r->h) * N) * a->d + r->t;"),
    "online_no_rescale": ("double carry = (m_run == -INFINITY) ? 0.0 : exp(m_run - m_new);",
                          "double carry = (m_run == -INFINITY) ? 0.0 : 1.0;"),
    "chunk_top_left_mask": ("const int64_t pos = (int64_t)Nk - Nq + i;", "const int64_t pos = i;"),
    "bwd_dq_without_scale": ("dqi[c] += scale * ds * Kw[j * d + c];", "dqi[c] += ds * Kw[j * d + c];"),
    "bwd_D_without_p": ("D += p[j] * dp[j];", "D += dp[j];"),
    "bwd_dk_from_dout": ("dkj[c] += scale * ds * qi[c];", "dkj[c] += scale * ds * doi[c];"),
    "bwd_dv_from_q": ("dvj[c] += pij * doi[c];", "dvj[c] += pij * qi[c];"),
    "bwd_flipped_ds": ("const double ds = pij * (dp - Dr[gi]);", "const double ds = pij * (Dr[gi] - dp);"),
    "bwd_causal_keys_from_zero": ("for (int64_t i = causal ? j : 0; i < N; ++i) {",
                                  "for (int64_t i = 0; i < N; ++i) {"),
}


def _pin_suite(lib):
    """The pins above, run against another build of the oracle; returns the
    names of the pins that fail."""
    failed = []
    checks = {
        "example": lambda: np.max(np.abs(
            oracle.online_softmax([1.0, 5.0, 3.0], [2, 1], lib=lib)[0]
            - oracle.softmax([1.0, 5.0, 3.0])[0])) < 1e-15,
        "xspy": lambda: np.max(np.abs(
            oracle.online_softmax([1.2, 3.4, 0.5, 2.1, 4.8, 1.1, 3.2, 0.9, 2.7], [3, 3, 3], lib=lib)[0]
            - oracle.softmax([1.2, 3.4, 0.5, 2.1, 4.8, 1.1, 3.2, 0.9, 2.7])[0])) < 1e-15,
    }

    def torch_pin(B, Hq, Hkv, N, d, causal):
        s = syn.Stream(11 + N + d)
        q = s.normal_bf16((B, Hq, N, d))
        k = s.normal_bf16((B, Hkv, N, d))
        v = s.normal_bf16((B, Hkv, N, d))
        o, lse = oracle.attention(q, k, v, B, Hq, Hkv, N, d, 0.125, causal, lib=lib)
        o_t, lse_t = _torch_reference(q, k, v, B, Hq, Hkv, N, d, 0.125, causal)
        return np.max(np.abs(o - o_t)) < 1e-12 and np.max(np.abs(lse - lse_t)) < 1e-12

    checks["torch_causal_gqa"] = lambda: torch_pin(1, 4, 2, 37, 16, True)
    checks["torch_dense"] = lambda: torch_pin(2, 2, 2, 20, 16, False)

    def chunk_pin():
        s = syn.Stream(99)
        q = s.normal_bf16((1, 2, 5, 16))
        k = s.normal_bf16((1, 1, 23, 16))
        v = s.normal_bf16((1, 1, 23, 16))
        o, lse = oracle.attention_kv(q, k, v, 1, 2, 1, 5, 23, 16, 0.3, True, lib=lib)
        o_t, lse_t = _torch_chunk(q, k, v, 1, 2, 1, 5, 23, 16, 0.3, True)
        return np.max(np.abs(o - o_t)) < 1e-12 and np.max(np.abs(lse - lse_t)) < 1e-12

    checks["torch_chunk"] = chunk_pin

    def bwd_pin(B, Hq, Hkv, N, d, causal):
        s = syn.Stream(31 + N)
        q = s.normal_bf16((B, Hq, N, d))
        k = s.normal_bf16((B, Hkv, N, d))
        v = s.normal_bf16((B, Hkv, N, d))
        do = s.normal_bf16((B, Hq, N, d))
        got = oracle.attention_bwd(q, k, v, do, B, Hq, Hkv, N, d, 0.3, causal, lib=lib)
        ref = _torch_bwd(q, k, v, do, B, Hq, Hkv, N, d, 0.3, causal)
        return all(np.max(np.abs(a - b)) < 1e-12 for a, b in zip(got, ref))

    checks["torch_bwd_causal_gqa"] = lambda: bwd_pin(1, 4, 2, 23, 8, True)
    checks["torch_bwd_dense"] = lambda: bwd_pin(1, 2, 2, 11, 8, False)
    for name, fn in checks.items():
        try:
            ok = bool(fn())
        except Exception:
            ok = False
        if not ok:
            failed.append(name)
    return failed


def test_pins_pass_on_the_real_oracle():
    assert _pin_suite(oracle._load()) == []


@pytest.mark.parametrize("name", sorted(MUTATIONS))
def test_planted_mistake_is_caught(name, tmp_path):
    if shutil.which("gcc") is None:
        pytest.skip("gcc not available")
    old, new = MUTATIONS[name]
    src = open(oracle._SRC).read()
    assert old in src, f"mutation anchor for {name} not found"
    path = tmp_path / "oracle_mut.c"
    path.write_text(src.replace(old, new, 1))
    so = tmp_path / "liboracle_mut.so"
    subprocess.check_call(["gcc", "-O2", "-fopenmp", "-shared", "-fPIC", "-std=c11",
                           str(path), "-o", str(so), "-lm"])
    failed = _pin_suite(oracle.bind(str(so)))
    assert failed, f"planted mistake {name} passed every pin"


# --------------------------------------------------------------------------
# a chunk of queries against a longer key sequence (chunked prefill)
# --------------------------------------------------------------------------

def _torch_chunk(q, k, v, B, Hq, Hkv, Nq, Nk, d, scale, causal):
    """torch fp64 SDPA with an explicit mask: row i of the chunk may see key
    j iff j <= Nk - Nq + i (bottom-right alignment)."""
    qt, kt, vt = (torch.from_numpy(_f64(a)) for a in (q, k, v))
    g = Hq // Hkv
    kr, vr = kt.repeat_interleave(g, dim=1), vt.repeat_interleave(g, dim=1)
    mask = None
    if causal:
        i = torch.arange(Nq)[:, None]
        j = torch.arange(Nk)[None, :]
        mask = j <= (Nk - Nq + i)
    o = torch.nn.functional.scaled_dot_product_attention(qt, kr, vr, attn_mask=mask, scale=scale)
    s = scale * qt @ kr.transpose(-1, -2)
    if causal:
        s = s.masked_fill(~mask, -math.inf)
    return o.reshape(-1, d).numpy(), torch.logsumexp(s, dim=-1).reshape(-1).numpy()


@pytest.mark.parametrize("B,Hq,Hkv,Nq,Nk,d,causal", [
    (2, 4, 2, 5, 37, 16, True),
    (1, 4, 4, 37, 37, 32, True),
    (1, 2, 1, 1, 130, 64, True),
    (2, 2, 2, 20, 50, 16, False),
    (1, 8, 2, 129, 300, 32, True),
])
def test_chunk_attention_matches_torch_fp64(B, Hq, Hkv, Nq, Nk, d, causal):
    s = syn.Stream(61 + Nq + Nk)
    q = s.normal_bf16((B, Hq, Nq, d))
    k = s.normal_bf16((B, Hkv, Nk, d))
    v = s.normal_bf16((B, Hkv, Nk, d))
    o, lse = oracle.attention_kv(q, k, v, B, Hq, Hkv, Nq, Nk, d, 0.3, causal)
    o_t, lse_t = _torch_chunk(q, k, v, B, Hq, Hkv, Nq, Nk, d, 0.3, causal)
    assert np.max(np.abs(o - o_t)) < 1e-12
    assert np.max(np.abs(lse - lse_t)) < 1e-12


def test_chunk_brute_force_tiny():
    B, Hq, Hkv, Nq, Nk, d = 1, 2, 1, 3, 7, 4
    s = syn.Stream(71)
    q = s.normal_bf16((B, Hq, Nq, d))
    k = s.normal_bf16((B, Hkv, Nk, d))
    v = s.normal_bf16((B, Hkv, Nk, d))
    o, lse = oracle.attention_kv(q, k, v, B, Hq, Hkv, Nq, Nk, d, 0.8, True)
    qf, kf, vf = _f64(q[0]), _f64(k[0]), _f64(v[0])
    for h in range(Hq):
        for i in range(Nq):
            pos = Nk - Nq + i
            w = [math.exp(0.8 * float(np.dot(qf[h, i], kf[0, j]))) for j in range(pos + 1)]
            ref = sum(wj * vf[0, j] for j, wj in enumerate(w)) / sum(w)
            r = h * Nq + i
            assert np.max(np.abs(o[r] - ref)) < 1e-12
            assert abs(lse[r] - math.log(sum(w))) < 1e-12


def test_chunk_equal_lengths_is_the_plain_forward():
    B, H, N, d = 2, 3, 70, 16
    s = syn.Stream(72)
    q, k, v = (s.normal_bf16((B, H, N, d)) for _ in range(3))
    for causal in (False, True):
        o1, l1 = oracle.attention(q, k, v, B, H, H, N, d, 0.25, causal)
        o2, l2 = oracle.attention_kv(q, k, v, B, H, H, N, N, d, 0.25, causal)
        assert np.array_equal(o1, o2) and np.array_equal(l1, l2)


def test_chunked_prefill_reproduces_the_whole_causal_forward():
    """xspy.com page, section 1: prefill split into chunks, each chunk's
    queries attending to the keys of all tokens up to its end, gives the rows
    of the whole causal forward."""
    B, H, N, d = 1, 2, 100, 16
    s = syn.Stream(73)
    q, k, v = (s.normal_bf16((B, H, N, d)) for _ in range(3))
    o_full, l_full = oracle.attention(q, k, v, B, H, H, N, d, 0.25, True)
    o_full = o_full.reshape(B, H, N, d)
    l_full = l_full.reshape(B, H, N)
    for a, b in ((0, 17), (17, 64), (64, 100)):
        qc = np.ascontiguousarray(q[:, :, a:b])
        kc = np.ascontiguousarray(k[:, :, :b])
        vc = np.ascontiguousarray(v[:, :, :b])
        o, l = oracle.attention_kv(qc, kc, vc, B, H, H, b - a, b, d, 0.25, True)
        assert np.array_equal(o.reshape(B, H, b - a, d), o_full[:, :, a:b])
        assert np.array_equal(l.reshape(B, H, b - a), l_full[:, :, a:b])


# --------------------------------------------------------------------------
# gradients (the backward pass): dQ, dK, dV of the forward's definition
# --------------------------------------------------------------------------

def _torch_bwd(q, k, v, dout, B, Hq, Hkv, N, d, scale, causal):
    """torch.autograd in fp64 through an explicit masked softmax (an
    independent differentiation of the same definition)."""
    qt, kt, vt = (torch.from_numpy(_f64(a)).requires_grad_(True) for a in (q, k, v))
    g = Hq // Hkv
    kr, vr = kt.repeat_interleave(g, dim=1), vt.repeat_interleave(g, dim=1)
    s = scale * qt @ kr.transpose(-1, -2)
    if causal:
        mask = torch.ones(N, N, dtype=torch.bool).tril()
        s = s.masked_fill(~mask, -math.inf)
    o = torch.softmax(s, dim=-1) @ vr
    o.backward(torch.from_numpy(_f64(dout)))
    return qt.grad.numpy(), kt.grad.numpy(), vt.grad.numpy()


@pytest.mark.parametrize("B,Hq,Hkv,N,d,causal", [
    (1, 4, 2, 37, 16, True),
    (2, 2, 2, 20, 16, False),
    (1, 3, 1, 9, 8, True),
    (1, 2, 1, 1, 8, True),
])
def test_bwd_matches_torch_autograd(B, Hq, Hkv, N, d, causal):
    s = syn.Stream(81 + N + d)
    q = s.normal_bf16((B, Hq, N, d))
    k = s.normal_bf16((B, Hkv, N, d))
    v = s.normal_bf16((B, Hkv, N, d))
    do = s.normal_bf16((B, Hq, N, d))
    dq, dk, dv = oracle.attention_bwd(q, k, v, do, B, Hq, Hkv, N, d, 0.3, causal)
    tq, tk, tv = _torch_bwd(q, k, v, do, B, Hq, Hkv, N, d, 0.3, causal)
    assert np.max(np.abs(dq - tq)) < 1e-12
    assert np.max(np.abs(dk - tk)) < 1e-12
    assert np.max(np.abs(dv - tv)) < 1e-12


def test_bwd_central_differences():
    """Brute-force derivative of L = sum(dO * O), O from the oracle forward:
    inputs are multiples of 1/8, so x +- 1/64 is exact in bf16; the central
    difference error is O(h^2)."""
    B, Hq, Hkv, N, d, scale = 1, 2, 1, 5, 4, 0.7
    rng = np.random.default_rng(5)

    def grid(shape):
        return rng.integers(-8, 9, size=shape).astype(np.float64) / 8.0

    qf, kf, vf = grid((B, Hq, N, d)), grid((B, Hkv, N, d)), grid((B, Hkv, N, d))
    do = syn.fp64_to_bf16_bits(grid((B, Hq, N, d)))
    dof = _f64(do).reshape(-1, d)
    bits = syn.fp64_to_bf16_bits
    h = 1.0 / 64
    for causal in (False, True):
        def loss(qx, kx, vx):
            o, _ = oracle.attention(bits(qx), bits(kx), bits(vx), B, Hq, Hkv, N, d, scale, causal)
            return float(np.sum(o * dof))

        dq, dk, dv = oracle.attention_bwd(bits(qf), bits(kf), bits(vf), do, B, Hq, Hkv, N, d, scale, causal)
        for which, base, grad in (("q", qf, dq), ("k", kf, dk), ("v", vf, dv)):
            for idx in np.ndindex(base.shape):
                xp, xm = base.copy(), base.copy()
                xp[idx] += h
                xm[idx] -= h
                args_p = {"q": (xp, kf, vf), "k": (qf, xp, vf), "v": (qf, kf, xp)}[which]
                args_m = {"q": (xm, kf, vf), "k": (qf, xm, vf), "v": (qf, kf, xm)}[which]
                fd = (loss(*args_p) - loss(*args_m)) / (2 * h)
                assert abs(fd - grad[idx]) < 2e-3, (which, idx, fd, grad[idx], causal)


def test_bwd_invariants():
    """Every softmax row sums to one, so sum_j dS_ij = 0: the key gradients of
    a (sequence, kv head) sum to zero, and the value gradients sum to the
    upstream gradients of the query rows (of all heads in the group)."""
    B, Hq, Hkv, N, d = 2, 4, 2, 50, 16
    s = syn.Stream(91)
    q = s.normal_bf16((B, Hq, N, d))
    k = s.normal_bf16((B, Hkv, N, d))
    v = s.normal_bf16((B, Hkv, N, d))
    do = s.normal_bf16((B, Hq, N, d))
    for causal in (False, True):
        dq, dk, dv = oracle.attention_bwd(q, k, v, do, B, Hq, Hkv, N, d, 0.25, causal)
        assert np.max(np.abs(dk.sum(axis=2))) < 1e-11
        dos = _f64(do).reshape(B, Hkv, Hq // Hkv, N, d).sum(axis=(2, 3))
        assert np.max(np.abs(dv.sum(axis=2) - dos)) < 1e-11


def test_bwd_single_visible_key():
    """Causal row 0 sees only key 0: P = [1], so dS = 0 there, and with N = 1
    dQ = dK = 0 while dV = the group's summed dO."""
    B, Hq, Hkv, N, d = 1, 3, 1, 1, 8
    s = syn.Stream(92)
    q, k, v = s.normal_bf16((B, Hq, N, d)), s.normal_bf16((B, Hkv, N, d)), s.normal_bf16((B, Hkv, N, d))
    do = s.normal_bf16((B, Hq, N, d))
    dq, dk, dv = oracle.attention_bwd(q, k, v, do, B, Hq, Hkv, N, d, 0.5, True)
    assert np.all(dq == 0) and np.all(dk == 0)
    assert np.max(np.abs(dv[0, 0] - _f64(do)[0].sum(axis=0))) < 1e-15


def test_bwd_units_subset():
    B, Hq, Hkv, N, d = 2, 4, 2, 30, 8
    s = syn.Stream(93)
    q = s.normal_bf16((B, Hq, N, d))
    k = s.normal_bf16((B, Hkv, N, d))
    v = s.normal_bf16((B, Hkv, N, d))
    do = s.normal_bf16((B, Hq, N, d))
    dq, dk, dv = oracle.attention_bwd(q, k, v, do, B, Hq, Hkv, N, d, 0.4, True)
    sq, sk, sv = oracle.attention_bwd(q, k, v, do, B, Hq, Hkv, N, d, 0.4, True, units=[3, 0])
    assert np.array_equal(sq[0], dq[1, 2:4]) and np.array_equal(sq[1], dq[0, 0:2])
    assert np.array_equal(sk[0], dk[1, 1]) and np.array_equal(sv[1], dv[0, 0])


# --------------------------------------------------------------------------
# FP8 (E4M3) inputs
# --------------------------------------------------------------------------

def test_e4m3_decode_matches_torch_on_every_code():
    codes = np.arange(256, dtype=np.uint8)
    ref = torch.from_numpy(codes).view(torch.float8_e4m3fn).to(torch.float64).numpy()
    got = oracle.e4m3_decode(codes)
    nan = np.isnan(ref)
    assert np.array_equal(np.isnan(got), nan) and nan.sum() == 2
    assert np.array_equal(got[~nan], ref[~nan])


def test_e4m3_encoder_of_the_inputs_round_trips():
    """The input generator's encoder and the oracle's decoder agree: decoding
    an encoded value gives the nearest E4M3 value (checked against torch's
    rounding), and re-encoding a decoded code gives the code back."""
    x = np.random.default_rng(7).normal(size=20000) * 60
    codes = syn.fp64_to_e4m3_bits(x)
    ref = torch.from_numpy(x).to(torch.float8_e4m3fn).to(torch.float64).numpy()
    assert np.array_equal(oracle.e4m3_decode(codes), ref)
    finite = np.array([c for c in range(256) if c not in (0x7F, 0xFF)], dtype=np.uint8)
    assert np.array_equal(syn.fp64_to_e4m3_bits(oracle.e4m3_decode(finite)), finite)


def test_fp8_attention_brute_force():
    """Tiny E4M3 problem against a pure-Python evaluation of softmax(QK^T)V
    on torch-decoded inputs (no max shift)."""
    B, Hq, Hkv, N, d, scale = 1, 2, 1, 6, 8, 0.35
    s = syn.Stream(5)
    inv = 32.0
    q8, k8, v8 = s.normal_e4m3((B, Hq, N, d), inv), s.normal_e4m3((B, Hkv, N, d), inv), s.normal_e4m3((B, Hkv, N, d), inv)
    dec = lambda a: torch.from_numpy(a).view(torch.float8_e4m3fn).to(torch.float64).numpy() / inv
    qf, kf, vf = dec(q8)[0], dec(k8)[0], dec(v8)[0]
    for causal in (False, True):
        o, lse = oracle.attention_fp8(q8, k8, v8, 1 / inv, 1 / inv, 1 / inv, B, Hq, Hkv, N, d, scale, causal)
        for h in range(Hq):
            for i in range(N):
                keys = range(i + 1) if causal else range(N)
                w = [math.exp(scale * float(np.dot(qf[h, i], kf[0, j]))) for j in keys]
                ref = sum(wj * vf[0, j] for wj, j in zip(w, keys)) / sum(w)
                assert np.max(np.abs(o[h * N + i] - ref)) < 1e-12
                assert abs(lse[h * N + i] - math.log(sum(w))) < 1e-12


def test_fp8_attention_rejects_inexact_scales():
    q8 = np.full((1, 1, 2, 4), 0x39, dtype=np.uint8)     # 1.125
    with pytest.raises(ValueError):
        oracle.attention_fp8(q8, q8, q8, 0.1, 1.0, 1.0, 1, 1, 1, 2, 4, 1.0, False)


@pytest.mark.parametrize("old,new", [
    ("np.exp2(e.astype(np.float64) - 7.0)", "np.exp2(e.astype(np.float64) - 8.0)"),     # exponent bias
    ("m * 2.0 ** -9", "m * 2.0 ** -10"),                                                   # subnormal step
    ("(1.0 + m / 8.0)", "(1.0 + m / 16.0)"),                                               # mantissa width
])
def test_planted_mistake_in_e4m3_decode_is_caught(old, new, tmp_path):
    """Each mistake planted into a copy of the oracle's decoder breaks the
    torch pin."""
    import importlib.util
    src = open(os.path.join(os.path.dirname(oracle.__file__), "__init__.py")).read()
    assert old in src
    path = tmp_path / "oracle_mut.py"
    path.write_text(src.replace(old, new, 1))
    spec = importlib.util.spec_from_file_location("oracle_mut", path)
    mod = importlib.util.module_from_spec(spec)
    spec.loader.exec_module(mod)
    codes = np.arange(256, dtype=np.uint8)
    ref = torch.from_numpy(codes).view(torch.float8_e4m3fn).to(torch.float64).numpy()
    got = mod.e4m3_decode(codes)
    nan = np.isnan(ref)
    assert not np.array_equal(got[~nan], ref[~nan])
