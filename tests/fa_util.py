"""Helpers shared by the GPU tests: move seeded inputs to the device, run the
C ABI, gather outputs in the oracle's row order, sample rows, and compare
with the tolerances of the attention forward (O max-abs 1e-2, O mean-abs 1e-3,
lse max-abs 1e-3 against the fp64 oracle on the same bf16 inputs)."""
from __future__ import annotations

import numpy as np

O_MAX_ABS = 1e-2
O_MEAN_ABS = 1e-3
LSE_MAX_ABS = 1e-3


def to_device(bits):
    import torch
    return torch.from_numpy(np.ascontiguousarray(bits).view(np.int16)).view(torch.bfloat16).cuda()


def run_gpu(w, q=None, k=None, v=None):
    """Runs the CUDA path on workload ``w``; returns (o [rows, d] fp64 in the
    oracle's row order, lse [rows] fp64, device status)."""
    import torch
    from exact_tiled_attention_32_b200 import binding as fa

    q = to_device(w.q) if q is None else q
    k = to_device(w.k) if k is None else k
    v = to_device(w.v) if v is None else v
    cu = None if w.cu_seqlens is None else torch.from_numpy(w.cu_seqlens).cuda()
    o, lse = fa.attention_forward(q, k, v, causal=w.causal, scale=w.scale, cu_seqlens=cu)
    torch.cuda.synchronize()
    st = fa.fa_get_device_status()
    return gather(w, o, lse) + (st,)


def gather(w, o, lse):
    of = o.float().cpu().numpy().astype(np.float64)
    lf = lse.cpu().numpy().astype(np.float64).reshape(-1)
    if w.packed:                  # [Ntot, Hq, d] -> rows h*Ntot + token
        of = of.transpose(1, 0, 2).reshape(-1, w.d)
    else:
        of = of.reshape(-1, w.d)
    return of, lf


def sample_rows(w, early=8, tile_stride=1, n_random=16, seed=0):
    """Row ids per (sequence, head): the first ``early`` rows, the first and
    last row of every ``tile_stride``-th 128-row tile, the last row, and
    ``n_random`` random rows."""
    rng = np.random.default_rng(seed)
    rows = []
    for h in range(w.Hq):
        for s, L in enumerate(w.lengths):
            if L == 0:
                continue
            if w.packed:
                base = h * w.N + int(w.cu_seqlens[s])
            else:
                base = (s * w.Hq + h) * w.N
            ts = set(range(min(early, L)))
            for m in range(0, (L + 127) // 128, tile_stride):
                ts.update((128 * m, min(128 * m + 127, L - 1)))
            ts.add(L - 1)
            ts.update(rng.integers(0, L, n_random).tolist())
            rows.extend(base + t for t in sorted(ts))
    return np.array(sorted(rows), dtype=np.int64)


def compare(o_gpu, lse_gpu, o_ref, lse_ref):
    """Returns (o max-abs, o mean-abs, lse max-abs); -inf lse must match."""
    e = np.abs(o_gpu - o_ref)
    finite = np.isfinite(lse_ref)
    assert np.array_equal(np.isfinite(lse_gpu), finite), "lse -inf pattern differs"
    el = np.abs(lse_gpu[finite] - lse_ref[finite]) if finite.any() else np.zeros(1)
    return float(e.max()), float(e.mean()), float(el.max())


def softmax_weighted_abs_v(w, scale, causal, lse_ref, q_bits=None, k_bits=None, v_bits=None):
    """Per row and column, sum_j p_j |v_j| with p_j = exp(s_j - lse) the row's
    softmax weights: the scores s_j are formed here in fp64 from the bf16
    inputs and normalised by the oracle's own logsumexp ``lse_ref`` (rows in
    the oracle's order).  Dense or packed workloads, keys j <= position when
    causal."""
    from exact_tiled_attention_32_b200 import synthetic as syn
    qf = syn.bf16_bits_to_float(w.q if q_bits is None else q_bits).astype(np.float64)
    kf = syn.bf16_bits_to_float(w.k if k_bits is None else k_bits).astype(np.float64)
    vf = np.abs(syn.bf16_bits_to_float(w.v if v_bits is None else v_bits).astype(np.float64))
    g = w.Hq // w.Hkv
    out = np.zeros((w.total_rows(), w.d))
    units = []
    if w.packed:
        for s_, L in enumerate(w.lengths):
            a = int(w.cu_seqlens[s_])
            for h in range(w.Hq):
                units.append((qf[a:a + L, h], kf[a:a + L, h // g], vf[a:a + L, h // g], h * w.N + a))
    else:
        for b in range(w.B):
            for h in range(w.Hq):
                units.append((qf[b, h], kf[b, h // g], vf[b, h // g], (b * w.Hq + h) * w.N))
    for Q, K, V, base in units:
        L = Q.shape[0]
        if L == 0:
            continue
        S = scale * (Q @ K.T)
        if causal:
            S[np.triu_indices(L, 1)] = -np.inf
        lse = lse_ref[base:base + L]
        P = np.exp(S - np.where(np.isfinite(lse), lse, 0.0)[:, None])
        out[base:base + L] = P @ V
    return out


def assert_bf16_bound(o_gpu, lse_gpu, o_ref, lse_ref, pv_abs, what=""):
    """Stress inputs outside the stated workloads (|O| up to ~4.5), where the
    bound is derived from the bf16 roundings the kernel makes instead:
    1e-2, plus the round-to-nearest of O to bf16 (relative error <= 2^-8, so
    2^-8 |O|), plus the round-to-nearest of each softmax weight to bf16
    before the P V product (relative <= 2^-8 per weight, so at most
    2^-8 sum_j p_j |v_j| on each output column; ``pv_abs`` is that sum, from
    softmax_weighted_abs_v).  The exponentials (ex2.approx, relative ~2^-22)
    and the fp32 accumulations are orders of magnitude below these terms.
    lse keeps its 1e-3 bound."""
    assert not np.isnan(o_gpu).any(), f"{what}: NaN in O"
    bound = 1e-2 + 2.0 ** -8 * np.abs(o_ref) + 2.0 ** -8 * pv_abs
    excess = np.abs(o_gpu - o_ref) - bound
    assert excess.max() <= 0, f"{what}: O error exceeds the bf16 bound by {excess.max():.3e}"
    _, _, lmx = compare(o_gpu, lse_gpu, o_ref, lse_ref)
    assert lmx <= LSE_MAX_ABS, f"{what}: lse max-abs {lmx:.3e} > {LSE_MAX_ABS}"


def assert_parity(o_gpu, lse_gpu, o_ref, lse_ref, what=""):
    assert not np.isnan(o_gpu).any(), f"{what}: NaN in O"
    mx, mean, lmx = compare(o_gpu, lse_gpu, o_ref, lse_ref)
    assert mx <= O_MAX_ABS, f"{what}: O max-abs {mx:.3e} > {O_MAX_ABS}"
    assert mean <= O_MEAN_ABS, f"{what}: O mean-abs {mean:.3e} > {O_MEAN_ABS}"
    assert lmx <= LSE_MAX_ABS, f"{what}: lse max-abs {lmx:.3e} > {LSE_MAX_ABS}"
    return mx, mean, lmx
