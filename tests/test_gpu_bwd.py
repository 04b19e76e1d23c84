"""fa_bwd on B200: dQ, dK, dV compared with the fp64 oracle of the
gradients on the same bf16 inputs.  The GPU forward supplies O and the
logsumexp, as in training; the oracle differentiates the exact definition.

Tolerance: the forward's bound carried over to the gradients, plus one bf16
rounding of the result (2^-7 |ref|: the output is bf16), since gradients are
O(1) quantities formed from bf16-rounded P and dS, like O."""
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


def _check(got, ref, what):
    assert not np.isnan(got).any(), f"{what}: NaN"
    err = np.abs(got - ref)
    bound = MAX_ABS + 2.0 ** -7 * np.abs(ref)
    assert (err - bound).max() <= 0, f"{what}: max error {err.max():.3e} (excess {(err - bound).max():.3e})"
    assert err.mean() <= MEAN_ABS, f"{what}: mean error {err.mean():.3e}"


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
    tag = f"{B},{Hq},{Hkv},{N},{d},{causal}"
    _check(dq, rq, f"dq {tag}")
    _check(dk, rk, f"dk {tag}")
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
        return fa.fa_bwd(*ptrs, a["B"], a["Hq"], a["Hkv"], a["N"], a["d"], a["scale"], a["causal"], ws, wb)

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
    _check(dq[0, h], rq[0, 0], "c3 dq head 5")
    _check(dk[0, h], rk[0], "c3 dk head 5")
    _check(dv[0, h], rv[0], "c3 dv head 5")
