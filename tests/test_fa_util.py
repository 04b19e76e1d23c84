"""The tolerance helper of the stress tests, on the CPU: with every |v| = 1
the softmax-weighted sum of |v| is the row sum of the softmax weights, which
is 1 for every row that has a key (the weights come from the oracle's own
logsumexp), for dense and packed layouts, causal or not."""
import numpy as np
import pytest

import oracle
from exact_tiled_attention_32_b200 import synthetic as syn
from fa_util import softmax_weighted_abs_v


@pytest.mark.parametrize("packed", [False, True])
@pytest.mark.parametrize("causal", [False, True])
def test_weights_sum_to_one(packed, causal):
    if packed:
        w = syn.packed_from_lengths("h", [5, 0, 17, 1], 4, 64, causal, 11, Hkv=2).draw()
    else:
        w = syn.Workload("h", 2, 4, 2, 37, 64, causal, 12).draw()
    ones = syn.fp64_to_bf16_bits(np.where(np.arange(2) == 0, 1.0, -1.0)[np.arange(w.v.size) % 2]
                                 .reshape(w.v.shape))
    _, lse = oracle.attention(w.q, w.k, ones, w.B, w.Hq, w.Hkv, w.N, w.d, w.scale, causal, w.cu_seqlens)
    a = softmax_weighted_abs_v(w, w.scale, causal, lse, v_bits=ones)
    assert np.allclose(a, 1.0, atol=1e-12)


def test_weights_match_a_brute_force_row():
    w = syn.Workload("h", 1, 2, 1, 9, 64, True, 13).draw()
    o, lse = oracle.attention(w.q, w.k, w.v, w.B, w.Hq, w.Hkv, w.N, w.d, 3.0, True)
    a = softmax_weighted_abs_v(w, 3.0, True, lse)
    qf, kf, vf = (syn.bf16_bits_to_float(x).astype(np.float64) for x in (w.q, w.k, w.v))
    h, t = 1, 6
    s = 3.0 * kf[0, 0, :t + 1] @ qf[0, h, t]
    p = np.exp(s - s.max())
    p /= p.sum()
    assert np.allclose(a[h * w.N + t], p @ np.abs(vf[0, 0, :t + 1]), rtol=1e-12)
