"""fa_fwd_splitkv on B200: decode-shaped problems (a few query rows against a
long cache), the keys cut into splits merged through the logsumexp, grouped
query heads packed into one tile.  Compared with the fp64 oracle of the query
chunk (the last Nq positions, bottom-right causal mask), with the same
tolerances as the other parity tests."""
import numpy as np
import pytest

import oracle
from exact_tiled_attention_32_b200 import synthetic as syn
from fa_util import assert_parity, to_device

pytestmark = pytest.mark.gpu


def _run(w, num_splits=None):
    import torch
    from exact_tiled_attention_32_b200 import binding as fa
    o, lse = fa.attention_forward_splitkv(to_device(w.q), to_device(w.k), to_device(w.v), causal=w.causal,
                                          scale=w.scale, num_splits=num_splits)
    torch.cuda.synchronize()
    assert fa.fa_get_device_status() == 0
    return o.float().cpu().numpy().astype(np.float64).reshape(-1, w.d), lse.cpu().numpy().astype(np.float64).reshape(-1)


CASES = [
    # B, Hq, Hkv, Nq, Nk, d, causal, splits (None: the library's choice)
    (2, 8, 2, 1, 1000, 128, True, None),     # decode step, 4 heads per tile
    (2, 8, 2, 1, 1000, 128, True, 1),        # no split: the packed heads alone
    (2, 8, 2, 1, 1000, 128, True, 3),
    (1, 8, 8, 1, 3000, 128, True, 7),        # no grouping: one row per tile
    (1, 16, 4, 4, 777, 128, True, 5),        # 4 rows x 4 heads, bottom-right causal
    (1, 32, 2, 10, 1500, 128, True, 4),      # 16 heads x 10 rows = 160: rows wrap across tiles
    (2, 4, 4, 5, 300, 64, True, 2),
    (1, 8, 2, 3, 640, 64, False, 6),
    (1, 4, 1, 130, 600, 128, True, 3),       # Nq >= 128: heads not packed, two tiles
    (1, 4, 2, 2, 300, 128, True, 16),        # more splits than key blocks: empty splits
    (1, 2, 1, 1, 129, 128, True, 2),         # split of one key block plus one key
]


@pytest.mark.parametrize("B,Hq,Hkv,Nq,Nk,d,causal,splits", CASES)
def test_splitkv_all_rows(B, Hq, Hkv, Nq, Nk, d, causal, splits):
    w = syn.Workload("decode", B, Hq, Hkv, Nq, d, causal, 800 + Nq + Nk, Nk=Nk).draw()
    o, lse = _run(w, splits)
    oo, lo = oracle.attention_kv(w.q, w.k, w.v, B, Hq, Hkv, Nq, Nk, d, w.scale, causal)
    assert_parity(o, lse, oo, lo, f"splitkv {B},{Hq},{Hkv},{Nq},{Nk},{d},{causal},{splits}")


def test_splitkv_agrees_with_the_unsplit_chunk_forward():
    import torch
    from exact_tiled_attention_32_b200 import binding as fa
    w = syn.Workload("decode", 2, 16, 4, 3, 128, True, 870, Nk=5000).draw()
    q, k, v = to_device(w.q), to_device(w.k), to_device(w.v)
    o1, l1 = fa.attention_forward_kvcache(q, k, v, causal=True)
    o2, l2 = fa.attention_forward_splitkv(q, k, v, causal=True, num_splits=9)
    torch.cuda.synchronize()
    assert (o1.float() - o2.float()).abs().max().item() <= 1e-2
    assert (l1 - l2).abs().max().item() <= 1e-3


def test_splitkv_chosen_split_count():
    from exact_tiled_attention_32_b200 import binding as fa
    # a decode batch with 64 (batch, kv head) units on a long cache is split
    s = fa.fa_splitkv_num_splits(8, 32, 8, 1, 32768, 128)
    assert 2 <= s <= 256
    # a problem that already fills the GPU is not
    assert fa.fa_splitkv_num_splits(4, 32, 32, 2048, 4096, 128) == 1


def test_dec_sampled_rows():
    """The decode workload the bench times: B=8, Hq=32, Hkv=8, one row against
    32768 keys; every row is checked (there are 256)."""
    w = syn.config("dec").draw()
    o, lse = _run(w)
    oo, lo = oracle.attention_kv(w.q, w.k, w.v, w.B, w.Hq, w.Hkv, w.N, w.Nk, w.d, w.scale, w.causal)
    assert_parity(o, lse, oo, lo, "dec")
