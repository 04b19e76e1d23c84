"""The entry point that allocates no device memory (fa_fwd_noalloc).

It is meant for callers that cannot allocate device memory -- a process whose
HBM is reserved up front by another allocator, a latency-critical loop that
must not pay cudaMalloc's device-wide synchronisation, or a policy that forbids
new allocations after start-up.  Its scratch is a fixed array inside the
library, shared by all calls.  Through the C ABI, two calls in a row must give
the same O and logsumexp as fa_fwd, within the tolerances of the other tests.
This file sorts last so that a run stopping at the first failure has run every
other test already; it also passes alone in a fresh process, where its first
call does the per-device set-up.
"""
import numpy as np
import pytest

from exact_tiled_attention_32_b200 import synthetic as syn
from fa_util import compare, gather, to_device

pytestmark = pytest.mark.gpu


@pytest.mark.parametrize("case", ["dense-causal-gqa", "packed-causal", "dense-d64"])
def test_noalloc_matches_fa_fwd_twice(case):
    import torch
    from exact_tiled_attention_32_b200 import binding as fa

    if case == "dense-causal-gqa":
        w = syn.Workload(case, 2, 8, 2, 777, 128, True, 901).draw()
    elif case == "packed-causal":
        w = syn.packed_from_lengths(case, [300, 1, 129, 513], 4, 128, True, 902, Hkv=2).draw()
    else:
        w = syn.Workload(case, 1, 4, 4, 1000, 64, False, 903).draw()
    q, k, v = to_device(w.q), to_device(w.k), to_device(w.v)
    cu = None if w.cu_seqlens is None else torch.from_numpy(w.cu_seqlens).cuda()
    lse_shape = (w.Hq, w.N) if w.packed else (w.B, w.Hq, w.N)
    stream = torch.cuda.current_stream()
    args = (w.B, w.Hq, w.Hkv, w.N, w.d, w.scale, w.causal, cu, stream)

    o_ref = torch.empty_like(q)
    lse_ref = torch.empty(lse_shape, dtype=torch.float32, device="cuda")
    assert fa.fa_fwd(q, k, v, o_ref, lse_ref, *args) == fa.FA_OK
    torch.cuda.synchronize()
    assert fa.fa_get_device_status() == fa.FA_OK
    ref_o, ref_lse = gather(w, o_ref, lse_ref)

    for call in range(2):
        o = torch.full_like(q, 5.0)
        lse = torch.full(lse_shape, 5.0, dtype=torch.float32, device="cuda")
        assert fa.fa_fwd_noalloc(q, k, v, o, lse, *args) == fa.FA_OK, f"call {call}"
        torch.cuda.synchronize()
        got_o, got_lse = gather(w, o, lse)
        mx, mean, lmx = compare(got_o, got_lse, ref_o, ref_lse)
        assert mx <= 1e-2 and mean <= 1e-3 and lmx <= 1e-3, (call, mx, mean, lmx)


def test_noalloc_rejects_bad_arguments_like_fa_fwd():
    from exact_tiled_attention_32_b200 import binding as fa
    p = 1 << 20
    assert fa.fa_fwd_noalloc(p, p, p, p, p, 1, 4, 3, 128, 128, 0.1, 0) == fa.FA_ERR_GQA
    assert fa.fa_fwd_noalloc(p, p, p, p, p, 1, 4, 4, 128, 96, 0.1, 0) == fa.FA_ERR_HEADDIM
    assert fa.fa_fwd_noalloc(p + 2, p, p, p, p, 1, 4, 4, 128, 128, 0.1, 0) == fa.FA_ERR_ALIGN
    assert fa.fa_fwd_noalloc(0, 0, 0, 0, 0, 0, 4, 4, 128, 128, 0.1, 0) == fa.FA_OK
