"""The entry point that allocates no device memory (fa_fwd_noalloc).

It is meant for callers that cannot allocate device memory -- a process whose
HBM is reserved up front by another allocator, a latency-critical loop that
must not pay cudaMalloc's device-wide synchronisation, or a policy that forbids
new allocations after start-up.  Its scratch is a fixed array inside the
library, shared by all calls.  Through the C ABI, two calls in a row must give
the same O and logsumexp as fa_fwd, within the tolerances of the other tests,
and the oracle's result within the same tolerances; its device-side errors
are read back with fa_get_noalloc_status; and in a fresh process its calls
leave the device's free memory unchanged.
This file sorts last so that a run stopping at the first failure has run every
other test already; it also passes alone in a fresh process, where its first
call does the per-device set-up.
"""
import os
import subprocess
import sys
import textwrap

import numpy as np
import pytest

import oracle
from exact_tiled_attention_32_b200 import synthetic as syn
from fa_util import assert_parity, compare, gather, to_device

pytestmark = pytest.mark.gpu

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _workload(case):
    if case == "dense-causal-gqa":
        return syn.Workload(case, 2, 8, 2, 777, 128, True, 901).draw()
    if case == "packed-causal":
        return syn.packed_from_lengths(case, [300, 1, 129, 513], 4, 128, True, 902, Hkv=2).draw()
    return syn.Workload(case, 1, 4, 4, 1000, 64, False, 903).draw()


@pytest.mark.parametrize("case", ["dense-causal-gqa", "packed-causal", "dense-d64"])
def test_noalloc_matches_fa_fwd_twice(case):
    import torch
    from exact_tiled_attention_32_b200 import binding as fa

    w = _workload(case)
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
    orc_o, orc_lse = oracle.attention(w.q, w.k, w.v, w.B, w.Hq, w.Hkv, w.N, w.d, w.scale, w.causal, w.cu_seqlens)

    for call in range(2):
        o = torch.full_like(q, 5.0)
        lse = torch.full(lse_shape, 5.0, dtype=torch.float32, device="cuda")
        assert fa.fa_fwd_noalloc(q, k, v, o, lse, *args) == fa.FA_OK, f"call {call}"
        assert fa.fa_get_noalloc_status(stream) == fa.FA_OK, f"call {call}"
        got_o, got_lse = gather(w, o, lse)
        mx, mean, lmx = compare(got_o, got_lse, ref_o, ref_lse)
        assert mx <= 1e-2 and mean <= 1e-3 and lmx <= 1e-3, (call, mx, mean, lmx)
        assert_parity(got_o, got_lse, orc_o, orc_lse, f"noalloc {case} call {call} against the oracle")


def test_noalloc_reports_bad_seqlens_through_its_status_reader():
    """Offsets that the host cannot check (they live on the device) are
    rejected by the kernel; the code lands in the library's fixed array and
    fa_get_noalloc_status returns it (and clears it)."""
    import torch
    from exact_tiled_attention_32_b200 import binding as fa
    H, d = 2, 64
    stream = torch.cuda.current_stream()
    q = torch.zeros((20, H, d), dtype=torch.bfloat16, device="cuda")
    o = torch.full_like(q, 3.0)
    lse = torch.zeros((H, 20), dtype=torch.float32, device="cuda")
    for bad in ([0, 10, 5, 20], [1, 5, 20], [0, 5, 19]):
        cu = torch.tensor(bad, dtype=torch.int32, device="cuda")
        assert fa.fa_fwd_noalloc(q, q, q, o, lse, len(bad) - 1, H, H, 20, d, 0.1, 1, cu, stream) == fa.FA_OK
        assert fa.fa_get_noalloc_status(stream) == fa.FA_ERR_SEQLENS, bad
        assert fa.fa_get_noalloc_status(stream) == fa.FA_OK        # the reader cleared it
        assert torch.all(o == 3.0)
    # fa_fwd's own word saw none of it
    assert fa.fa_get_device_status(stream) == fa.FA_OK
    # and the next good call starts from a clean word
    good = torch.tensor([0, 5, 20], dtype=torch.int32, device="cuda")
    assert fa.fa_fwd_noalloc(q, q, q, o, lse, 2, H, H, 20, d, 0.1, 1, good, stream) == fa.FA_OK
    assert fa.fa_get_noalloc_status(stream) == fa.FA_OK


_FRESH = textwrap.dedent("""
    import json, sys
    import numpy as np
    import torch
    sys.path.insert(0, {root!r})
    from exact_tiled_attention_32_b200 import binding as fa
    from exact_tiled_attention_32_b200 import synthetic as syn
    torch.cuda.set_device(0)
    w = syn.Workload("fresh", 1, 4, 2, 1000, 128, True, 904).draw()
    dev = lambda a: torch.from_numpy(a.view(np.int16)).view(torch.bfloat16).cuda()
    q, k, v = dev(w.q), dev(w.k), dev(w.v)
    o = torch.empty_like(q)
    lse = torch.empty((w.B, w.Hq, w.N), dtype=torch.float32, device="cuda")
    s = torch.cuda.current_stream()
    torch.cuda.synchronize()
    # the library's first CUDA call loads its modules (eagerly, with the
    # fixed array); the status reader makes it without allocating anything
    assert fa.fa_get_noalloc_status(s) == 0
    torch.cuda.synchronize()
    free0 = torch.cuda.mem_get_info(0)[0]
    frees = []
    for _ in range(2):
        assert fa.fa_fwd_noalloc(q, k, v, o, lse, w.B, w.Hq, w.Hkv, w.N, w.d, w.scale, 1, None, s) == 0
        torch.cuda.synchronize()
        frees.append(torch.cuda.mem_get_info(0)[0])
    st = fa.fa_get_noalloc_status(s)
    print(json.dumps({{"free0": free0, "frees": frees, "status": st,
                      "finite": bool(torch.isfinite(o.float()).all())}}))
""")


def test_noalloc_leaves_free_device_memory_unchanged_in_a_fresh_process():
    """In a new process whose first forward call is fa_fwd_noalloc (modules
    loaded eagerly, so that loading them is not counted), the device's free
    memory is the same before and after each of two calls."""
    import json
    env = dict(os.environ, CUDA_MODULE_LOADING="EAGER")
    r = subprocess.run([sys.executable, "-c", _FRESH.format(root=ROOT)], env=env, capture_output=True, text=True,
                       timeout=300)
    assert r.returncode == 0, r.stderr[-2000:]
    out = json.loads(r.stdout.strip().splitlines()[-1])
    assert out["status"] == 0 and out["finite"], out
    assert out["frees"] == [out["free0"], out["free0"]], out


def test_noalloc_rejects_bad_arguments_like_fa_fwd():
    from exact_tiled_attention_32_b200 import binding as fa
    p = 1 << 20
    assert fa.fa_fwd_noalloc(p, p, p, p, p, 1, 4, 3, 128, 128, 0.1, 0) == fa.FA_ERR_GQA
    assert fa.fa_fwd_noalloc(p, p, p, p, p, 1, 4, 4, 128, 96, 0.1, 0) == fa.FA_ERR_HEADDIM
    assert fa.fa_fwd_noalloc(p + 2, p, p, p, p, 1, 4, 4, 128, 128, 0.1, 0) == fa.FA_ERR_ALIGN
    assert fa.fa_fwd_noalloc(0, 0, 0, 0, 0, 0, 4, 4, 128, 128, 0.1, 0) == fa.FA_OK
