"""The C ABI on a machine without a GPU: the library loads, exports every
function that include/*.h declares, and rejects bad arguments before it
touches a device (no compute call is made here)."""
import ctypes
import glob
import os
import re

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _declared():
    names = set()
    for h in glob.glob(os.path.join(ROOT, "include", "*.h")):
        src = re.sub(r"/\*.*?\*/", "", open(h).read(), flags=re.S)
        names.update(re.findall(r"\b(fa_[a-z0-9_]+)\s*\(", src))
    return names


def test_library_exports_every_declared_symbol():
    from exact_tiled_attention_32_b200 import binding as fa
    lib = ctypes.CDLL(fa.LIB_PATH)
    declared = _declared()
    assert {"fa_fwd", "fa_get_device_status", "fa_status_string"} <= declared
    for name in declared:
        assert hasattr(lib, name), f"{name} declared in include/ but not exported"


def test_status_strings():
    from exact_tiled_attention_32_b200 import binding as fa
    for code in range(0, -10, -1):
        s = fa.fa_status_string(code)
        assert s and s != "unknown status"
    assert fa.fa_status_string(-100) == "unknown status"


def test_argument_errors_found_on_the_host():
    from exact_tiled_attention_32_b200 import binding as fa
    p = 1 << 20          # an aligned address that is never dereferenced
    ok = dict(B=1, Hq=4, Hkv=2, N=128, d=128, scale=0.1, causal=1)

    def call(**kw):
        a = dict(ok)
        ptrs = kw.pop("ptrs", (p, p, p, p, p))
        a.update(kw)
        return fa.fa_fwd(*ptrs, a["B"], a["Hq"], a["Hkv"], a["N"], a["d"], a["scale"],
                         a["causal"], kw.get("cu"), None)

    assert call(d=96) == fa.FA_ERR_HEADDIM
    assert call(d=256) == fa.FA_ERR_HEADDIM
    assert call(Hq=4, Hkv=3) == fa.FA_ERR_GQA
    assert call(Hkv=0) == fa.FA_ERR_GQA
    assert call(B=-1) == fa.FA_ERR_SHAPE
    assert call(N=-5) == fa.FA_ERR_SHAPE
    assert call(Hq=0) == fa.FA_ERR_SHAPE
    assert call(ptrs=(p, 0, p, p, p)) == fa.FA_ERR_NULL
    assert call(ptrs=(p, p, p, p, 0)) == fa.FA_ERR_NULL
    assert call(ptrs=(p + 8, p, p, p, p)) == fa.FA_ERR_ALIGN
    assert call(ptrs=(p, p, p, p + 2, p)) == fa.FA_ERR_ALIGN
    assert call(ptrs=(p, p, p, p, p + 1)) == fa.FA_ERR_ALIGN
    assert call(cu=p + 2) == fa.FA_ERR_ALIGN
    assert call(B=1025, cu=p) == fa.FA_ERR_SHAPE
    # empty problems: nothing to do, pointers may be NULL
    assert call(B=0, ptrs=(0, 0, 0, 0, 0)) == fa.FA_OK
    assert call(N=0, ptrs=(0, 0, 0, 0, 0)) == fa.FA_OK


def test_chunk_partial_merge_noalloc_argument_errors_found_on_the_host():
    """fa_fwd_kvcache, fa_fwd_partial, fa_merge_partials and fa_fwd_noalloc
    reject bad arguments before touching a device."""
    from exact_tiled_attention_32_b200 import binding as fa
    p = 1 << 20
    P5 = (p, p, p, p, p)
    for fn in (fa.fa_fwd_kvcache, fa.fa_fwd_partial):
        def call(B=1, Hq=4, Hkv=2, Nq=64, Nk=256, d=128, causal=1, ptrs=P5):
            return fn(*ptrs, B, Hq, Hkv, Nq, Nk, d, 0.1, causal)
        assert call(d=80) == fa.FA_ERR_HEADDIM
        assert call(Hkv=3) == fa.FA_ERR_GQA
        assert call(Nq=-1) == fa.FA_ERR_SHAPE
        assert call(Nk=0) == fa.FA_ERR_SHAPE
        assert call(Nq=300, Nk=256, causal=1) == fa.FA_ERR_SHAPE      # causal needs Nk >= Nq
        assert call(ptrs=(p, p, 0, p, p)) == fa.FA_ERR_NULL
        assert call(ptrs=(p, p, p, p + 4, p)) == fa.FA_ERR_ALIGN
        assert call(ptrs=(p, p, p, p, p + 2)) == fa.FA_ERR_ALIGN
        assert call(Nq=0, ptrs=(0, 0, 0, 0, 0)) == fa.FA_OK
        assert call(B=0, ptrs=(0, 0, 0, 0, 0)) == fa.FA_OK

    def merge(nparts=2, rows=10, d=128, ptrs=(p, p, p, p)):
        return fa.fa_merge_partials(ptrs[0], ptrs[1], nparts, rows, d, ptrs[2], ptrs[3])
    assert merge(nparts=0) == fa.FA_ERR_SHAPE
    assert merge(nparts=4097) == fa.FA_ERR_SHAPE
    assert merge(rows=-1) == fa.FA_ERR_SHAPE
    assert merge(d=32) == fa.FA_ERR_HEADDIM
    assert merge(ptrs=(p, 0, p, p)) == fa.FA_ERR_NULL
    assert merge(ptrs=(p + 4, p, p, p)) == fa.FA_ERR_ALIGN
    assert merge(rows=0, ptrs=(0, 0, 0, 0)) == fa.FA_OK
    # one block of the merge kernel per 8 rows: the grid's x limit bounds rows
    assert merge(nparts=1, rows=8 * (2 ** 31 - 1) + 1) == fa.FA_ERR_SHAPE

    def noalloc(B=1, Hq=4, Hkv=2, N=128, d=128, cu=None, ptrs=P5):
        return fa.fa_fwd_noalloc(*ptrs, B, Hq, Hkv, N, d, 0.1, 1, cu)
    assert noalloc(d=96) == fa.FA_ERR_HEADDIM
    assert noalloc(Hkv=3) == fa.FA_ERR_GQA
    assert noalloc(B=-1) == fa.FA_ERR_SHAPE
    assert noalloc(ptrs=(0, p, p, p, p)) == fa.FA_ERR_NULL
    assert noalloc(ptrs=(p, p, p, p + 2, p)) == fa.FA_ERR_ALIGN
    assert noalloc(B=1025, cu=p) == fa.FA_ERR_SHAPE
    assert noalloc(cu=p + 2) == fa.FA_ERR_ALIGN
    assert noalloc(N=0, ptrs=(0, 0, 0, 0, 0)) == fa.FA_OK


def test_splitkv_argument_errors_found_on_the_host():
    from exact_tiled_attention_32_b200 import binding as fa
    p = 1 << 20
    ok = dict(B=2, Hq=8, Hkv=2, Nq=1, Nk=4096, d=128, scale=0.1, causal=1, S=4)

    def call(ptrs=(p, p, p, p, p), ws=p, wbytes=1 << 30, **kw):
        a = dict(ok)
        a.update(kw)
        return fa.fa_fwd_splitkv(*ptrs, a["B"], a["Hq"], a["Hkv"], a["Nq"], a["Nk"], a["d"], a["scale"],
                                 a["causal"], a["S"], ws, wbytes, None)

    assert call(d=96) == fa.FA_ERR_HEADDIM
    assert call(Hkv=3) == fa.FA_ERR_GQA
    assert call(S=0) == fa.FA_ERR_SHAPE
    assert call(S=257) == fa.FA_ERR_SHAPE
    assert call(Nk=0) == fa.FA_ERR_SHAPE
    assert call(Nq=8, Nk=4) == fa.FA_ERR_SHAPE          # causal chunk longer than the keys
    assert call(ws=0) == fa.FA_ERR_NULL
    assert call(ws=p + 4) == fa.FA_ERR_ALIGN
    need = fa.fa_splitkv_workspace_bytes(2, 8, 1, 128, 4)
    assert call(wbytes=need - 1) == fa.FA_ERR_SHAPE
    assert call(ptrs=(p, p, 0, p, p)) == fa.FA_ERR_NULL
    assert call(B=0, ptrs=(0, 0, 0, 0, 0), ws=0, wbytes=0) == fa.FA_OK
    # one split needs no workspace
    assert fa.fa_splitkv_workspace_bytes(2, 8, 1, 128, 1) == 0


def test_splitkv_workspace_bytes():
    from exact_tiled_attention_32_b200 import binding as fa
    # num_splits x rows x (d + 1) fp32 values
    assert fa.fa_splitkv_workspace_bytes(2, 8, 3, 128, 4) == 4 * 2 * 8 * 3 * 129 * 4
    assert fa.fa_splitkv_workspace_bytes(1, 32, 1, 64, 16) == 16 * 32 * 65 * 4
    assert fa.fa_splitkv_workspace_bytes(1, 1, 1, 96, 2) == 0      # bad head dim
    assert fa.fa_splitkv_workspace_bytes(1, 1, 1, 64, 0) == 0      # bad split count
    assert fa.fa_splitkv_workspace_bytes(1, 1, 1, 64, 257) == 0


def test_bwd_argument_errors_and_workspace_bytes():
    from exact_tiled_attention_32_b200 import binding as fa
    p = 1 << 20
    # B * Hq * Npad * (d + 2) * 4 with Npad = N rounded up to 128
    assert fa.fa_bwd_workspace_bytes(2, 4, 300, 128) == 2 * 4 * 384 * 130 * 4
    assert fa.fa_bwd_workspace_bytes(1, 1, 128, 64) == 128 * 66 * 4
    assert fa.fa_bwd_workspace_bytes(1, 1, 128, 96) == 0
    # packed: Hq * Npad * (d + 2) * 4 + (3 B + 4) * 4 with Npad = N + 128 B rounded up to 128
    assert fa.fa_bwd_workspace_bytes(3, 4, 300, 128, True) == 4 * 768 * 130 * 4 + (3 * 3 + 4) * 4
    assert fa.fa_bwd_workspace_bytes(1025, 4, 300, 128, True) == 0

    def call(ptrs=(p,) * 9, ws=p, wb=1 << 30, B=1, Hq=4, Hkv=2, N=100, d=128, cu=None):
        return fa.fa_bwd(*ptrs, B, Hq, Hkv, N, d, 0.1, 1, cu, ws, wb)

    assert call(d=96) == fa.FA_ERR_HEADDIM
    assert call(Hkv=3) == fa.FA_ERR_GQA
    assert call(N=-1) == fa.FA_ERR_SHAPE
    assert call(ws=0) == fa.FA_ERR_NULL
    assert call(ptrs=(p,) * 8 + (0,)) == fa.FA_ERR_NULL
    assert call(ws=p + 4) == fa.FA_ERR_ALIGN
    assert call(ptrs=(p + 2,) + (p,) * 8) == fa.FA_ERR_ALIGN
    assert call(wb=fa.fa_bwd_workspace_bytes(1, 4, 100, 128) - 16) == fa.FA_ERR_SHAPE
    assert call(B=0, ptrs=(0,) * 9, ws=0, wb=0) == fa.FA_OK
    assert call(B=1025, cu=p) == fa.FA_ERR_SHAPE
    assert call(cu=p + 2) == fa.FA_ERR_ALIGN
    assert call(B=3, cu=p, wb=fa.fa_bwd_workspace_bytes(3, 4, 100, 128, True) - 4) == fa.FA_ERR_SHAPE


def test_fp8_argument_errors_found_on_the_host():
    from exact_tiled_attention_32_b200 import binding as fa
    p = 1 << 20
    call = lambda d=128, qs=1.0, Hkv=2, ptrs=(p,) * 5, B=1: fa.fa_fwd_fp8(*ptrs, B, 4, Hkv, 256, d, 0.1, 1, qs, 1.0, 1.0)
    assert call(d=96) == fa.FA_ERR_HEADDIM      # d = 64 and 128 are supported
    assert call(qs=0.0) == fa.FA_ERR_SHAPE
    assert call(qs=float("nan")) == fa.FA_ERR_SHAPE
    assert call(Hkv=3) == fa.FA_ERR_GQA
    assert call(ptrs=(p, p, 0, p, p)) == fa.FA_ERR_NULL
    assert call(ptrs=(p + 1, p, p, p, p)) == fa.FA_ERR_ALIGN
    assert call(B=0, ptrs=(0,) * 5) == fa.FA_OK


def test_fp8_varlen_argument_errors_found_on_the_host():
    from exact_tiled_attention_32_b200 import binding as fa
    p = 1 << 20

    def call(B=2, d=128, cu=p, ptrs=(p, p, p, p, p)):
        return fa.fa_fwd_fp8_varlen(*ptrs, B, 2, 2, 128, d, 0.1, 1, 1, 1, 1, cu)
    assert call(d=96) == fa.FA_ERR_HEADDIM
    assert call(cu=0) == fa.FA_ERR_NULL
    assert call(cu=p + 2) == fa.FA_ERR_ALIGN
    assert call(B=1025) == fa.FA_ERR_SHAPE
    assert call(ptrs=(p, p, p, p, p + 2)) == fa.FA_ERR_ALIGN
    assert call(B=0, cu=0, ptrs=(0,) * 5) == fa.FA_OK


def test_kvcache_varlen_argument_errors_found_on_the_host():
    from exact_tiled_attention_32_b200 import binding as fa
    p = 1 << 20

    def call(B=2, Nq=64, Nk=256, d=128, cq=p, ck=p, ptrs=(p, p, p, p, p)):
        return fa.fa_fwd_kvcache_varlen(*ptrs, B, 4, 2, Nq, Nk, d, 0.1, 1, cq, ck)
    assert call(d=80) == fa.FA_ERR_HEADDIM
    assert call(cq=0) == fa.FA_ERR_NULL
    assert call(ck=0) == fa.FA_ERR_NULL
    assert call(ck=p + 2) == fa.FA_ERR_ALIGN
    assert call(B=1025) == fa.FA_ERR_SHAPE
    assert call(Nk=0) == fa.FA_ERR_SHAPE
    assert call(Nq=0, ptrs=(0,) * 5, cq=0, ck=0) == fa.FA_OK


def test_no_device_means_launch_error():
    import torch
    if torch.cuda.is_available():
        pytest.skip("a GPU is present")
    from exact_tiled_attention_32_b200 import binding as fa
    p = 1 << 20
    assert fa.fa_fwd(p, p, p, p, p, 1, 1, 1, 128, 64, 0.1, 0) == fa.FA_ERR_LAUNCH
    assert fa.fa_get_device_status() == fa.FA_ERR_LAUNCH
    assert fa.fa_get_noalloc_status() == fa.FA_ERR_LAUNCH
    assert fa.fa_splitkv_num_splits(1, 32, 8, 1, 32768, 128) == fa.FA_ERR_LAUNCH


def test_binding_refuses_to_run_without_the_library(tmp_path, monkeypatch):
    """The product path has no fallback: a missing libfa.so is an ImportError."""
    import importlib.util
    import shutil
    pkg = tmp_path / "pkgcopy"
    pkg.mkdir()
    shutil.copy(os.path.join(ROOT, "exact_tiled_attention_32_b200", "binding.py"), pkg / "binding.py")
    spec = importlib.util.spec_from_file_location("binding_copy", pkg / "binding.py")
    mod = importlib.util.module_from_spec(spec)
    with pytest.raises(ImportError):
        spec.loader.exec_module(mod)
