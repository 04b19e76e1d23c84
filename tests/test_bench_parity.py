"""bench.py's host logic on the CPU: the rows it checks against the oracle
are picked out of the output tensors in the oracle's row order (dense and
packed layouts), a correct output passes and a perturbed one fails, and the
ncu table lookup reads only rows taken on the current kernel source."""
import os
import sys

import numpy as np

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
sys.path.insert(0, ROOT)

import bench  # noqa: E402
import oracle  # noqa: E402
from exact_tiled_attention_32_b200 import synthetic as syn  # noqa: E402


def _as_tensors(w, o_rows, l_rows):
    """Oracle-ordered rows -> the kernel's output layouts (CPU tensors)."""
    import torch
    if w.packed:
        o = torch.from_numpy(o_rows.reshape(w.Hq, w.N, w.d).transpose(1, 0, 2).copy())
        lse = torch.from_numpy(l_rows.reshape(w.Hq, w.N).copy())
    else:
        o = torch.from_numpy(o_rows.reshape(w.B, w.Hq, w.N, w.d).copy())
        lse = torch.from_numpy(l_rows.reshape(w.B, w.Hq, w.N).copy())
    return o.to(torch.bfloat16), lse.float()


def _check(w):
    o_all, l_all = oracle.attention(w.q, w.k, w.v, w.B, w.Hq, w.Hkv, w.N, w.d, w.scale, w.causal, w.cu_seqlens)
    o, lse = _as_tensors(w, o_all, l_all)
    rng = np.random.default_rng(3)
    kept = []
    for _ in range(3):
        rows = bench.oracle_sample_rows(w, 16, rng)
        kept.append((rows, *bench.oracle_rows(w, rows)))
    rec = bench.parity_of_sample(w, o, lse, kept)
    assert rec["checked"] and rec["ok"], rec
    bad = o.clone()
    r0 = int(kept[0][0][0])
    if w.packed:
        bad[r0 % w.N, r0 // w.N, 0] += 0.5
    else:
        bad.view(-1, w.d)[r0, 0] += 0.5
    rec = bench.parity_of_sample(w, bad, lse, kept)
    assert not rec["ok"] and rec["o_max_abs"] > 0.4


def test_dense_rows_are_checked():
    _check(syn.Workload("d", 2, 4, 2, 200, 64, True, 5).draw())


def test_packed_rows_are_checked():
    _check(syn.packed_from_lengths("p", [130, 7, 0, 64], 4, 64, True, 6, Hkv=2).draw())


def test_ncu_table_lookup_matches_current_source(tmp_path, monkeypatch):
    sha = bench.source_sha("fwd")
    (tmp_path / "profiles").mkdir()
    (tmp_path / "profiles" / "fa_configs.md").write_text(
        "| config | kernel | sha | ms | GHz | tensor | mufu | rd | wr | issue |\n"
        "|---|---|---|---|---|---|---|---|---|---|\n"
        f"| c3 | fwd | 0123456789abcdef | 1.0 | 1.9 | 50 | 50 | 1e9 | 1e8 | 30 |\n"
        f"| c3 | fwd | {sha} | 2.0 | 1.8 | 61.5 | 63.0 | 2e9 | 1e8 | 35.5 |\n")
    monkeypatch.setattr(bench, "ROOT", str(tmp_path))
    monkeypatch.setattr(bench, "source_sha", lambda kernel="fwd": sha)
    prof = bench.profiled_ncu("c3", "fwd")
    assert prof["tensor_pipe_pct"] == 61.5 and prof["mufu_pct"] == 63.0
    assert prof["dram_bytes"] == 2.1e9
    assert abs(prof["hbm_gbs_ncu"] - 2.1e9 / 2e-3 / 1e9) < 1e-9
    assert bench.profiled_ncu("c4", "fwd") is None
    r = bench.add_ncu_fields({}, "c2c", "fwd", 1.0)
    assert r["traffic"] is None and r["ncu"] is None
