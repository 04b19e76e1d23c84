#!/usr/bin/env python
"""Benchmark of the exact attention forward on B200.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--config c3] [--impl ours|reference]
                    [--pass fwd|bwd]

A step is one fa_fwd call over the whole workload (default: causal B=1, H=32,
N=16384, d=128, the configuration the throughput target is quoted on).  The
inputs are seeded synthetic bf16 N(0,1) tensors already resident in HBM; they
are 384 MiB, larger than the 126 MiB L2, so no flush runs between steps.  With
N > 1 GPUs (one process each, launched by torch.distributed.run) every rank
solves its own independent problem of the same shape: there is no exchange step
in the attention forward, so no data-path collective exists and the scaling is
weak; the timing is the maximum over ranks.

Rank 0 prints one JSON line.  ``--impl reference`` times the fp64 CPU oracle
on the host cores instead (rank 0 only), each step a bounded sample of the same
workload's query rows.

``--pass bwd`` times the backward pass instead (fa_bwd: dQ, dK, dV from the
forward's O and logsumexp and a seeded upstream gradient), counted as 2.5x the
forward's FLOPs (five matrix products per block instead of two); its CPU
baseline is the fp64 gradient oracle on one (batch, kv head) unit.
"""
from __future__ import annotations

import argparse
import hashlib
import json
import math
import os
import re
import subprocess
import sys
import threading
import time

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

METRIC = "attention fwd TFLOP/s (bf16) and % of B200 dense BF16 tensor peak"
METRIC_BWD = "attention bwd TFLOP/s (bf16; 2.5x the forward's FLOPs) and % of B200 dense BF16 tensor peak"
BWD_FLOP_FACTOR = 2.5
UNIT = "TFLOP/s"
FALLBACK_PEAK_TFLOPS = 1590.0


def parse_args():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=200)
    ap.add_argument("--warmup", type=int, default=10)
    ap.add_argument("--config", default="c3")
    ap.add_argument("--impl", choices=["ours", "reference"], default="ours")
    ap.add_argument("--e2e-steps", type=int, default=8)
    ap.add_argument("--cpu-seconds", type=float, default=12.0,
                    help="CPU time budget of the oracle baseline sample")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--pass", dest="pass_", choices=["fwd", "bwd"], default="fwd")
    return ap.parse_args()


def workload_desc(w):
    if w.chunk:
        return (f"{w.name}: {'causal' if w.causal else 'non-causal'} query chunk of {w.N} rows (the last "
                f"positions) against {w.Nk} keys, B={w.B} Hq={w.Hq} Hkv={w.Hkv} d={w.d}, bf16 N(0,1), "
                "scale=1/sqrt(d)")
    if w.fp8:
        shape = (f"packed {w.B} sequences (lengths {min(w.seqlens)}..{max(w.seqlens)}), H={w.Hq}" if w.packed
                 else f"B={w.B} Hq={w.Hq} Hkv={w.Hkv} N={w.N}")
        return (f"{w.name}: {'causal' if w.causal else 'non-causal'} {shape} d={w.d}, "
                "Q/K/V E4M3 codes of N(0,1)*32 (per-tensor scale 1/32), scale=1/sqrt(d)")
    if w.packed:
        shape = f"packed {w.B} sequences (lengths {min(w.seqlens)}..{max(w.seqlens)}), H={w.Hq}"
    else:
        shape = f"B={w.B} Hq={w.Hq} Hkv={w.Hkv} N={w.N}"
    return f"{w.name}: {'causal' if w.causal else 'non-causal'} {shape} d={w.d}, bf16 N(0,1), scale=1/sqrt(d)"


def config_dict(w, extra=None):
    c = {
        "workload": workload_desc(w),
        "B": w.B, "Hq": w.Hq, "Hkv": w.Hkv, "N": w.N, "d": w.d, "causal": w.causal,
        "seed": w.seed, "flops_per_step": w.flops(),
        "l2": "inputs larger than L2 (no flush between steps)",
    }
    if w.packed:
        c["seqlens"] = list(w.seqlens)
    if w.chunk:
        c["Nk"] = w.Nk
    if extra:
        c.update(extra)
    return c


# ----------------------------------------------------------------- peaks
def load_peak():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    try:
        with open(path) as f:
            pk = json.load(f)
        return float(pk["bf16_tflops"]), float(pk.get("bf16_tflops_sustained", 0)) or None, "measured"
    except Exception:
        return FALLBACK_PEAK_TFLOPS, None, "fallback"


def load_hbm_peak():
    try:
        with open(os.path.join(ROOT, "MEASURED_PEAKS.json")) as f:
            return float(json.load(f)["hbm_gbs"]), "measured"
    except Exception:
        return 6650.0, "fallback"


def source_sha(kernel="fwd"):
    """sha256[:16] of the source files of the forward (fa_fwd.cu) or backward
    (fa_bwd.cu) kernel, with the shared PTX wrappers."""
    h = hashlib.sha256()
    main = "fa_fwd.cu" if kernel == "fwd" else "fa_bwd.cu"
    for rel in (f"exact_tiled_attention_32_b200/csrc/{main}", "exact_tiled_attention_32_b200/csrc/sm100_ptx.cuh"):
        with open(os.path.join(ROOT, rel), "rb") as f:
            h.update(f.read())
    return h.hexdigest()[:16]


PROFILE_TABLE = os.path.join("profiles", "fa_configs.md")


def profiled_ncu(key, kernel="fwd"):
    """The ncu figures of one launch of the workload's dominant kernel, from
    the committed per-configuration table (row `key`), if they were taken on
    the current kernel source; else None.  Table rows:
    | config | kernel | source sha | ncu ms | SM GHz | tensor % | MUFU % | DRAM read B | DRAM write B | issue % |
    """
    path = os.path.join(ROOT, PROFILE_TABLE)
    if not os.path.exists(path):
        return None
    sha = source_sha(kernel)
    num = r"\s*([0-9.eE+-]+)\s*\|"
    pat = re.compile(r"\|\s*([\w-]+)\s*\|\s*(fwd|bwd)\s*\|\s*([0-9a-f]{16})\s*\|" + num * 7)
    for line in open(path):
        m = pat.match(line)
        if m and m.group(1) == key and m.group(2) == kernel and m.group(3) == sha:
            ms, ghz, tensor, xu, rd, wr, issue = (float(m.group(i)) for i in range(4, 11))
            return {"tensor_pipe_pct": tensor, "mufu_pct": xu, "issue_active_pct": issue,
                    "dram_bytes": rd + wr, "ncu_ms": ms, "ncu_sm_ghz": ghz,
                    "hbm_gbs_ncu": (rd + wr) / (ms * 1e-3) / 1e9,
                    "source": f"ncu, one launch, {PROFILE_TABLE} row {key}/{kernel}, source sha {sha}"}
    return None


def add_ncu_fields(roofline, key, kernel, ms_per_step):
    """traffic (DRAM bytes per launch of the dominant kernel) and the ncu
    utilisation figures of the profiled launch, with HBM GB/s = that traffic
    over this run's time per step; null when the table has no row for the
    current source."""
    prof = profiled_ncu(key, kernel)
    if prof is None:
        roofline.update({"traffic": None, "traffic_source": f"none: no {PROFILE_TABLE} row for this source",
                         "ncu": None})
        return roofline
    roofline["traffic"] = prof["dram_bytes"]
    roofline["traffic_source"] = prof["source"]
    roofline["ncu"] = {"tensor_pipe_pct": prof["tensor_pipe_pct"], "mufu_pct": prof["mufu_pct"],
                       "issue_active_pct": prof["issue_active_pct"], "hbm_gbs_ncu": prof["hbm_gbs_ncu"],
                       "hbm_gbs": prof["dram_bytes"] / (ms_per_step * 1e-3) / 1e9,
                       "ncu_ms": prof["ncu_ms"], "ncu_sm_ghz": prof["ncu_sm_ghz"], "source": prof["source"]}
    return roofline


# ---------------------------------------------------------------- clocks
class ClockSampler:
    """nvidia-smi samples of SM clock and throttle reasons, tagged with host time."""

    FIELDS = ("clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.hw_slowdown,"
              "clocks_event_reasons.hw_thermal_slowdown,clocks_event_reasons.sw_thermal_slowdown,"
              "clocks_event_reasons.sw_power_cap")

    def __init__(self, gpu_id):
        self.samples = []
        self.proc = None
        self.gpu_id = gpu_id
        self.thread = None

    def start(self):
        cmd = ["nvidia-smi", f"--query-gpu={self.FIELDS}", "--format=csv,noheader,nounits", "-lms", "100"]
        if self.gpu_id:
            cmd += ["-i", self.gpu_id]
        try:
            self.proc = subprocess.Popen(cmd, stdout=subprocess.PIPE, stderr=subprocess.DEVNULL, text=True)
        except Exception:
            self.proc = None
            return
        self.thread = threading.Thread(target=self._read, daemon=True)
        self.thread.start()

    def _read(self):
        for line in self.proc.stdout:
            parts = [p.strip() for p in line.split(",")]
            if len(parts) == 7:
                self.samples.append((time.time(), parts))

    def stop(self):
        if self.proc:
            self.proc.terminate()
            try:
                self.proc.wait(timeout=5)
            except Exception:
                self.proc.kill()

    def summary(self, t0, t1):
        def num(x):
            try:
                return float(x)
            except ValueError:
                return None
        inside = [p for (t, p) in self.samples if t0 <= t <= t1]
        if not inside:        # short timed region: nearest samples after it started
            inside = [p for (t, p) in self.samples if t >= t0][:3]
        if not inside:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": [], "samples": 0}
        sm = sorted(v for v in (num(p[0]) for p in inside) if v is not None)
        names = ("hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap")
        reasons = sorted({names[i] for p in inside for i in range(4) if p[3 + i].lower() == "active"})
        return {"sm_mhz": sm[len(sm) // 2] if sm else None, "sm_max_mhz": num(inside[0][1]),
                "reasons": reasons, "samples": len(inside),
                "power_w_max": max((num(p[2]) or 0) for p in inside)}


# ------------------------------------------------------------ CPU oracle
def oracle_sample_rows(w, nrows, rng):
    """Random query rows of the workload (all heads, all positions)."""
    import numpy as np
    rows = rng.integers(0, w.total_rows(), nrows)
    return np.unique(rows)


def row_flops(w, rows):
    """4*d*(keys attended) per sampled row: the per-row share of the metric's
    4*N^2*d (halved when causal)."""
    import numpy as np
    if w.packed:
        tok = rows % w.N
        cu = w.cu_seqlens
        s = np.searchsorted(cu, tok, side="right") - 1
        t = tok - cu[s]
        L = cu[s + 1] - cu[s]
    elif w.chunk:
        t = rows % w.N
        keys = (w.Nk - w.N + t + 1) if w.causal else np.full_like(t, w.Nk)
        return float(np.sum(4.0 * w.d * keys))
    else:
        t = rows % w.N
        L = np.full_like(t, w.N)
    keys = (t + 1) if w.causal else L
    return float(np.sum(4.0 * w.d * keys))


def oracle_rows(w, rows):
    """The oracle on the given query rows of workload ``w``."""
    import oracle
    if w.fp8:
        from exact_tiled_attention_32_b200 import synthetic as syn
        s = syn.FP8_SCALE
        return oracle.attention_fp8(w.q, w.k, w.v, s, s, s, w.B, w.Hq, w.Hkv, w.N, w.d, w.scale, w.causal,
                                    rows=rows, cu_seqlens=w.cu_seqlens)
    if w.chunk:
        return oracle.attention_kv(w.q, w.k, w.v, w.B, w.Hq, w.Hkv, w.N, w.Nk, w.d, w.scale, w.causal,
                                   rows=rows)
    return oracle.attention(w.q, w.k, w.v, w.B, w.Hq, w.Hkv, w.N, w.d, w.scale, w.causal,
                            w.cu_seqlens, rows=rows)


def time_oracle(w, seconds, seed=0, keep=4):
    """Times the oracle on random row samples until ``seconds`` have passed.
    Returns the baseline record and the oracle's results on the last ``keep``
    samples (rows, O, lse), which the caller compares with the GPU output."""
    import numpy as np
    import oracle
    rng = np.random.default_rng(seed)
    flops = 0.0
    rows_done = 0
    kept = []
    t0 = time.perf_counter()
    while True:
        rows = oracle_sample_rows(w, 64, rng)
        o_ref, l_ref = oracle_rows(w, rows)
        kept = (kept + [(rows, o_ref, l_ref)])[-keep:]
        flops += row_flops(w, rows)
        rows_done += len(rows)
        if time.perf_counter() - t0 >= seconds:
            break
    dt = time.perf_counter() - t0
    rec = {"value": flops / dt / 1e12, "unit": UNIT, "cores": oracle.num_threads(), "kind": "oracle",
           "sample": f"{rows_done} random query rows of the workload (fp64, materialised score rows), "
                     f"{dt:.1f} s on the host cores"}
    return rec, kept


def gpu_rows(w, o, lse, rows):
    """Rows ``rows`` (in the oracle's row order) of the GPU's O and logsumexp,
    as fp64 numpy arrays."""
    import numpy as np
    import torch
    idx = torch.from_numpy(np.asarray(rows, dtype=np.int64)).to(o.device)
    if w.packed:        # O [N, Hq, d], oracle row h * N + token; lse [Hq, N] is already in that order
        og = o.permute(1, 0, 2).reshape(-1, w.d).index_select(0, idx)
    else:
        og = o.reshape(-1, w.d).index_select(0, idx)
    lg = lse.reshape(-1).index_select(0, idx)
    return og.float().cpu().numpy().astype(np.float64), lg.cpu().numpy().astype(np.float64)


def parity_of_sample(w, o, lse, kept):
    """The timed output against the oracle on the rows the CPU baseline
    computed: O max-abs / mean-abs and lse max-abs, checked against the
    forward's tolerances (O 1e-2 / 1e-3, lse 1e-3) for bf16 paths.  The FP8
    path's tolerance is a per-element bound derived in its tests, so here its
    errors are recorded only."""
    import numpy as np
    rows = np.concatenate([r for r, _, _ in kept])
    o_ref = np.concatenate([x for _, x, _ in kept])
    l_ref = np.concatenate([x for _, _, x in kept])
    og, lg = gpu_rows(w, o, lse, rows)
    e = np.abs(og - o_ref)
    fin = np.isfinite(l_ref)
    el = float(np.abs(lg[fin] - l_ref[fin]).max()) if fin.any() else 0.0
    rec = {"rows": int(len(rows)), "o_max_abs": float(e.max()), "o_mean_abs": float(e.mean()),
           "lse_max_abs": el, "nan": bool(np.isnan(og).any())}
    if w.fp8:
        rec["checked"] = False
        rec["tolerance"] = "recorded only (FP8: per-element E4M3 bound in the tests)"
    else:
        rec["checked"] = True
        rec["tolerance"] = "O max-abs <= 1e-2, O mean-abs <= 1e-3, lse max-abs <= 1e-3"
        rec["ok"] = (not rec["nan"]) and rec["o_max_abs"] <= 1e-2 and rec["o_mean_abs"] <= 1e-3 and el <= 1e-3 \
            and bool(np.array_equal(np.isfinite(lg), fin))
    return rec


def bwd_unit_flops(w):
    """Backward FLOPs of one (batch, kv head) unit: 2.5x the forward's."""
    return BWD_FLOP_FACTOR * w.flops() / (w.B * w.Hkv)


def time_oracle_bwd(w, do, seconds):
    """The gradient oracle on whole (batch, kv head) units until ``seconds``
    have passed (at least one unit)."""
    import oracle
    units = 0
    t0 = time.perf_counter()
    while True:
        oracle.attention_bwd(w.q, w.k, w.v, do, w.B, w.Hq, w.Hkv, w.N, w.d, w.scale, w.causal,
                             units=[units % (w.B * w.Hkv)])
        units += 1
        if time.perf_counter() - t0 >= seconds:
            break
    dt = time.perf_counter() - t0
    return {"value": units * bwd_unit_flops(w) / dt / 1e12, "unit": UNIT, "cores": oracle.num_threads(),
            "kind": "oracle", "sample": f"{units} whole (batch, kv head) units of the workload's gradients "
                                        f"(fp64, materialised score rows), {dt:.1f} s on the host cores"}


def bwd_dout(w):
    """The seeded upstream gradient of the backward bench (bf16 N(0,1))."""
    from exact_tiled_attention_32_b200 import synthetic as syn
    return syn.Stream(w.seed + 77).normal_bf16(w.q_shape())


def run_reference(args, rank):
    """--impl reference: the oracle timed on the host cores (rank 0 only)."""
    if rank != 0:
        return
    if getattr(args, "pass_", "fwd") == "bwd":
        from exact_tiled_attention_32_b200 import synthetic as syn
        import oracle
        w = syn.config(args.config).draw()
        do = bwd_dout(w)
        t0 = time.perf_counter()
        for k in range(args.steps):
            oracle.attention_bwd(w.q, w.k, w.v, do, w.B, w.Hq, w.Hkv, w.N, w.d, w.scale, w.causal,
                                 units=[k % (w.B * w.Hkv)])
        dt = time.perf_counter() - t0
        value = args.steps * bwd_unit_flops(w) / dt / 1e12
        line = {
            "impl": "reference", "metric": METRIC_BWD, "value": value, "unit": UNIT, "n_gpus": args.gpus,
            "steps": args.steps, "warmup": args.warmup, "ms_per_step": dt * 1e3 / max(args.steps, 1),
            "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f64", "data": "synthetic",
            "config": config_dict(w, {"pass": "bwd", "step": "one whole (batch, kv head) unit per step"}),
            "cpu_baseline": {"value": value, "unit": UNIT, "cores": oracle.num_threads(), "kind": "oracle",
                             "sample": f"{args.steps} (batch, kv head) units"},
            "e2e": {"value": value, "unit": UNIT, "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
        }
        print(json.dumps(line), flush=True)
        return
    import numpy as np
    import oracle
    from exact_tiled_attention_32_b200 import synthetic as syn
    w = syn.config(args.config).draw()
    rng = np.random.default_rng(1)
    nrows = 32
    for _ in range(args.warmup):
        oracle_rows(w, oracle_sample_rows(w, nrows, rng))
    flops = 0.0
    rows_done = 0
    t0 = time.perf_counter()
    for _ in range(args.steps):
        rows = oracle_sample_rows(w, nrows, rng)
        oracle_rows(w, rows)
        flops += row_flops(w, rows)
        rows_done += len(rows)
    dt = time.perf_counter() - t0
    value = flops / dt / 1e12
    line = {
        "impl": "reference", "metric": METRIC, "value": value, "unit": UNIT, "n_gpus": args.gpus,
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": dt * 1e3 / max(args.steps, 1),
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f64",
        "data": "synthetic",
        "config": config_dict(w, {"step": f"{nrows} random query rows per step"}),
        "cpu_baseline": {"value": value, "unit": UNIT, "cores": oracle.num_threads(), "kind": "oracle",
                         "sample": f"{rows_done} random query rows over {args.steps} steps"},
        "e2e": {"value": value, "unit": UNIT, "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
    }
    print(json.dumps(line), flush=True)


# ------------------------------------------------------------- ranks
def max_over_ranks(x: float, world: int, device=None) -> float:
    """Maximum of a per-rank number over all ranks (the job's time is the
    slowest rank's); identity on one rank."""
    if world <= 1:
        return x
    import torch
    import torch.distributed as dist
    t = torch.tensor([x], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def whole_job_tflops(flops_per_step: float, world: int, steps: int, ms: float) -> float:
    """Throughput of the whole job: every rank ran ``steps`` steps of
    ``flops_per_step`` in ``ms`` milliseconds (the maximum over ranks)."""
    return flops_per_step * world * steps / (ms / 1e3) / 1e12


def step_percentiles(per_step_ms):
    """Median, p10 and p90 of the per-step device times (milliseconds), taken
    from one CUDA event recorded after each step inside the timed region."""
    import numpy as np
    a = np.asarray(per_step_ms, dtype=np.float64)
    if a.size == 0:
        return None
    return {"median": float(np.median(a)), "p10": float(np.percentile(a, 10)),
            "p90": float(np.percentile(a, 90)), "n": int(a.size)}


def pipelined_e2e(steps, host_in, run, host_out, dev, world):
    """Times ``steps`` end-to-end steps through host buffers: each step copies
    ``host_in`` (pinned) to the device, calls ``run(device inputs)`` (the public
    API; returns the device outputs) and copies the outputs into ``host_out``
    (pinned).  The copies run on their own streams so that step i+1's uploads
    and step i-1's downloads overlap step i's kernels, as a serving loop would
    run them; every step still moves all of its bytes.  Two device input
    buffers alternate.  CUDA events bracket the whole loop on the compute
    stream (the upload stream waits for the start event).  Returns the time in
    ms, the max over ranks."""
    import torch
    import torch.distributed as dist

    comp = torch.cuda.current_stream(dev)
    s_in = torch.cuda.Stream(dev)
    s_out = torch.cuda.Stream(dev)
    bufs = [[torch.empty(h.shape, dtype=h.dtype, device=dev) for h in host_in] for _ in range(2)]

    def go(n):
        done = [None, None]        # compute-done events of the steps that last used each input buffer
        last = None
        for i in range(n):
            b = i % 2
            if done[b] is not None:
                s_in.wait_event(done[b])
            with torch.cuda.stream(s_in):
                for d, h in zip(bufs[b], host_in):
                    d.copy_(h, non_blocking=True)
            ev_in = torch.cuda.Event()
            ev_in.record(s_in)
            comp.wait_event(ev_in)
            outs = run(bufs[b])
            ev_c = torch.cuda.Event()
            ev_c.record(comp)
            done[b] = ev_c
            s_out.wait_event(ev_c)
            with torch.cuda.stream(s_out):
                for h, d in zip(host_out, outs):
                    h.copy_(d, non_blocking=True)
                    d.record_stream(s_out)
            last = torch.cuda.Event()
            last.record(s_out)
        comp.wait_event(last)

    go(2)                          # warm-up: allocations, first copies
    torch.cuda.synchronize(dev)
    if world > 1:
        dist.barrier()
    e0 = torch.cuda.Event(enable_timing=True)
    e1 = torch.cuda.Event(enable_timing=True)
    e0.record(comp)
    s_in.wait_event(e0)
    go(steps)
    e1.record(comp)
    e1.synchronize()
    return max_over_ranks(e0.elapsed_time(e1), world, dev)


def timed_steps(step, steps, stream):
    """Runs ``steps`` steps between CUDA events on ``stream``: one event
    before the first step and one after every step.  Returns the total device
    time (first to last event) and the per-step times, in milliseconds."""
    import torch
    evs = [torch.cuda.Event(enable_timing=True) for _ in range(steps + 1)]
    evs[0].record(stream)
    for i in range(steps):
        step()
        evs[i + 1].record(stream)
    evs[-1].synchronize()
    per = [evs[i].elapsed_time(evs[i + 1]) for i in range(steps)]
    return evs[0].elapsed_time(evs[-1]), per


# ------------------------------------------------------------- GPU path
def main():
    args = parse_args()
    rank = int(os.environ.get("RANK", "0"))
    world = int(os.environ.get("WORLD_SIZE", "1"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    if args.impl == "reference":
        run_reference(args, rank)
        return

    import numpy as np
    import torch
    import torch.distributed as dist
    from exact_tiled_attention_32_b200 import binding as fa
    from exact_tiled_attention_32_b200 import synthetic as syn

    torch.cuda.set_device(local)
    dev = torch.device("cuda", local)
    if world > 1:
        from datetime import timedelta
        dist.init_process_group("nccl", timeout=timedelta(seconds=300), device_id=dev)

    w = syn.config(args.config)
    w.seed += rank              # independent problem per rank
    w.draw()
    if args.pass_ == "bwd":
        if w.packed or w.chunk:
            raise SystemExit("--pass bwd runs on dense workloads (c1, c2nc, c2c, c3, c4)")
        return run_bwd(args, w, rank, world, dev)
    if w.fp8:
        q, k, v = (torch.from_numpy(a).to(dev) for a in (w.q, w.k, w.v))      # E4M3 codes
    else:
        q = torch.from_numpy(w.q.view(np.int16)).view(torch.bfloat16).to(dev)
        k = torch.from_numpy(w.k.view(np.int16)).view(torch.bfloat16).to(dev)
        v = torch.from_numpy(w.v.view(np.int16)).view(torch.bfloat16).to(dev)
    cu = None if w.cu_seqlens is None else torch.from_numpy(w.cu_seqlens).to(dev)
    o = torch.empty(q.shape, dtype=torch.bfloat16, device=dev)
    lse_shape = (w.Hq, w.N) if w.packed else (w.B, w.Hq, w.N)
    lse = torch.empty(lse_shape, dtype=torch.float32, device=dev)
    stream = torch.cuda.current_stream(dev)
    splits, ws, ws_bytes = 1, None, 0
    if w.decode:
        splits = fa.fa_splitkv_num_splits(w.B, w.Hq, w.Hkv, w.N, w.Nk, w.d)
        if splits < 0:
            raise fa.FAError(splits, "fa_splitkv_num_splits")
        ws_bytes = fa.fa_splitkv_workspace_bytes(w.B, w.Hq, w.N, w.d, splits)
        ws = torch.empty(max(ws_bytes, 16), dtype=torch.uint8, device=dev)

    fp8_scale = syn.FP8_SCALE

    def step():
        if w.fp8 and w.packed:
            rc = fa.fa_fwd_fp8_varlen(q, k, v, o, lse, w.B, w.Hq, w.Hkv, w.N, w.d, w.scale, w.causal, fp8_scale,
                                      fp8_scale, fp8_scale, cu, stream)
        elif w.fp8:
            rc = fa.fa_fwd_fp8(q, k, v, o, lse, w.B, w.Hq, w.Hkv, w.N, w.d, w.scale, w.causal, fp8_scale, fp8_scale,
                               fp8_scale, stream)
        elif w.decode:
            rc = fa.fa_fwd_splitkv(q, k, v, o, lse, w.B, w.Hq, w.Hkv, w.N, w.Nk, w.d, w.scale, w.causal,
                                   splits, ws, ws_bytes, stream)
        elif w.chunk:
            rc = fa.fa_fwd_kvcache(q, k, v, o, lse, w.B, w.Hq, w.Hkv, w.N, w.Nk, w.d, w.scale, w.causal,
                                   stream)
        else:
            rc = fa.fa_fwd(q, k, v, o, lse, w.B, w.Hq, w.Hkv, w.N, w.d, w.scale, w.causal, cu, stream)
        if rc != 0:
            raise fa.FAError(rc)

    gpu_id = None
    try:
        gpu_id = "GPU-" + str(torch.cuda.get_device_properties(dev).uuid)
    except Exception:
        pass
    sampler = ClockSampler(gpu_id)
    sampler.start()
    time.sleep(0.3)

    for _ in range(max(args.warmup, 0)):
        step()
    torch.cuda.synchronize(dev)
    if world > 1:
        dist.barrier()
    torch.cuda.synchronize(dev)
    t_host0 = time.time()
    ms, per_step = timed_steps(step, args.steps, stream)
    torch.cuda.synchronize(dev)
    t_host1 = time.time()
    if world > 1:
        dist.barrier()
    ms = max_over_ranks(ms, world, dev)
    sampler.stop()
    status = fa.fa_get_device_status(stream)
    if status != 0:
        raise fa.FAError(status, "device status after the timed region")

    ms_per_step = ms / max(args.steps, 1)
    value = whole_job_tflops(w.flops(), world, args.steps, ms)
    achieved = w.flops() / (ms_per_step / 1e3) / 1e12          # one launch = one step
    peak, peak_sustained, peak_kind = load_peak()

    # ---- end to end through the public call, host buffers, copies timed
    e2e = None
    if args.e2e_steps > 0:
        if w.fp8:
            qh, kh, vh = (torch.from_numpy(a).pin_memory() for a in (w.q, w.k, w.v))
        else:
            qh = torch.from_numpy(w.q.view(np.int16)).view(torch.bfloat16).pin_memory()
            kh = torch.from_numpy(w.k.view(np.int16)).view(torch.bfloat16).pin_memory()
            vh = torch.from_numpy(w.v.view(np.int16)).view(torch.bfloat16).pin_memory()
        oh = torch.empty(q.shape, dtype=torch.bfloat16).pin_memory()
        lh = torch.empty(lse_shape, dtype=torch.float32).pin_memory()

        def e2e_run(inputs):
            qd, kd, vd = inputs
            if w.fp8:
                od, ld = fa.attention_forward_fp8(qd, kd, vd, fp8_scale, fp8_scale, fp8_scale, causal=w.causal,
                                                  scale=w.scale, cu_seqlens=cu)
            elif w.decode:
                od, ld = fa.attention_forward_splitkv(qd, kd, vd, causal=w.causal, scale=w.scale,
                                                      num_splits=splits, workspace=ws)
            elif w.chunk:
                od, ld = fa.attention_forward_kvcache(qd, kd, vd, causal=w.causal, scale=w.scale)
            else:
                od, ld = fa.attention_forward(qd, kd, vd, causal=w.causal, scale=w.scale, cu_seqlens=cu)
            return od, ld

        ems = pipelined_e2e(args.e2e_steps, (qh, kh, vh), e2e_run, (oh, lh), dev, world)
        e2e = {"value": whole_job_tflops(w.flops(), world, args.e2e_steps, ems), "unit": UNIT,
               "h2d_bytes_per_step": int(qh.nbytes + kh.nbytes + vh.nbytes),
               "d2h_bytes_per_step": int(oh.nbytes + lh.nbytes),
               "ms_per_step": ems / args.e2e_steps, "steps": args.e2e_steps,
               "copies": "pinned host buffers; uploads and downloads on their own streams, overlapping "
                         "the neighbouring steps' kernels"}

    cpu = None
    parity = None
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        # the oracle baseline; its sampled rows also check the output the
        # timed steps wrote (inputs unchanged, so every step wrote the same)
        cpu, kept = time_oracle(w, args.cpu_seconds)
        parity = parity_of_sample(w, o, lse, kept)

    if world > 1:
        dist.barrier()
        dist.destroy_process_group()
    if rank != 0:
        return
    clocks = sampler.summary(t_host0, t_host1)
    launches_per_step = 1
    if w.decode:
        # HBM-bound: the forward streams the K/V cache once; the roofline is
        # bytes over the whole step (forward + the split merge), against the
        # measured copy bandwidth
        launches_per_step = 2 if splits > 1 else 1
        hbm_peak, hbm_kind = load_hbm_peak()
        gbs = w.hbm_bytes() / (ms_per_step / 1e3) / 1e9
        roofline = {"bound": "hbm", "achieved": gbs, "peak": hbm_peak, "unit": "GB/s",
                    "frac": gbs / hbm_peak,
                    "peak_source": f"MEASURED_PEAKS.json hbm_gbs, of {hbm_kind}",
                    "algorithmic_bytes": w.hbm_bytes(),
                    "timed": f"whole step: split-key forward + merge of {splits} splits"}
    elif w.fp8:
        # the FP8 peak: the measured bf16 peak times the nominal FP8 / BF16 ratio (4.5 / 2.25)
        roofline = {"bound": "tensor", "achieved": achieved, "peak": 2 * peak, "unit": UNIT,
                    "frac": achieved / (2 * peak),
                    "peak_source": f"2 x MEASURED_PEAKS.json bf16_tflops (burst; nominal fp8/bf16 ratio), of {peak_kind}",
                    "frac_of_sustained": (achieved / (2 * peak_sustained)) if peak_sustained else None}
    else:
        roofline = {"bound": "tensor", "achieved": achieved, "peak": peak, "unit": UNIT,
                    "frac": achieved / peak,
                    "peak_source": f"MEASURED_PEAKS.json bf16_tflops (burst), of {peak_kind}",
                    "frac_of_sustained": (achieved / peak_sustained) if peak_sustained else None}
    add_ncu_fields(roofline, args.config, "fwd", ms_per_step)
    line = {
        "metric": METRIC, "value": value, "unit": UNIT, "n_gpus": world, "steps": args.steps,
        "warmup": args.warmup, "ms_per_step": ms_per_step, "higher_is_better": True,
        "scaling": "weak", "vs_baseline": None, "dtype": "e4m3" if w.fp8 else "bf16", "data": "synthetic",
        "config": config_dict(w, {"parallelism": f"replicas x{world} (independent problems, no collective)",
                                  **({"num_splits": splits} if w.decode else {})}),
        "roofline": roofline,
        "cpu_baseline": cpu,
        "e2e": e2e,
        "gpu_launches": args.steps * launches_per_step,
        "clocks": clocks,
        "step_ms": step_percentiles(per_step),
    }
    if parity is not None:
        line["parity_sample"] = parity
    print(json.dumps(line), flush=True)
    if parity is not None and parity.get("checked") and not parity["ok"]:
        raise SystemExit(f"the timed output differs from the oracle on sampled rows: {parity}")


def run_bwd(args, w, rank, world, dev):
    """The backward pass (fa_bwd) timed like the forward: CUDA events over K
    steps, each step one fa_bwd call (three kernel launches) on resident
    inputs."""
    import numpy as np
    import torch
    import torch.distributed as dist
    from exact_tiled_attention_32_b200 import binding as fa

    def dev_bits(a):
        return torch.from_numpy(np.ascontiguousarray(a).view(np.int16)).view(torch.bfloat16).to(dev)

    do_bits = bwd_dout(w)
    q, k, v, do = dev_bits(w.q), dev_bits(w.k), dev_bits(w.v), dev_bits(do_bits)
    o, lse = fa.attention_forward(q, k, v, causal=w.causal, scale=w.scale)
    ws_bytes = fa.fa_bwd_workspace_bytes(w.B, w.Hq, w.N, w.d, False)
    ws = torch.empty(ws_bytes, dtype=torch.uint8, device=dev)
    dq, dk, dv = torch.empty_like(q), torch.empty_like(k), torch.empty_like(v)
    stream = torch.cuda.current_stream(dev)
    flops = BWD_FLOP_FACTOR * w.flops()

    def step():
        rc = fa.fa_bwd(q, k, v, o, lse, do, dq, dk, dv, w.B, w.Hq, w.Hkv, w.N, w.d, w.scale, w.causal, None, ws,
                       ws_bytes, stream)
        if rc != 0:
            raise fa.FAError(rc, "fa_bwd")

    gpu_id = None
    try:
        gpu_id = "GPU-" + str(torch.cuda.get_device_properties(dev).uuid)
    except Exception:
        pass
    sampler = ClockSampler(gpu_id)
    sampler.start()
    time.sleep(0.3)
    for _ in range(max(args.warmup, 0)):
        step()
    torch.cuda.synchronize(dev)
    if world > 1:
        dist.barrier()
    torch.cuda.synchronize(dev)
    t_host0 = time.time()
    ms, per_step = timed_steps(step, args.steps, stream)
    torch.cuda.synchronize(dev)
    t_host1 = time.time()
    ms = max_over_ranks(ms, world, dev)
    sampler.stop()
    status = fa.fa_get_device_status(stream)
    if status != 0:
        raise fa.FAError(status, "device status after the timed region")
    ms_per_step = ms / max(args.steps, 1)
    value = whole_job_tflops(flops, world, args.steps, ms)
    achieved = flops / (ms_per_step / 1e3) / 1e12
    peak, peak_sustained, peak_kind = load_peak()

    e2e = None
    if args.e2e_steps > 0:
        host = [torch.from_numpy(np.ascontiguousarray(a).view(np.int16)).view(torch.bfloat16).pin_memory()
                for a in (w.q, w.k, w.v, do_bits)]
        oh = o.cpu().pin_memory()
        lh = lse.cpu().pin_memory()
        outs = [torch.empty(t.shape, dtype=torch.bfloat16).pin_memory() for t in (dq, dk, dv)]

        def e2e_run(inputs):
            qd, kd, vd, dod, od, ld = inputs
            return fa.attention_backward(qd, kd, vd, od, ld, dod, causal=w.causal, scale=w.scale, workspace=ws)

        ems = pipelined_e2e(args.e2e_steps, tuple(host) + (oh, lh), e2e_run, outs, dev, world)
        e2e = {"value": whole_job_tflops(flops, world, args.e2e_steps, ems), "unit": UNIT,
               "h2d_bytes_per_step": int(sum(t.nbytes for t in host) + oh.nbytes + lh.nbytes),
               "d2h_bytes_per_step": int(sum(t.nbytes for t in outs)),
               "ms_per_step": ems / args.e2e_steps, "steps": args.e2e_steps,
               "copies": "pinned host buffers; uploads and downloads on their own streams, overlapping "
                         "the neighbouring steps' kernels"}

    cpu = None
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        cpu = time_oracle_bwd(w, do_bits, args.cpu_seconds)
    if world > 1:
        dist.barrier()
        dist.destroy_process_group()
    if rank != 0:
        return
    line = {
        "metric": METRIC_BWD, "value": value, "unit": UNIT, "n_gpus": world, "steps": args.steps,
        "warmup": args.warmup, "ms_per_step": ms_per_step, "higher_is_better": True,
        "scaling": "weak", "vs_baseline": None, "dtype": "bf16", "data": "synthetic",
        "config": config_dict(w, {"pass": "bwd", "flops_per_step": flops,
                                  "parallelism": f"replicas x{world} (independent problems, no collective)"}),
        "roofline": add_ncu_fields(
            {"bound": "tensor", "achieved": achieved, "peak": peak, "unit": UNIT, "frac": achieved / peak,
             "peak_source": f"MEASURED_PEAKS.json bf16_tflops (burst), of {peak_kind}",
             "frac_of_sustained": (achieved / peak_sustained) if peak_sustained else None,
             "timed": "whole step: D / accumulator prep, the backward kernel, dQ conversion"},
            args.config, "bwd", ms_per_step),
        "cpu_baseline": cpu,
        "e2e": e2e,
        "gpu_launches": 3 * args.steps,
        "clocks": sampler.summary(t_host0, t_host1),
        "step_ms": step_percentiles(per_step),
    }
    print(json.dumps(line), flush=True)


if __name__ == "__main__":
    main()
