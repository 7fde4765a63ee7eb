#!/usr/bin/env python
"""Throughput of the fused indexer score + exact top-k (ftk_select).

Workload: the FP8 prefill chunk of the FlashTopK README "Quick start" --
q [4096, 32, 128] and kv [131072, 128] FP8-e4m3 from N(0,1), kv_scales in
(0.5, 1], weights N(0,1)/sqrt(32), causal windows ke[t] = 126976 + t + 1,
topk 2048 -- seeded and synthetic (sparse_attention_indexer_ftk_b200.workloads).

One step = one ftk_select call over the whole 4096-query batch (sample pass,
thresholds, pruning decision, scan, refine, recovery).  Inputs are resident
in HBM; the L2 is flushed (a 256 MB write) between timed steps, outside the
timed events.  Beside the metric, on one GPU: per-stage times, the scan's
roofline (with the DRAM traffic of the committed ncu summary while the
kernel source is unchanged), an end-to-end figure through host buffers, a
64-query (decode-shaped) call, the row top-k (ftk_topk_rows) on the 64-row
bf16 / fp32 batches and a 1024-row bf16 batch with a warm-L2 time and a
trivial read-reduce over the same bytes, and the CPU oracle's rate.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl ours|reference]
                    [--no-rows] [--only-rows [--rows-workload NAME]] [--no-decode]
                    [--no-cpu-baseline]

Multi-GPU (launched with torch.distributed.run): every rank runs its own
independent batch of the same shape (weak scaling; no data-path collective);
the step time is the max over ranks.  Beside it, one batch split into
contiguous row blocks across the ranks (strong scaling), its blocks gathered
on rank 0 after the timed region and checked bit for bit against the
single-GPU result.

Prints one JSON line (rank 0).
"""
from __future__ import annotations

import argparse
import json
import os
import statistics
import subprocess
import sys
import tempfile
import time

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

METRIC = "fused score+top-k queries/s & dense-eq TFLOP/s (4096q×128K FP8, k=2048)"
WORKLOAD = "fp8_prefill"
PROFILE_TRAFFIC = os.path.join(ROOT, "profiles", "scan_kernel_fp8_prefill.md")


def parse_args():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=200)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--impl", choices=["ours", "reference"], default="ours")
    ap.add_argument("--e2e-steps", type=int, default=20)
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--no-rows", action="store_true", help="skip the row top-k section")
    ap.add_argument("--only-rows", action="store_true", help="run only the row top-k section")
    ap.add_argument("--rows-workload", default="",
                    help="with --only-rows: only this row workload (rows_bf16, rows_f32, rows_bf16_1024)")
    ap.add_argument("--no-decode", action="store_true", help="skip the 64-query (decode-shaped) section")
    ap.add_argument("--no-extras", action="store_true",
                    help="skip the decode-shaped, packed-workload and FP8 GEMM reference sections")
    ap.add_argument("--cpu-seconds", type=float, default=12.0)
    ap.add_argument("--oracle-configs", action="store_true",
                    help="time only the CPU oracle on every workload configuration (no GPU)")
    ap.add_argument("--rows", type=int, default=0,
                    help="use only the first ROWS queries of the batch (profiling captures)")
    return ap.parse_args()


def dist_env():
    ws = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    return ws, rank, local


def measured_peaks():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(path):
        with open(path) as f:
            d = json.load(f)
        return d, "measured"
    return {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0}, "fallback"


def profiled_traffic():
    """DRAM bytes per scan-kernel launch from the committed ncu summary."""
    try:
        text = open(PROFILE_TRAFFIC).read()
    except OSError:
        return None
    import re
    m = re.search(r"traffic_bytes_per_launch:\s*([0-9.eE+]+)", text)
    s = re.search(r"kernel_source_hash:\s*([0-9a-f]+)", text)
    if not m:
        return None
    if s and s.group(1) != scan_kernel_hash():
        return None  # the kernel changed since the counters were taken
    return float(m.group(1))


def strip_comments(src: str) -> str:
    """C++ source without comments and with whitespace collapsed."""
    import re
    src = re.sub(r"/\*.*?\*/", " ", src, flags=re.S)
    src = re.sub(r"//[^\n]*", " ", src)
    return " ".join(src.split())


def scan_kernel_hash(read=None) -> str:
    """Hash of the scan kernel's sources, comments and layout ignored (a
    comment edit does not invalidate the profiled counters)."""
    import hashlib
    h = hashlib.sha1()
    for f in ("ftk_score.cuh", "ftk_device.cuh"):
        path = os.path.join("sparse_attention_indexer_ftk_b200", "csrc", f)
        if read is None:
            with open(os.path.join(ROOT, path)) as fh:
                text = fh.read()
        else:
            text = read(path)
        h.update(strip_comments(text).encode())
    return h.hexdigest()[:12]


class ClockSampler:
    """nvidia-smi clocks / throttle reasons sampled during the timed region."""

    FIELDS = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, gpu_index: int):
        self.idx = gpu_index
        self.proc = None
        self.path = None

    def __enter__(self):
        fd, self.path = tempfile.mkstemp(suffix=".csv")
        os.close(fd)
        try:
            self.proc = subprocess.Popen(
                ["nvidia-smi", f"--query-gpu={self.FIELDS}", "--format=csv,noheader,nounits",
                 "-i", str(self.idx), "-lms", "50", "-f", self.path],
                stdout=subprocess.DEVNULL, stderr=subprocess.DEVNULL)
            time.sleep(0.3)
        except OSError:
            self.proc = None
        return self

    def __exit__(self, *exc):
        if self.proc is not None:
            time.sleep(0.1)
            self.proc.terminate()
            try:
                self.proc.wait(timeout=5)
            except subprocess.TimeoutExpired:
                self.proc.kill()
        return False

    def summary(self):
        rows = []
        try:
            for line in open(self.path):
                p = [x.strip() for x in line.split(",")]
                if len(p) >= 9 and p[1].isdigit():
                    rows.append(p)
        except OSError:
            pass
        finally:
            if self.path:
                try:
                    os.unlink(self.path)
                except OSError:
                    pass
        if not rows:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["unsampled"], "samples": 0}
        sm = [int(r[1]) for r in rows]
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        reasons = sorted({n for r in rows for n, v in zip(names, r[5:9]) if v.lower() == "active"})
        power = []
        for r in rows:
            try:
                power.append(float(r[3]))
            except ValueError:  # "[N/A]" or empty
                pass
        return {"sm_mhz": statistics.median(sm), "sm_max_mhz": int(rows[0][2]), "reasons": reasons,
                "samples": len(rows), "power_w_max": max(power) if power else None}


def gpu_index(local_rank: int) -> int:
    vis = os.environ.get("CUDA_VISIBLE_DEVICES")
    if vis:
        ids = [v for v in vis.split(",") if v.strip()]
        if local_rank < len(ids) and ids[local_rank].strip().isdigit():
            return int(ids[local_rank])
    return local_rank


def cpu_baseline(c, seconds: float):
    """The oracle as it stands, on a bounded row sample of the same workload."""
    from oracle import oracle as orc
    from sparse_attention_indexer_ftk_b200 import workloads as wl

    threads = orc.num_threads()
    n = max(2, threads)
    done, t_total, rows_total = 0, 0.0, 0
    seed = 0
    while t_total < seconds and rows_total < c.T:
        rows = wl.sample_rows(c.T, min(n, c.T), seed=seed)
        t0 = time.perf_counter()
        orc.fused_select(c.q, c.kv, c.kv_scales, c.weights, c.ks, c.ke, c.topk, rows=rows)
        t_total += time.perf_counter() - t0
        rows_total += len(rows)
        seed += 1
        done += 1
    return {"value": rows_total / t_total, "unit": "queries/s", "cores": threads, "kind": "oracle",
            "sample": f"{rows_total} seeded query rows of the {c.T}-row batch (first and last "
                      f"included), fp64 score + full sort per row, {t_total:.1f} s on {threads} threads"}


# Oracle timing per workload configuration: the small BF16 and row top-k
# workloads on all rows, the FP8 workloads on 64 seeded rows (first and
# last included).
ORACLE_CONFIGS = [("bf16_small", None), ("rows_bf16", None), ("rows_f32", None),
                  ("fp8_prefill", 64), ("fp8_packed", 64), ("fp8_large", 64), ("fp8_prefill_64h", 64)]


def oracle_configs():
    """--oracle-configs: one JSON line per configuration with the oracle's
    rows/s on the host cores (no GPU involved)."""
    from oracle import oracle as orc
    from sparse_attention_indexer_ftk_b200 import workloads as wl

    threads = orc.num_threads()
    for name, nrows in ORACLE_CONFIGS:
        c = wl.get(name)
        if isinstance(c, wl.RowsInputs):
            t0 = time.perf_counter()
            orc.topk_rows(c.x, c.topk)
            dt = time.perf_counter() - t0
            rows = c.x.shape[0]
            extra = {"cols": c.x.shape[1], "input_mb": c.x.numel() * c.x.element_size() / 1e6}
        else:
            sel = wl.sample_rows(c.T, nrows or c.T, seed=0)
            t0 = time.perf_counter()
            orc.fused_select(c.q, c.kv, c.kv_scales, c.weights, c.ks, c.ke, c.topk, rows=sel)
            dt = time.perf_counter() - t0
            rows = len(sel)
            L = (c.ke - c.ks).double()
            pairs = float(L[torch_index(sel)].sum())
            heads = c.q.shape[1]
            extra = {"T": c.T, "S": c.S, "heads": heads, "dense_eq_gflops": pairs * 2 * heads * 128 / dt / 1e9}
        print(json.dumps({"workload": name, "kind": "oracle", "rows": rows, "seconds": round(dt, 3),
                          "rows_per_s": rows / dt, "threads": threads, "topk": c.topk, **extra}), flush=True)


def torch_index(rows):
    import torch
    return torch.tensor(rows, dtype=torch.long)


def run_reference(args):
    """--impl reference: the oracle, timed on the host cores (rank 0 only)."""
    ws, rank, _ = dist_env()
    if rank != 0:
        return
    from oracle import oracle as orc
    from sparse_attention_indexer_ftk_b200 import workloads as wl

    c = wl.get(WORKLOAD)
    threads = orc.num_threads()
    per_step = threads  # one query row per host thread: every core busy, a step ~ one row's time
    seed = 0

    def step():
        nonlocal seed
        rows = wl.sample_rows(c.T, per_step, seed=seed)
        seed += 1
        orc.fused_select(c.q, c.kv, c.kv_scales, c.weights, c.ks, c.ke, c.topk, rows=rows)
        return len(rows)

    for _ in range(args.warmup):
        step()
    t0 = time.perf_counter()
    rows = sum(step() for _ in range(args.steps))
    dt = time.perf_counter() - t0
    value = rows / dt
    pairs_per_row = c.pairs() / c.T
    out = {
        "metric": METRIC, "value": value, "unit": "queries/s", "n_gpus": args.gpus,
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": dt / args.steps * 1e3,
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f64",
        "data": "synthetic", "impl": "reference",
        "config": {"workload": WORKLOAD, "T": c.T, "S": c.S, "topk": c.topk, "dtype_in": "fp8_e4m3",
                   "rows_per_step": per_step, "l2": "host"},
        "dense_eq_tflops": value * pairs_per_row * 2 * 32 * 128 / 1e12,
        "cpu_baseline": {"value": value, "unit": "queries/s", "cores": min(threads, per_step), "kind": "oracle",
                         "sample": f"{per_step} seeded query rows per step (one per host thread), "
                                   f"{rows} rows in {dt:.1f} s"},
        "e2e": {"value": value, "unit": "queries/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
    }
    print(json.dumps(out), flush=True)


def bench_rows(name: str, dev, reps: int = 64):
    """Row top-k (ftk_topk_rows) on a row workload, HBM-bound.  Rotates over
    enough input copies that each launch reads data not in the L2."""
    import torch
    from sparse_attention_indexer_ftk_b200 import ftk
    from sparse_attention_indexer_ftk_b200 import workloads as wl

    c = wl.get(name)
    x = c.x.to(dev)
    rows, cols = x.shape
    esz = x.element_size()
    in_bytes = rows * cols * esz
    out_bytes = rows * c.topk * (4 + esz)
    l2 = torch.cuda.get_device_properties(dev).L2_cache_size
    ncopy = max(2, -(-3 * l2 // in_bytes))
    xs = [x.clone() for _ in range(ncopy)]
    oi = torch.empty((rows, c.topk), dtype=torch.int32, device=dev)
    ov = torch.empty((rows, c.topk), dtype=x.dtype, device=dev)
    for i in range(3):
        ftk.topk_rows(xs[i % ncopy], c.topk, out_idx=oi, out_val=ov)
    torch.cuda.synchronize()
    evs = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)) for _ in range(reps)]
    for i in range(reps):
        evs[i][0].record()
        ftk.topk_rows(xs[i % ncopy], c.topk, out_idx=oi, out_val=ov)
        evs[i][1].record()
    torch.cuda.synchronize()
    ms = sorted(a.elapsed_time(b) for a, b in evs)
    mean = sum(ms) / reps

    def timed(fn, rotate: bool) -> float:
        """Mean ms per call of fn(input) over `reps` calls (rotating copies or one)."""
        for i in range(3):
            fn(xs[i % ncopy] if rotate else xs[0])
        torch.cuda.synchronize()
        ev = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)) for _ in range(reps)]
        for i in range(reps):
            ev[i][0].record()
            fn(xs[i % ncopy] if rotate else xs[0])
            ev[i][1].record()
        torch.cuda.synchronize()
        return sum(a.elapsed_time(b) for a, b in ev) / reps

    # The same call with its input resident in L2 (labelled as such), and the
    # bandwidth a trivial read-reduce reaches over the same bytes from HBM
    # (torch.amax: a reference measurement only, not part of the product).
    warm = timed(lambda t: ftk.topk_rows(t, c.topk, out_idx=oi, out_val=ov), rotate=False)
    rr = timed(lambda t: torch.amax(t), rotate=True)
    peaks, src = measured_peaks()
    gbs = (in_bytes + out_bytes) / (mean * 1e-3) / 1e9
    return {"workload": name, "rows": rows, "cols": cols, "topk": c.topk, "dtype": str(x.dtype),
            "us_per_call": mean * 1e3, "us_min": ms[0] * 1e3, "rows_per_s": rows / (mean * 1e-3),
            "roofline": {"bound": "hbm", "achieved": gbs, "peak": peaks["hbm_gbs"], "unit": "GB/s",
                         "frac": gbs / peaks["hbm_gbs"], "bytes_per_call": in_bytes + out_bytes,
                         "peak_source": src},
            "us_per_call_warm_l2": warm * 1e3,
            "read_reduce_baseline": {"op": "torch.amax over the same rotating inputs",
                                     "us_per_call": rr * 1e3,
                                     "gbs": in_bytes / (rr * 1e-3) / 1e9,
                                     "frac": in_bytes / (rr * 1e-3) / 1e9 / peaks["hbm_gbs"]},
            "inputs": f"{ncopy} rotating copies (> L2) so every call reads from HBM"}


def stage_breakdown(ftk, step, flush, n):
    """Per-stage times of n more calls, each with an event recorded at every
    stage boundary.  Separate from the timed calls: recording the events
    costs device time of its own."""
    import torch
    evs = [ftk.stage_events() for _ in range(n)]
    for i in range(n):
        flush.zero_()
        with evs[i]:
            step()
    torch.cuda.synchronize()
    return [e.times_ms() for e in evs]


def bench_decode(c, dev, rows: int = 64, reps: int = 50):
    """A decode-shaped call: the first `rows` query rows of the batch (each
    with its long causal window) through the same ftk_select, inputs in
    HBM, L2 flushed between calls.  Reported beside the metric, not as it."""
    import torch
    from sparse_attention_indexer_ftk_b200 import ftk
    from sparse_attention_indexer_ftk_b200 import workloads as wl

    d = wl.SelectInputs(c.name + f"[:{rows}]", c.q[:rows].contiguous(), c.kv, c.kv_scales,
                        c.weights[:rows].contiguous(), c.ks[:rows].contiguous(),
                        c.ke[:rows].contiguous(), c.topk).to(dev)
    ws = torch.empty(ftk.select_workspace_size(d.T, d.S, d.topk), dtype=torch.uint8, device=dev)
    oi = torch.empty((d.T, d.topk), dtype=torch.int32, device=dev)
    ov = torch.empty((d.T, d.topk), dtype=torch.float32, device=dev)
    flush = torch.empty(256 << 20, dtype=torch.uint8, device=dev)
    step = lambda: ftk.select(d.q, d.kv, d.weights, d.ks, d.ke, d.kv_scales, d.topk, return_scores=True,
                              workspace=ws, out_idx=oi, out_val=ov)
    for _ in range(3):
        step()
    ev = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)) for _ in range(reps)]
    for i in range(reps):
        flush.zero_()
        ev[i][0].record()
        step()
        ev[i][1].record()
    torch.cuda.synchronize()
    ms = sum(a.elapsed_time(b) for a, b in ev) / reps
    stages = stage_breakdown(ftk, step, flush, min(reps, 10))
    info = ftk.read_info(ws)
    pairs = d.pairs()
    return {"workload": d.name, "T": d.T, "S": d.S, "topk": d.topk, "ms_per_call": ms,
            "queries_per_s": d.T / (ms * 1e-3), "dense_eq_tflops": 2.0 * 32 * 128 * pairs / (ms * 1e-3) / 1e12,
            "stage_ms": {name: sum(s[name] for s in stages) / len(stages) for name in stages[0]},
            "kernel_launches": int(info["kernel_launches"]), "prune_enabled": info["prune_enabled"],
            "rows_recovered": info["rows_overflow"] + info["rows_underflow"]}


def fp8_gemm_peak(dev, n: int = 8192, reps: int = 10):
    """Dense FP8-e4m3 GEMM throughput of the vendor library on this GPU
    (torch._scaled_mm, n x n x n, best of `reps`): a measured FP8
    denominator reported beside the roofline's 2 x BF16 one.  A reference
    measurement only; no part of the product calls it."""
    import torch
    try:
        g = torch.Generator(device="cpu").manual_seed(1)
        a = torch.randn((n, n), generator=g).to(dev).to(torch.float8_e4m3fn)
        b = torch.randn((n, n), generator=g).to(dev).to(torch.float8_e4m3fn).t()
        one = torch.ones((), dtype=torch.float32, device=dev)
        mm = lambda: torch._scaled_mm(a, b, scale_a=one, scale_b=one, out_dtype=torch.bfloat16)
        for _ in range(3):
            mm()
        best = float("inf")
        for _ in range(reps):
            e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
            e0.record()
            mm()
            e1.record()
            torch.cuda.synchronize()
            best = min(best, e0.elapsed_time(e1))
        return {"op": f"torch._scaled_mm e4m3 {n}^3, best of {reps}", "tflops": 2.0 * n ** 3 / (best * 1e-3) / 1e12}
    except Exception as e:  # the library may not offer FP8 GEMMs here
        return {"op": "torch._scaled_mm e4m3", "unavailable": str(e)[:200]}


def bench_config(name: str, dev, reps: int = 10):
    """One other workload through the same call: time per call, and the
    pruning decision and pruned share of (row tile, key block) pairs."""
    import torch
    from sparse_attention_indexer_ftk_b200 import ftk
    from sparse_attention_indexer_ftk_b200 import workloads as wl

    d = wl.get(name).to(dev)
    heads = d.q.shape[1]
    ws = torch.empty(ftk.select_workspace_size(d.T, d.S, d.topk, None, heads), dtype=torch.uint8, device=dev)
    oi = torch.empty((d.T, d.topk), dtype=torch.int32, device=dev)
    ov = torch.empty((d.T, d.topk), dtype=torch.float32, device=dev)
    flush = torch.empty(256 << 20, dtype=torch.uint8, device=dev)
    step = lambda: ftk.select(d.q, d.kv, d.weights, d.ks, d.ke, d.kv_scales, d.topk, return_scores=True,
                              workspace=ws, out_idx=oi, out_val=ov)
    for _ in range(3):
        step()
    ev = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)) for _ in range(reps)]
    for i in range(reps):
        flush.zero_()
        ev[i][0].record()
        step()
        ev[i][1].record()
    torch.cuda.synchronize()
    ms = sum(a.elapsed_time(b) for a, b in ev) / reps
    info = ftk.read_info(ws)
    # Tensor roofline of the whole call: the BF16 dense peak for BF16 operands,
    # 2 x that (nominal FP8 : BF16 ratio) for FP8.
    peaks, src = measured_peaks()
    bf16 = d.q.dtype == torch.bfloat16
    peak = peaks["bf16_tflops"] * (1.0 if bf16 else 2.0)
    dense = 2.0 * heads * 128 * d.pairs() / (ms * 1e-3) / 1e12
    rt = (8 if bf16 else 16) // (2 if heads == 64 else 1)
    executed = 2.0 * heads * 128 * (int(info["blocks_total"]) - int(info["blocks_pruned"])) * rt * 128 \
        / (ms * 1e-3) / 1e12
    return {"workload": name, "T": d.T, "S": d.S, "topk": d.topk, "heads": heads,
            "dtype": "bf16 x bf16 -> f32" if bf16 else "fp8_e4m3 x fp8_e4m3 -> f32", "ms_per_call": ms,
            "queries_per_s": d.T / (ms * 1e-3), "dense_eq_tflops": dense, "executed_tflops": executed,
            "roofline": {"bound": "tensor", "achieved": dense, "peak": peak, "unit": "TFLOP/s",
                         "frac": dense / peak,
                         "peak_source": f"{'1' if bf16 else '2'} x bf16_tflops ({src}, burst)",
                         "scope": "whole call (every stage), dense-equivalent work"},
            "prune_enabled": info["prune_enabled"], "blocks_total": info["blocks_total"],
            "blocks_pruned": info["blocks_pruned"],
            "rows_recovered": info["rows_overflow"] + info["rows_underflow"]}


def e2e_pipelined(ftk, host: dict, ws, T: int, k: int, E: int, dev, ref_idx, ref_val):
    """End to end through the public API with the copies overlapped: while
    step j computes, the inputs of step j+1 go up on one stream and the
    results of step j-1 come back on another (device inputs and outputs
    double-buffered, ordered by events).  Every step still copies its own
    inputs from pinned host memory and its own results back.  Returns
    (ms per step, ok): ok says the last step's results, as copied back,
    equal ref_idx / ref_val bit for bit (the same inputs, computed without
    overlap)."""
    import torch
    comp = torch.cuda.current_stream(dev)
    up, down = torch.cuda.Stream(dev), torch.cuda.Stream(dev)
    names = list(host)
    din = [{n: torch.empty(host[n].shape, dtype=host[n].dtype, device=dev) for n in names} for _ in range(2)]
    oidx = [torch.empty((T, k), dtype=torch.int32, device=dev) for _ in range(2)]
    oval = [torch.empty((T, k), dtype=torch.float32, device=dev) for _ in range(2)]
    hidx = [torch.empty((T, k), dtype=torch.int32).pin_memory() for _ in range(2)]
    hval = [torch.empty((T, k), dtype=torch.float32).pin_memory() for _ in range(2)]
    ev_up = [torch.cuda.Event() for _ in range(2)]    # inputs of buffer b are on the device
    ev_comp = [torch.cuda.Event() for _ in range(2)]  # step on buffer b done (inputs free, results ready)
    ev_down = [torch.cuda.Event() for _ in range(2)]  # results of buffer b are on the host
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)

    def issue_up(j):
        b = j % 2
        with torch.cuda.stream(up):
            if j >= 2:
                up.wait_event(ev_comp[b])  # step j-2 has finished reading din[b]
            for n in names:
                din[b][n].copy_(host[n], non_blocking=True)
            ev_up[b].record(up)

    torch.cuda.synchronize(dev)
    e0.record(comp)
    up.wait_event(e0)
    down.wait_event(e0)
    issue_up(0)
    for j in range(E):
        b = j % 2
        if j + 1 < E:
            issue_up(j + 1)
        comp.wait_event(ev_up[b])
        if j >= 2:
            comp.wait_event(ev_down[b])  # the results of step j-2 have left oidx[b] / oval[b]
        d = din[b]
        ftk.select(d["q"], d["kv"], d["weights"], d["ks"], d["ke"], d["kv_scales"], k, return_scores=True,
                   workspace=ws, out_idx=oidx[b], out_val=oval[b])
        ev_comp[b].record(comp)
        with torch.cuda.stream(down):
            down.wait_event(ev_comp[b])
            hidx[b].copy_(oidx[b], non_blocking=True)
            hval[b].copy_(oval[b], non_blocking=True)
            ev_down[b].record(down)
    for j in range(max(0, E - 2), E):
        comp.wait_event(ev_down[j % 2])
    e1.record(comp)
    torch.cuda.synchronize(dev)
    last = (E - 1) % 2
    ok = bool(torch.equal(hidx[last], ref_idx.cpu())
              and torch.equal(hval[last].view(torch.int32), ref_val.cpu().view(torch.int32)))
    return e0.elapsed_time(e1) / E, ok


def bench_sharded(c, g, dev, pg, world: int, rank: int, ref_idx, ref_val, reps: int = 20):
    """One batch split across the ranks: rank r runs ftk_select on its
    contiguous block of query rows (shard.row_shard; kv replicated), the
    step time is the max over ranks, and the blocks gathered on rank 0
    (NCCL, outside the timed region) must equal the single-GPU result of the
    whole batch bit for bit.  Every rank takes the same collective steps."""
    import torch
    from sparse_attention_indexer_ftk_b200 import ftk, shard
    from sparse_attention_indexer_ftk_b200 import workloads as wl

    lo, hi = shard.row_shard(c.T, world, rank)
    d = wl.SelectInputs(c.name + f"[{lo}:{hi}]", g.q[lo:hi].contiguous(), g.kv, g.kv_scales,
                        g.weights[lo:hi].contiguous(), g.ks[lo:hi].contiguous(), g.ke[lo:hi].contiguous(),
                        c.topk)
    ws = torch.empty(ftk.select_workspace_size(d.T, d.S, d.topk), dtype=torch.uint8, device=dev)
    oi = torch.empty((d.T, d.topk), dtype=torch.int32, device=dev)
    ov = torch.empty((d.T, d.topk), dtype=torch.float32, device=dev)
    flush = torch.empty(256 << 20, dtype=torch.uint8, device=dev)
    step = lambda: ftk.select(d.q, d.kv, d.weights, d.ks, d.ke, d.kv_scales, d.topk, return_scores=True,
                              workspace=ws, out_idx=oi, out_val=ov)
    for _ in range(3):
        step()
    ev = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)) for _ in range(reps)]
    pg.barrier()
    torch.cuda.synchronize(dev)
    for i in range(reps):
        flush.zero_()
        ev[i][0].record()
        step()
        ev[i][1].record()
    torch.cuda.synchronize(dev)
    pg.barrier()
    ms = shard.max_over_ranks(sum(a.elapsed_time(b) for a, b in ev) / reps, dev)
    got_idx = shard.gather_rows(oi, c.T, dev)
    got_val = shard.gather_rows(ov, c.T, dev)
    out = {"T": c.T, "rows_per_rank": hi - lo, "ms_per_step": ms, "value": c.T / (ms * 1e-3),
           "unit": "queries/s", "scaling": "strong",
           "gather": "out_idx / out_val gathered on rank 0 (NCCL) after the timed region"}
    if rank == 0:
        out["matches_single_gpu"] = bool(torch.equal(got_idx, ref_idx)
                                         and torch.equal(got_val.view(torch.int32), ref_val.view(torch.int32)))
    return out


def run_ours(args):
    from sparse_attention_indexer_ftk_b200 import shard

    world, rank, local = dist_env()
    # Set up once, destroyed exactly once on the way out (errors included).
    with shard.ProcessGroup(world, local, "nccl") as pg:
        _run_ours(args, pg, world, rank, local)


def _run_ours(args, pg, world, rank, local):
    import torch

    dev = torch.device("cuda", local if world > 1 else 0)
    torch.cuda.set_device(dev)

    from sparse_attention_indexer_ftk_b200 import ftk, shard
    from sparse_attention_indexer_ftk_b200 import workloads as wl

    c = wl.get(WORKLOAD)
    if args.rows and args.rows < c.T:
        c = wl.SelectInputs(c.name, c.q[:args.rows].contiguous(), c.kv, c.kv_scales,
                            c.weights[:args.rows].contiguous(), c.ks[:args.rows].contiguous(),
                            c.ke[:args.rows].contiguous(), c.topk)
    g = c.to(dev)
    T, S, k = c.T, c.S, c.topk
    pairs = c.pairs()
    ws = torch.empty(ftk.select_workspace_size(T, S, k), dtype=torch.uint8, device=dev)
    out_idx = torch.empty((T, k), dtype=torch.int32, device=dev)
    out_val = torch.empty((T, k), dtype=torch.float32, device=dev)
    flush = torch.empty(256 << 20, dtype=torch.uint8, device=dev)
    stream = torch.cuda.current_stream(dev)

    def step():
        ftk.select(g.q, g.kv, g.weights, g.ks, g.ke, g.kv_scales, k, return_scores=True,
                   workspace=ws, out_idx=out_idx, out_val=out_val)

    for _ in range(max(3, args.warmup)):
        step()
    torch.cuda.synchronize()
    info = ftk.read_info(ws)

    barrier = pg.barrier

    K = args.steps
    ev = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)) for _ in range(K)]
    with ClockSampler(gpu_index(local)) as clk:
        barrier()
        torch.cuda.synchronize()
        for i in range(K):
            flush.zero_()  # evict the L2 between timed steps (outside the events)
            ev[i][0].record(stream)
            step()
            ev[i][1].record(stream)
        torch.cuda.synchronize()
        barrier()
    clocks = clk.summary()
    step_ms = [a.elapsed_time(b) for a, b in ev]
    mean_ms = sum(step_ms) / K
    stages = stage_breakdown(ftk, step, flush, min(K, 10))
    stage_mean = {name: sum(s[name] for s in stages) / len(stages) for name in stages[0]}
    mean_ms = shard.max_over_ranks(mean_ms, dev)  # the step time is the slowest rank's

    # end to end through the public API: inputs from pinned host memory,
    # results back to pinned host memory, every step.
    host = {name: getattr(c, name).pin_memory() for name in ("q", "kv", "kv_scales", "weights", "ks", "ke")}
    dev_in = {name: torch.empty_like(getattr(g, name)) for name in host}
    h_idx = torch.empty((T, k), dtype=torch.int32).pin_memory()
    h_val = torch.empty((T, k), dtype=torch.float32).pin_memory()
    h2d = sum(t.numel() * t.element_size() for t in host.values())
    d2h = h_idx.numel() * 4 + h_val.numel() * 4
    E = args.e2e_steps
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    barrier()
    torch.cuda.synchronize()
    e0.record(stream)
    for _ in range(E):
        for name, t in host.items():
            dev_in[name].copy_(t, non_blocking=True)
        ftk.select(dev_in["q"], dev_in["kv"], dev_in["weights"], dev_in["ks"], dev_in["ke"],
                   dev_in["kv_scales"], k, return_scores=True, workspace=ws, out_idx=out_idx,
                   out_val=out_val)
        h_idx.copy_(out_idx, non_blocking=True)
        h_val.copy_(out_val, non_blocking=True)
    e1.record(stream)
    torch.cuda.synchronize()
    serial_ms = e0.elapsed_time(e1) / E
    serial_ms = shard.max_over_ranks(serial_ms, dev)
    # The same with the copies overlapped across steps (a serving loop).
    # Self-checked: the copied-back results must equal the timed run's bits,
    # and no end-to-end step can beat the device-only step; otherwise (or on
    # any error) the serial figure stands.  Every rank takes the same
    # collective steps either way.
    ref_idx, ref_val = out_idx.clone(), out_val.clone()
    pipe_note = ""
    try:
        pipe_ms, pipe_ok = e2e_pipelined(ftk, host, ws, T, k, E, dev, ref_idx, ref_val)
        if not pipe_ok:
            pipe_note = "results differ from the plain run"
        elif pipe_ms < 0.98 * mean_ms:
            pipe_note = f"faster than the device-only step ({pipe_ms:.3f} < {mean_ms:.3f} ms)"
    except Exception as ex:  # noqa: BLE001 -- any failure falls back to the serial figure
        pipe_ms, pipe_note = float("inf"), f"{type(ex).__name__}: {ex}"
    pipe_ms = shard.max_over_ranks(pipe_ms if not pipe_note else float("inf"), dev)
    if pipe_ms != float("inf"):
        e2e_ms, e2e_mode = pipe_ms, ("pipelined: inputs of step j+1 and results of step j-1 copied "
                                      "while step j computes; last step's results checked bit-exact")
    else:
        e2e_ms, e2e_mode = serial_ms, "serial" + (f" (pipelined run rejected: {pipe_note})" if pipe_note else "")

    # One batch split over the ranks (strong scaling), checked against the
    # single-GPU result of the whole batch; every rank takes part.
    sharded = None
    if world > 1:
        sharded = bench_sharded(c, g, dev, pg, world, rank, ref_idx, ref_val)
    if rank != 0:
        return

    peaks, peak_src = measured_peaks()
    fp8_peak = 2.0 * peaks["bf16_tflops"]   # FP8 dense = 2 x BF16 dense (nominal ratio)
    scan_ms = stage_mean["scan"]
    scan_flops = 2.0 * 32 * 128 * pairs
    achieved = scan_flops / (scan_ms * 1e-3) / 1e12
    traffic = profiled_traffic()
    value = world * T / (mean_ms * 1e-3)
    # Executed work: every (16-row tile, 128-key block) pair the scan ran
    # (in-window or not), i.e. minus the pruned ones.
    rt = 16 if c.q.dtype == torch.float8_e4m3fn else 8
    exec_pairs = (int(info["blocks_total"]) - int(info["blocks_pruned"])) * rt * 128
    fp8_direct = fp8_gemm_peak(dev) if world == 1 and not args.no_extras else None
    out = {
        "metric": METRIC,
        "value": value,
        "unit": "queries/s",
        "n_gpus": world,
        "steps": K,
        "warmup": args.warmup,
        "ms_per_step": mean_ms,
        "higher_is_better": True,
        "scaling": "weak",
        "vs_baseline": None,
        "dtype": "fp8_e4m3 x fp8_e4m3 -> f32",
        "data": "synthetic",
        "config": {"workload": WORKLOAD, "T": T, "S": S, "topk": k, "pairs": pairs,
                   "l2": "flushed between steps (256 MB write)", "parallelism": f"dp{world} (independent batches)"},
        "dense_eq_tflops": world * scan_flops / (mean_ms * 1e-3) / 1e12,
        "stage_ms": stage_mean,
        "info": info,
        "roofline": {"kernel": "score_kernel<fp8, COLLECT> (dense scan)", "bound": "tensor",
                     "achieved": achieved, "peak": fp8_peak, "unit": "TFLOP/s",
                     "frac": achieved / fp8_peak, "traffic": traffic,
                     "peak_source": f"2 x bf16_tflops ({peak_src}, burst) -- FP8 dense = 2 x BF16",
                     "frac_of_sustained": achieved / (2.0 * peaks.get("bf16_tflops_sustained", peaks["bf16_tflops"])),
                     "executed_tflops": 2.0 * 32 * 128 * exec_pairs / (scan_ms * 1e-3) / 1e12,
                     "fp8_gemm_measured": fp8_direct,
                     "frac_of_fp8_gemm_measured": (achieved / fp8_direct["tflops"])
                     if fp8_direct and "tflops" in fp8_direct else None},
        "e2e": {"value": world * T / (e2e_ms * 1e-3), "unit": "queries/s",
                "h2d_bytes_per_step": h2d, "d2h_bytes_per_step": d2h, "ms_per_step": e2e_ms,
                "mode": e2e_mode, "steps": E,
                "serial": {"value": world * T / (serial_ms * 1e-3), "ms_per_step": serial_ms}},
        "gpu_launches": int(info["kernel_launches"]) * K,
        "clocks": clocks,
    }
    if world == 1 and not (args.no_decode or args.no_extras):
        out["decode_64q"] = bench_decode(c, dev)
        out["bf16_small"] = bench_config("bf16_small", dev, reps=50)
        out["fp8_packed"] = bench_config("fp8_packed", dev)
        out["fp8_large"] = bench_config("fp8_large", dev, reps=5)
        out["fp8_prefill_64h"] = bench_config("fp8_prefill_64h", dev)
    if world == 1 and not args.no_rows:
        out["row_topk"] = [bench_rows("rows_bf16", dev), bench_rows("rows_f32", dev),
                           bench_rows("rows_bf16_1024", dev, reps=16)]
    if world == 1 and not args.no_cpu_baseline:
        out["cpu_baseline"] = cpu_baseline(c, args.cpu_seconds)
    if sharded is not None:
        out["sharded_one_batch"] = sharded
    print(json.dumps(out), flush=True)


def main():
    args = parse_args()
    if args.oracle_configs:
        oracle_configs()
        return
    if args.only_rows:
        import torch
        dev = torch.device("cuda")
        names = [args.rows_workload] if args.rows_workload else ["rows_bf16", "rows_f32", "rows_bf16_1024"]
        print(json.dumps({"row_topk": [bench_rows(n, dev, reps=16 if n == "rows_bf16_1024" else 64)
                                       for n in names]}), flush=True)
        return
    if args.impl == "reference":
        run_reference(args)
    else:
        run_ours(args)


if __name__ == "__main__":
    main()
