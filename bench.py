"""Benchmark: exact attention forward + backward TFLOPS on B200.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--workload NAME] [--impl ours|reference]
    python bench.py --sweep [--sweep-reps R] [--warmup W]

One step = one pass of the whole hot path over one batch: attn_fwd (O, LSE) then
attn_bwd (dQ, dK, dV) for workloads that train, attn_fwd alone for forward-only
ones.  Inputs are synthetic and seeded (attn_inputs), resident in HBM when the
timed region starts, and larger than the 126 MB L2, so no flush is needed.
Timing uses CUDA events on the launching stream, W warm-up steps, then K steps
bracketed by a barrier and a synchronize; with N > 1 ranks each rank processes
its own batch (independent (b, kv-head) units, no collective on the data path)
and the max time over ranks is reported.

Printed as one JSON line by rank 0.  ``--impl reference`` times the fp64 CPU
oracle instead (the reference arm), on a bounded sample of the same workload.
``--sweep`` times attn_fwd and attn_bwd separately over the sequence-length sweep
(B*N and Hq*d fixed, N from 1K to 32K, d 64 and 128, causal and not) on one GPU
and prints one JSON line per point: the median of R timed calls after W warm-up
calls, each call's inputs larger than L2.
"""
from __future__ import annotations

import argparse
import hashlib
import json
import re
import os
import statistics
import subprocess
import sys
import threading
import time

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

from attn_inputs import (DECODE_WORKLOADS, WINDOW_WORKLOADS, WORKLOADS, Workload, make_decode_inputs,  # noqa: E402
                         make_inputs, sweep_workloads)
from io_aware_exact_26_b200 import accounting as acc  # noqa: E402

# The largest single-GPU workload (forward + backward, causal, d = 128, N = 32768).
DEFAULT_WORKLOAD = "long_causal_b1_h32_n32768_d128"
PEAKS_FILE = os.path.join(ROOT, "MEASURED_PEAKS.json")
TRAFFIC_FILE = os.path.join(ROOT, "profiles", "dram_traffic.json")
FALLBACK_PEAKS = {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0}


def load_peaks():
    try:
        with open(PEAKS_FILE) as f:
            p = json.load(f)
        return p, "measured"
    except (OSError, ValueError):
        return dict(FALLBACK_PEAKS), "fallback"


def code_text(src: str) -> str:
    """CUDA source without comments and with whitespace collapsed: what the compiler sees."""
    src = re.sub(r"/\*.*?\*/", " ", src, flags=re.S)
    src = re.sub(r"//[^\n]*", " ", src)
    return " ".join(src.split())


# The sources each pass's kernels (the ones the bench line times) are compiled from.
# Other kernels of the library (decoding, merges) live in other files and change
# neither.
KERNEL_SOURCES = {"fwd": ("sm100.cuh", "fwd.cuh", "fwd_pp.cuh"), "bwd": ("sm100.cuh", "bwd.cuh")}


def kernel_source_hash(pas="fwd", csrc=None):
    """Fingerprint of one pass's kernel sources; comment or layout edits leave it unchanged."""
    h = hashlib.sha256()
    csrc = csrc or os.path.join(ROOT, "io_aware_exact_26_b200", "csrc")
    for name in KERNEL_SOURCES[pas]:
        with open(os.path.join(csrc, name), encoding="utf-8") as f:
            h.update(name.encode() + code_text(f.read()).encode())
    return h.hexdigest()[:16]


def measured_traffic(workload, kernel):
    """DRAM bytes per launch from a committed ncu capture, if it was taken on this source."""
    try:
        with open(TRAFFIC_FILE) as f:
            t = json.load(f)
    except (OSError, ValueError):
        return None
    e = t.get(workload, {}).get(kernel)
    if not e or e.get("source_hash") != kernel_source_hash(kernel):
        return None
    return e.get("bytes_per_launch")


class ClockSampler:
    """nvidia-smi clocks and throttle reasons sampled while the timed region runs."""

    FIELDS = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, gpu_index):
        self.gpu = gpu_index
        self.proc = None
        self.lines = []
        self.thread = None

    def start(self):
        try:
            self.proc = subprocess.Popen(
                ["nvidia-smi", "-i", str(self.gpu), f"--query-gpu={self.FIELDS}", "--format=csv,noheader,nounits",
                 "-lms", "50"], stdout=subprocess.PIPE, stderr=subprocess.DEVNULL, text=True)
        except OSError:
            self.proc = None
            return
        self.thread = threading.Thread(target=self._read, daemon=True)
        self.thread.start()

    def _read(self):
        for line in self.proc.stdout:
            self.lines.append(line.strip())

    def stop(self):
        if self.proc is None:
            return None
        self.proc.terminate()
        try:
            self.proc.wait(timeout=5)
        except subprocess.TimeoutExpired:
            self.proc.kill()
        if self.thread:
            self.thread.join(timeout=2)
        sm, smax, reasons = [], None, set()
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        for ln in self.lines:
            parts = [x.strip() for x in ln.split(",")]
            if len(parts) < 9:
                continue
            try:
                sm.append(float(parts[1]))
                smax = float(parts[2])
            except ValueError:
                continue
            for n, v in zip(names, parts[5:9]):
                if v.lower() == "active":
                    reasons.add(n)
        if not sm:
            return None
        return {"sm_mhz": statistics.median(sm), "sm_max_mhz": smax, "reasons": sorted(reasons),
                "samples": len(sm)}


def cpu_info():
    """The host the oracle runs on: CPU model, logical CPUs, CPUs this process may use."""
    model = None
    try:
        with open("/proc/cpuinfo") as f:
            for line in f:
                if line.startswith("model name"):
                    model = line.split(":", 1)[1].strip()
                    break
    except OSError:
        pass
    try:
        usable = len(os.sched_getaffinity(0))
    except (AttributeError, OSError):
        usable = os.cpu_count()
    return {"model": model, "logical_cpus": os.cpu_count(), "usable_cpus": usable}


def blas_threads():
    try:
        from threadpoolctl import threadpool_info
        return max((i.get("num_threads", 1) for i in threadpool_info() if i.get("user_api") == "blas"), default=1)
    except Exception:
        return os.cpu_count() or 1


ORACLE_BLOCK = 1024


def time_oracle(w: Workload, budget_s: float, max_blocks=None, min_blocks=1, seed_offset=0):
    """Time the fp64 oracle on 1024-row blocks of one head of the workload.

    Rows are independent, so the oracle's cost for a whole step is the cost of one
    row block times the number of row blocks in the step (B * Hq * ceil(N / 1024));
    the oracle materialises the full masked score block whatever the mask, so every
    block of a head costs the same.  Blocks are drawn from one synthetic head of the
    workload's shape and distribution until ``budget_s`` seconds are spent (at least
    ``min_blocks``).  Returns a dict with the extrapolated step time and rate.
    Test infrastructure: only the baseline legs of the benchmark run the oracle.
    """
    import numpy as np
    from attn_inputs import to_f64
    from oracle import reference as ref
    has_bwd = "bwd" in w.passes
    x = make_inputs(1, 1, 1, w.N, w.d, seed=w.seed + 17 + seed_offset, qk_std=w.qk_std, vo_std=w.vo_std,
                    boost_frac=w.boost_frac, boost=w.boost, with_grad=has_bwd)
    qh, kh, vh = to_f64(x["q"][0, 0]), to_f64(x["k"][0, 0]), to_f64(x["v"][0, 0])
    doh = to_f64(x["do"][0, 0]) if has_bwd else None
    nblk = (w.N + ORACLE_BLOCK - 1) // ORACLE_BLOCK
    order = np.random.default_rng(w.seed + seed_offset).permutation(nblk)
    spent, blocks, rows = 0.0, 0, 0
    while True:
        a = int(order[blocks % nblk]) * ORACLE_BLOCK
        r = np.arange(a, min(w.N, a + ORACLE_BLOCK))
        t0 = time.perf_counter()
        ref.attend_head(qh, kh, vh, w.scale, w.causal, rows=r)
        if has_bwd:
            ref.grad_rows(qh, kh, vh, doh, w.scale, w.causal, r)
        spent += time.perf_counter() - t0
        blocks += 1
        rows += len(r)
        if (spent >= budget_s and blocks >= min_blocks) or (max_blocks and blocks >= max_blocks):
            break
    # step time at the sampled per-row cost (rows of the last block may be fewer)
    step_rows = w.B * w.Hq * w.N
    step_s = spent / rows * step_rows
    return {"tflops": sum(step_flops(w)) / step_s / 1e12, "step_ms": step_s * 1e3, "seconds": spent,
            "blocks": blocks, "rows": rows, "step_rows": step_rows, "threads": blas_threads()}


def single_thread_oracle(budget_s=2.0):
    """The oracle forward with one BLAS thread on the single-head N=256 d=64 workload."""
    try:
        from threadpoolctl import threadpool_limits
    except Exception:
        return None
    w = WORKLOADS["single_head_n256_d64"]
    with threadpool_limits(limits=1, user_api="blas"):
        r = time_oracle(w, budget_s)
    return {"workload": w.name, "tflops": round(r["tflops"], 6), "seconds": round(r["seconds"], 2),
            "calls": r["blocks"], "threads": 1}


def oracle_sample_text(w: Workload, r):
    return (f"{r['blocks']} row blocks of {ORACLE_BLOCK} ({r['rows']} query rows, "
            f"{'forward + backward' if 'bwd' in w.passes else 'forward'}) of one synthetic head of {w.name}, "
            f"{r['seconds']:.1f} s; the step's {r['step_rows']} rows are extrapolated at that per-row cost")


def step_flops(w: Workload):
    f = acc.flops_fwd(w.B, w.Hq, w.N, w.d, w.causal)
    fb = acc.flops_bwd(w.B, w.Hq, w.N, w.d, w.causal) if "bwd" in w.passes else 0.0
    return f, fb


def config_dict(w: Workload, n_gpus, shard=False):
    par = (f"one job, contiguous (b, kv-head) slices over {n_gpus} ranks" if shard
           else f"independent replicas x{n_gpus}")
    return {"workload": w.name, "B": w.B, "Hq": w.Hq, "Hkv": w.Hkv, "N": w.N, "d": w.d, "causal": w.causal,
            "passes": w.passes, "scale": "1/sqrt(d)", "parallelism": par,
            "l2": "inputs larger than L2 (126 MB); no flush"}


def rank_seed(w: Workload, rank: int) -> int:
    """Each rank times its own replica of the workload on its own synthetic inputs."""
    return w.seed + 101 * rank


def shard_units(total, rank, world):
    """Contiguous, balanced slice [u0, u1) of ``total`` independent (b, kv-head) units for
    one rank (the first ``total % world`` ranks take one more)."""
    base, extra = divmod(total, world)
    u0 = rank * base + min(rank, extra)
    return u0, u0 + base + (1 if rank < extra else 0)


def shard_views(x, w, rank, world):
    """This rank's slice of one batch: [B][H][N][d] is [B*H][N][d] in memory, so the
    units [u0, u1) of the flattened (b, kv-head) order are the kv-heads u0..u1-1 and the
    q-heads G*u0..G*u1-1 of a batch of one.  Returns (views, units)."""
    G = w.Hq // w.Hkv
    u0, u1 = shard_units(w.B * w.Hkv, rank, world)
    out = {}
    for n, t in x.items():
        flat = t.view(1, t.shape[0] * t.shape[1], t.shape[2], t.shape[3])
        g = G if n in ("q", "do") else 1
        out[n] = flat[:, u0 * g:u1 * g]
    return out, u1 - u0


def max_over_ranks(values, dist, device):
    """Element-wise max of per-rank timings (the slowest rank sets the job's time)."""
    import torch
    t = torch.tensor(values, dtype=torch.float64, device=device)
    if dist is not None:
        dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return t.tolist()


def weak_scaling_tflops(flops_per_rank, world, ms):
    """Whole-job throughput: every rank processes flops_per_rank in ms (the max over ranks)."""
    return flops_per_rank * world / (ms * 1e-3) / 1e12


def run_reference(args, rank, world):
    """The reference arm: the fp64 oracle on the host cores, a bounded sample per step."""
    if rank != 0:
        return
    w = WORKLOADS[args.workload]
    budget = min(2.0, max(0.2, 90.0 / max(1, args.steps + args.warmup)))
    t_run = time.perf_counter()
    vals, step_ms, blocks, rows, secs = [], [], 0, 0, 0.0
    threads = 1
    for i in range(args.warmup + args.steps):
        r = time_oracle(w, budget, seed_offset=i)
        threads = r["threads"]
        if i >= args.warmup:
            vals.append(r["tflops"])
            step_ms.append(r["step_ms"])
            blocks += r["blocks"]
            rows += r["rows"]
            secs += r["seconds"]
    value = statistics.median(vals) if vals else None
    ms = statistics.median(step_ms) if step_ms else None
    sample = (f"{blocks} row blocks of {ORACLE_BLOCK} ({rows} query rows) of synthetic heads shaped like "
              f"{w.name}, {secs:.1f} s over {args.steps} timed steps; each step's time is extrapolated from "
              f"its own sample at the sampled per-row cost")
    line = {"impl": "reference", "metric": "attention fwd+bwd TFLOPS" if "bwd" in w.passes else "attention fwd TFLOPS",
            "value": value, "unit": "TFLOPS", "n_gpus": args.gpus, "steps": args.steps, "warmup": args.warmup,
            "ms_per_step": ms, "ms_per_step_extrapolated": True, "higher_is_better": True, "scaling": "weak",
            "vs_baseline": None, "dtype": "f64", "data": "synthetic", "config": config_dict(w, args.gpus),
            "cpu_baseline": {"value": value, "unit": "TFLOPS", "cores": threads, "kind": "oracle",
                             "extrapolated": True, "sample": sample, "host": cpu_info()},
            "e2e": {"value": value, "unit": "TFLOPS", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0,
                    "note": "the oracle reads and writes host memory; no copies"},
            "run_seconds": round(time.perf_counter() - t_run, 1)}
    print(json.dumps(line), flush=True)


def run_sweep(args):
    """One JSON line per sweep point: forward and backward timed apart, median over calls."""
    import torch
    import io_aware_exact_26_b200 as attn

    peaks, peaks_kind = load_peaks()
    peak = float(peaks["bf16_tflops"])
    dev = torch.device("cuda", 0)
    torch.cuda.set_device(dev)
    stream = torch.cuda.current_stream()
    for w in sweep_workloads():
        x = make_inputs(w.B, w.Hq, w.Hkv, w.N, w.d, seed=w.seed, device=dev, with_grad=True)
        q, k, v, do = x["q"], x["k"], x["v"], x["do"]
        o = torch.empty_like(q)
        lse = torch.empty((w.B, w.Hq, w.N), dtype=torch.float32, device=dev)
        dq, dk, dv = torch.empty_like(q), torch.empty_like(k), torch.empty_like(v)
        ws = torch.empty(attn.attn_bwd_workspace_size(w.B, w.Hq, w.Hkv, w.N, w.d, w.causal), dtype=torch.uint8,
                         device=dev)

        def fwd():
            attn.attn_fwd(q, k, v, o, lse, scale=w.scale, causal=w.causal)

        def bwd():
            attn.attn_bwd(q, k, v, o, lse, do, dq, dk, dv, scale=w.scale, causal=w.causal, workspace=ws)

        f_fwd, f_bwd = step_flops(w)
        point = {"sweep": "B*N=16384, Hq*d=2048", "workload": w.name, "B": w.B, "Hq": w.Hq, "N": w.N, "d": w.d,
                 "causal": w.causal, "reps": args.sweep_reps, "warmup": args.warmup,
                 "peak": peak, "peak_source": f"{peaks_kind} bf16 dense (burst)"}
        sampler = ClockSampler(0)
        sampler.start()
        for name, fn, flops in (("fwd", fwd, f_fwd), ("bwd", bwd, f_bwd)):
            for _ in range(args.warmup):
                fn()
            evs = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True))
                   for _ in range(args.sweep_reps)]
            for a, b in evs:
                a.record(stream)
                fn()
                b.record(stream)
            torch.cuda.synchronize()
            if attn.attn_get_device_status() != 0:
                raise SystemExit(f"device-side error in the sweep at {w.name} ({name})")
            ms = statistics.median(a.elapsed_time(b) for a, b in evs)
            tf = flops / (ms * 1e-3) / 1e12
            point[name] = {"ms": round(ms, 4), "tflops": round(tf, 1), "frac_of_peak": round(tf / peak, 4)}
        point["clocks"] = sampler.stop()
        print(json.dumps(point), flush=True)
        del x, q, k, v, do, o, lse, dq, dk, dv, ws
        torch.cuda.empty_cache()


def run_decode(args):
    """Split-KV decoding, timed apart: one JSON line per decode workload.  The path is bound
    by HBM, so the roofline is algorithmic bytes (Q, K, V read once, O and LSE written)
    over the event-timed duration, against the measured copy bandwidth."""
    import torch
    import io_aware_exact_26_b200 as attn

    peaks, peaks_kind = load_peaks()
    hbm = float(peaks["hbm_gbs"])
    dev = torch.device("cuda", 0)
    torch.cuda.set_device(dev)
    stream = torch.cuda.current_stream()
    names = [args.decode_workload] if args.decode_workload else list(DECODE_WORKLOADS)
    for name in names:
        w = DECODE_WORKLOADS[name]
        x = make_decode_inputs(w, device=dev)
        o = torch.empty_like(x["q"])
        lse = torch.empty((w.B, w.Hq, w.Nq), dtype=torch.float32, device=dev)
        ws = torch.empty(max(1, attn.attn_decode_workspace_size(w.B, w.Hq, w.Hkv, w.Nq, w.Nk, w.d, w.causal)),
                         dtype=torch.uint8, device=dev)
        # inputs of one call are smaller than L2 for some shapes: rotate through copies
        kv_bytes = 2 * x["k"].numel() * 2
        copies = max(1, -(-2 * 126 * 2 ** 20 // kv_bytes))
        bufs = [x] + [{n: t.clone() for n, t in x.items()} for _ in range(copies - 1)]

        def call(i):
            b = bufs[i % len(bufs)]
            attn.attn_decode(b["q"], b["k"], b["v"], o, lse, scale=w.scale, causal=w.causal, workspace=ws)

        for i in range(args.warmup):
            call(i)
        evs = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True))
               for _ in range(args.sweep_reps)]
        sampler = ClockSampler(0)
        sampler.start()
        for i, (a, b) in enumerate(evs):
            a.record(stream)
            call(i)
            b.record(stream)
        torch.cuda.synchronize()
        clocks = sampler.stop()
        if attn.attn_get_device_status() != 0:
            raise SystemExit(f"device-side error in decode {name}")
        ms = statistics.median(a.elapsed_time(b) for a, b in evs)
        nbytes = acc.min_bytes_decode(w.B, w.Hq, w.Hkv, w.Nq, w.Nk, w.d)
        gbs = nbytes / (ms * 1e-3) / 1e9
        splits = attn.attn_decode_splits(w.B, w.Hq, w.Hkv, w.Nq, w.Nk, w.d, w.causal)
        print(json.dumps({
            "decode": name, "B": w.B, "Hq": w.Hq, "Hkv": w.Hkv, "Nq": w.Nq, "Nk": w.Nk, "d": w.d,
            "causal": w.causal, "splits": splits, "reps": args.sweep_reps, "warmup": args.warmup, "ms": round(ms, 4),
            "tflops": round(acc.flops_decode(w.B, w.Hq, w.Nq, w.Nk, w.d, w.causal) / (ms * 1e-3) / 1e12, 2),
            "roofline": {"bound": "hbm", "achieved": round(gbs, 1), "peak": hbm, "unit": "GB/s",
                         "frac": round(gbs / hbm, 4), "algorithmic_bytes": nbytes,
                         "peak_source": f"{peaks_kind} copy bandwidth"},
            "l2": f"{len(bufs)} input copies rotated (K+V {kv_bytes / 1e6:.0f} MB each)",
            "gpu_launches_per_call": 2 + (splits > 1), "clocks": clocks}), flush=True)
        del x, bufs, o, lse, ws
        torch.cuda.empty_cache()


def run_fp8(args):
    """FP8 forward (e4m3 inputs) next to the bf16 forward on the same shapes, timed apart.
    The fp8 roofline peak is the measured bf16 dense peak times the nominal fp8 : bf16
    ratio of 2 (4.5 vs 2.25 PFLOP/s dense)."""
    import torch
    import io_aware_exact_26_b200 as attn
    from attn_inputs import make_fp8_inputs

    peaks, peaks_kind = load_peaks()
    peak16 = float(peaks["bf16_tflops"])
    dev = torch.device("cuda", 0)
    torch.cuda.set_device(dev)
    stream = torch.cuda.current_stream()
    for name in ("causal_b8_h16_n4096_d128", "long_causal_b1_h32_n32768_d128", "gqa_causal_b4_hq32_hkv8_n8192_d128",
                 "gpt2_medium_b64_h16_n1024_d64"):
        w = WORKLOADS[name]
        x8 = make_fp8_inputs(w.B, w.Hq, w.Hkv, w.N, w.d, seed=w.seed, qk_std=w.qk_std, device=dev)
        x16 = make_inputs(w.B, w.Hq, w.Hkv, w.N, w.d, seed=w.seed, qk_std=w.qk_std, vo_std=w.vo_std,
                          boost_frac=w.boost_frac, boost=w.boost, device=dev, with_grad=False)
        o = torch.empty(x16["q"].shape, dtype=torch.bfloat16, device=dev)
        lse = torch.empty((w.B, w.Hq, w.N), dtype=torch.float32, device=dev)
        calls = {
            "fp8": lambda: attn.attn_fwd_fp8(x8["q"], x8["k"], x8["v"], o, lse, q_descale=x8["q_descale"],
                                             k_descale=x8["k_descale"], v_descale=x8["v_descale"], causal=w.causal),
            "bf16": lambda: attn.attn_fwd(x16["q"], x16["k"], x16["v"], o, lse, scale=w.scale, causal=w.causal)}
        f_fwd = acc.flops_fwd(w.B, w.Hq, w.N, w.d, w.causal)
        line = {"fp8_forward": name, "reps": args.sweep_reps, "warmup": args.warmup}
        sampler = ClockSampler(0)
        sampler.start()
        for kind, fn in calls.items():
            for _ in range(args.warmup):
                fn()
            evs = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True))
                   for _ in range(args.sweep_reps)]
            for a, b in evs:
                a.record(stream)
                fn()
                b.record(stream)
            torch.cuda.synchronize()
            ms = statistics.median(a.elapsed_time(b) for a, b in evs)
            tf = f_fwd / (ms * 1e-3) / 1e12
            peak = peak16 * (2 if kind == "fp8" else 1)
            line[kind] = {"ms": round(ms, 4), "tflops": round(tf, 1), "peak": peak, "frac": round(tf / peak, 4),
                          "peak_source": f"{peaks_kind} bf16 dense (burst)" + (" x 2 (nominal fp8:bf16)" if kind == "fp8"
                                                                             else "")}
        line["clocks"] = sampler.stop()
        if attn.attn_get_device_status() != 0:
            raise SystemExit(f"device-side error in the fp8 run at {name}")
        print(json.dumps(line), flush=True)
        del x8, x16, o, lse
        torch.cuda.empty_cache()


def run_window(args):
    """Local (sliding-window) attention: forward and backward timed apart, TFLOPS over the
    visible (query, key) pairs only, one JSON line per window workload."""
    import torch
    import io_aware_exact_26_b200 as attn

    peaks, peaks_kind = load_peaks()
    peak = float(peaks["bf16_tflops"])
    dev = torch.device("cuda", 0)
    torch.cuda.set_device(dev)
    stream = torch.cuda.current_stream()
    for name, (w, window) in WINDOW_WORKLOADS.items():
        x = make_inputs(w.B, w.Hq, w.Hkv, w.N, w.d, seed=w.seed, device=dev, with_grad=True)
        q, k, v, do = x["q"], x["k"], x["v"], x["do"]
        o = torch.empty_like(q)
        lse = torch.empty((w.B, w.Hq, w.N), dtype=torch.float32, device=dev)
        dq, dk, dv = torch.empty_like(q), torch.empty_like(k), torch.empty_like(v)
        ws = torch.empty(attn.attn_bwd_workspace_size(w.B, w.Hq, w.Hkv, w.N, w.d, False), dtype=torch.uint8,
                         device=dev)
        fns = {"fwd": lambda: attn.attn_fwd_window(q, k, v, o, lse, window=window, scale=w.scale),
               "bwd": lambda: attn.attn_bwd_window(q, k, v, o, lse, do, dq, dk, dv, window=window, scale=w.scale,
                                                   workspace=ws)}
        line = {"window": name, "B": w.B, "Hq": w.Hq, "Hkv": w.Hkv, "N": w.N, "d": w.d, "left": window[0],
                "right": window[1], "reps": args.sweep_reps, "warmup": args.warmup,
                "peak": peak, "peak_source": f"{peaks_kind} bf16 dense (burst)"}
        sampler = ClockSampler(0)
        sampler.start()
        for kind, fn in fns.items():
            for _ in range(args.warmup):      # the forward runs first, so o and lse are set for the backward
                fn()
            evs = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True))
                   for _ in range(args.sweep_reps)]
            for a, b in evs:
                a.record(stream)
                fn()
                b.record(stream)
            torch.cuda.synchronize()
            ms = statistics.median(a.elapsed_time(b) for a, b in evs)
            fl = acc.flops_window(w.B, w.Hq, w.N, w.d, window[0], window[1], bwd=(kind == "bwd"))
            tf = fl / (ms * 1e-3) / 1e12
            line[kind] = {"ms": round(ms, 4), "tflops": round(tf, 1), "frac_of_peak": round(tf / peak, 4)}
        line["clocks"] = sampler.stop()
        if attn.attn_get_device_status() != 0:
            raise SystemExit(f"device-side error in the window run at {name}")
        print(json.dumps(line), flush=True)
        del x, q, k, v, do, o, lse, dq, dk, dv, ws
        torch.cuda.empty_cache()


# Peer-to-peer copy bandwidth per direction per GPU, measured between B200s over
# NVLink 5 and NVSwitch (the ring's exchange is one such copy per step and direction).
PEER_COPY_GBS = 770.0
RING_WORLDS = (2, 4, 8)


def ring_step_bytes(w: Workload, world: int, layout: str):
    """Bytes one rank sends per ring step: the K/V shard it holds (bf16), and in the
    backward also that shard's fp32 dK/dV accumulators, which travel with it."""
    from io_aware_exact_26_b200 import ring
    m = len(ring.shard_chunks(0, world, layout))
    rows = w.N // world                                   # rows per shard (m chunks of N / (m W))
    kv = 2 * w.B * w.Hkv * rows * w.d * 2
    return {"fwd": kv, "bwd": kv + 2 * w.B * w.Hkv * rows * w.d * 4, "chunks_per_shard": m}


def run_ring(args):
    """Sequence parallelism (ring of W ranks), its compute measured on one GPU: the W
    ranks' chunk-pair partials, merges and accumulations (``ring.rank_chunk_pairs``, the
    order ring_attention_fwd / _bwd take them) run one rank after another, each timed
    with CUDA events; no exchange runs.  The link time is modelled from the bytes a rank
    sends per step at the measured peer copy bandwidth.  One JSON line per W."""
    import torch
    import io_aware_exact_26_b200 as attn
    from io_aware_exact_26_b200 import ring

    w = WORKLOADS[args.workload]
    peaks, peaks_kind = load_peaks()
    peak = float(peaks["bf16_tflops"])
    dev = torch.device("cuda", 0)
    torch.cuda.set_device(dev)
    stream = torch.cuda.current_stream()
    x = make_inputs(w.B, w.Hq, w.Hkv, w.N, w.d, seed=w.seed, qk_std=w.qk_std, vo_std=w.vo_std,
                    boost_frac=w.boost_frac, boost=w.boost, device=dev, with_grad=True)
    o, lse = attn.attn_fwd(x["q"], x["k"], x["v"], causal=w.causal)   # the rows' global O and LSE
    f_fwd, f_bwd = step_flops(w)
    layout = "zigzag" if w.causal else "contiguous"
    for world in RING_WORLDS:
        m = len(ring.shard_chunks(0, world, layout))
        nch = m * world
        if w.N % (nch * 128):
            continue
        c = w.N // nch
        ch = lambda t, a: t[:, :, a * c:(a + 1) * c].contiguous()
        qc, kc, vc, doc = ([ch(x[t], a) for a in range(nch)] for t in ("q", "k", "v", "do"))
        oc = [ch(o, a) for a in range(nch)]
        lsec = [lse[:, :, a * c:(a + 1) * c].contiguous() for a in range(nch)]
        shp, kshp = (w.B, w.Hq, c, w.d), (w.B, w.Hkv, c, w.d)
        o_p = torch.empty(shp, dtype=torch.bfloat16, device=dev)
        lse_p = torch.empty(shp[:3], dtype=torch.float32, device=dev)
        o_acc = [torch.empty(shp, dtype=torch.float32, device=dev) for _ in range(m)]
        lse_acc = [torch.empty(shp[:3], dtype=torch.float32, device=dev) for _ in range(m)]
        out = [torch.empty(shp, dtype=torch.bfloat16, device=dev) for _ in range(m)]
        dq_p, dk_p, dv_p = (torch.empty(s_, dtype=torch.bfloat16, device=dev) for s_ in (shp, kshp, kshp))
        dq_acc = [torch.zeros(shp, dtype=torch.float32, device=dev) for _ in range(m)]
        dkv_acc = [[torch.zeros(kshp, dtype=torch.float32, device=dev) for _ in range(2)] for _ in range(m)]
        ws = torch.empty(attn.attn_bwd_workspace_size(w.B, w.Hq, w.Hkv, c, w.d, True), dtype=torch.uint8,
                         device=dev)

        def fwd_rank(pairs):
            for _, i, a, j, b, kind in pairs:
                attn.attn_fwd(qc[a], kc[b], vc[b], o_p, lse_p, causal=(kind == ring.CAUSAL), scale=w.scale)
                attn.attn_merge(o_acc[i], lse_acc[i], o_p, lse_p, out[i])

        def bwd_rank(pairs):
            for _, i, a, j, b, kind in pairs:
                attn.attn_bwd(qc[a], kc[b], vc[b], oc[a], lsec[a], doc[a], dq_p, dk_p, dv_p, scale=w.scale,
                              causal=(kind == ring.CAUSAL), workspace=ws)
                attn.attn_accumulate(dq_acc[i], dq_p)
                attn.attn_accumulate(dkv_acc[j][0], dk_p)
                attn.attn_accumulate(dkv_acc[j][1], dv_p)

        sampler = ClockSampler(0)
        sampler.start()
        ms = {"fwd": [], "bwd": []}
        for r in range(world):
            pairs = ring.rank_chunk_pairs(r, world, w.causal, layout)
            for kind, fn in (("fwd", fwd_rank), ("bwd", bwd_rank)):
                times = []
                for rep in range(args.warmup + args.sweep_reps):
                    for t_ in lse_acc:
                        t_.fill_(float("-inf"))                 # empty accumulators, before the timed region
                    a_, b_ = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
                    a_.record(stream)
                    fn(pairs)
                    b_.record(stream)
                    if rep >= args.warmup:
                        times.append((a_, b_))
                torch.cuda.synchronize()
                ms[kind].append(statistics.median(a_.elapsed_time(b_) for a_, b_ in times))
        clocks = sampler.stop()
        if attn.attn_get_device_status() != 0:
            raise SystemExit(f"device-side error in the ring run at W={world}")
        sb = ring_step_bytes(w, world, layout)
        line = {"ring": w.name, "ranks": world, "layout": layout, "chunk_rows": c, "reps": args.sweep_reps,
                "warmup": args.warmup, "emulated": "the ranks' compute runs one rank after another on one GPU; "
                "no exchange runs; the link time is modelled at the measured peer copy bandwidth",
                "peer_copy_gbs": PEER_COPY_GBS, "peak": peak, "peak_source": f"{peaks_kind} bf16 dense (burst)"}
        for kind, fl in (("fwd", f_fwd), ("bwd", f_bwd)):
            worst = max(ms[kind])
            link_ms = sb[kind] / (PEER_COPY_GBS * 1e9) * 1e3
            step_ms = worst / world                               # compute per ring step (mean over steps)
            modelled = max(worst, world * link_ms)
            line[kind] = {"ms_per_rank": [round(v, 4) for v in ms[kind]], "ms_max_rank": round(worst, 4),
                          "compute_tflops": round(fl / (worst * 1e-3) / 1e12, 1),
                          "compute_tflops_per_gpu": round(fl / (worst * 1e-3) / 1e12 / world, 1),
                          "frac_of_peak_per_gpu": round(fl / (worst * 1e-3) / 1e12 / world / peak, 4),
                          "bytes_sent_per_step": sb[kind], "link_ms_per_step": round(link_ms, 4),
                          "compute_ms_per_step": round(step_ms, 4),
                          "modelled_tflops": round(fl / (modelled * 1e-3) / 1e12, 1)}
        line["clocks"] = clocks
        print(json.dumps(line), flush=True)
        del qc, kc, vc, doc, oc, lsec, o_acc, lse_acc, out, dq_acc, dkv_acc, ws
        torch.cuda.empty_cache()


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=30)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--workload", default=DEFAULT_WORKLOAD, choices=sorted(WORKLOADS))
    ap.add_argument("--impl", default="ours", choices=["ours", "reference"])
    ap.add_argument("--e2e-steps", type=int, default=None,
                    help="end-to-end steps timed (default: --steps); the pipeline's first H2D and last D2H "
                         "are amortised over them")
    ap.add_argument("--cpu-budget", type=float, default=12.0, help="seconds of oracle time for cpu_baseline")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--sweep", action="store_true", help="time the sequence-length sweep, one line per point")
    ap.add_argument("--sweep-reps", type=int, default=50)
    ap.add_argument("--decode", action="store_true", help="time split-KV decoding, one line per decode workload")
    ap.add_argument("--fp8", action="store_true", help="time the fp8 forward next to the bf16 forward")
    ap.add_argument("--window", action="store_true", help="time local (sliding-window) attention, fwd and bwd")
    ap.add_argument("--ring", action="store_true",
                    help="sequence parallelism: each rank's compute of a W-rank ring, emulated on one GPU")
    ap.add_argument("--shard", action="store_true",
                    help="N > 1: split one job's (b, kv-head) units across the ranks (strong scaling) "
                         "instead of running N replicas")
    ap.add_argument("--decode-workload", default=None, choices=sorted(DECODE_WORKLOADS))
    args = ap.parse_args()
    args.warmup = max(3, args.warmup)
    if args.sweep:
        run_sweep(args)
        return
    if args.decode:
        run_decode(args)
        return
    if args.fp8:
        run_fp8(args)
        return
    if args.window:
        run_window(args)
        return
    if args.ring:
        run_ring(args)
        return

    rank = int(os.environ.get("RANK", "0"))
    world = int(os.environ.get("WORLD_SIZE", "1"))
    local = int(os.environ.get("LOCAL_RANK", "0"))

    if args.impl == "reference":
        run_reference(args, rank, world)
        return

    import torch
    import io_aware_exact_26_b200 as attn

    torch.cuda.set_device(local)
    dist = None
    if world > 1:
        import datetime
        import torch.distributed as dist
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120),
                                device_id=torch.device("cuda", local))

    w = WORKLOADS[args.workload]
    has_bwd = "bwd" in w.passes
    dev = torch.device("cuda", local)
    if args.shard:
        # one job split across the ranks: the same inputs everywhere, each rank takes a
        # contiguous slice of the (b, kv-head) units
        full = make_inputs(w.B, w.Hq, w.Hkv, w.N, w.d, seed=w.seed, qk_std=w.qk_std, vo_std=w.vo_std,
                           boost_frac=w.boost_frac, boost=w.boost, device=dev, with_grad=has_bwd)
        views, units = shard_views(full, w, rank, world)
        x = {n: t.contiguous() for n, t in views.items()}
        del full
        w = Workload(w.name, 1, units * (w.Hq // w.Hkv), units, w.N, w.d, w.causal, w.passes, w.qk_std, w.vo_std,
                     w.boost_frac, w.boost, w.seed)
    else:
        x = make_inputs(w.B, w.Hq, w.Hkv, w.N, w.d, seed=rank_seed(w, rank), qk_std=w.qk_std, vo_std=w.vo_std,
                        boost_frac=w.boost_frac, boost=w.boost, device=dev, with_grad=has_bwd)
    q, k, v = x["q"], x["k"], x["v"]
    do = x.get("do")
    o = torch.empty_like(q)
    lse = torch.empty((w.B, w.Hq, w.N), dtype=torch.float32, device=dev)
    if has_bwd:
        dq, dk, dv = torch.empty_like(q), torch.empty_like(k), torch.empty_like(v)
        ws = torch.empty(attn.attn_bwd_workspace_size(w.B, w.Hq, w.Hkv, w.N, w.d, w.causal), dtype=torch.uint8,
                         device=dev)
    stream = torch.cuda.current_stream()

    def step(ev_a=None, ev_b=None, ev_c=None):
        if ev_a is not None:
            ev_a.record(stream)
        attn.attn_fwd(q, k, v, o, lse, scale=w.scale, causal=w.causal)
        if ev_b is not None:
            ev_b.record(stream)
        if has_bwd:
            attn.attn_bwd(q, k, v, o, lse, do, dq, dk, dv, scale=w.scale, causal=w.causal, workspace=ws)
        if ev_c is not None:
            ev_c.record(stream)

    for _ in range(args.warmup):
        step()
    torch.cuda.synchronize()
    if attn.attn_get_device_status() != 0:
        raise SystemExit("device-side error during warm-up")

    evs = [[torch.cuda.Event(enable_timing=True) for _ in range(3)] for _ in range(args.steps)]
    start, stop = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    if dist:
        dist.barrier()
    torch.cuda.synchronize()
    sampler = ClockSampler(local)
    sampler.start()
    time.sleep(0.1)
    start.record(stream)
    for s in range(args.steps):
        step(*evs[s])
    stop.record(stream)
    torch.cuda.synchronize()
    clocks = sampler.stop()
    if dist:
        dist.barrier()
    if attn.attn_get_device_status() != 0:
        raise SystemExit("device-side error during the timed steps")

    total_ms = start.elapsed_time(stop)
    fwd_ms = [a.elapsed_time(b) for a, b, _ in evs]
    bwd_ms = [b.elapsed_time(c) for _, b, c in evs] if has_bwd else []
    total_ms, fwd_avg, bwd_avg = max_over_ranks(
        [total_ms, statistics.mean(fwd_ms), statistics.mean(bwd_ms) if bwd_ms else 0.0], dist, dev)
    ms_per_step = total_ms / args.steps
    f_fwd, f_bwd = step_flops(w)
    # whole-job FLOPs per step: every replica's, or (shard) the one job's
    job_flops = sum(step_flops(WORKLOADS[args.workload])) if args.shard else (f_fwd + f_bwd) * world
    value = job_flops / (ms_per_step * 1e-3) / 1e12

    # ---- end to end through the public API with host buffers (pinned), copies inside the timed region.
    # Each step copies its own inputs from pinned host memory and reads its results (O, LSE and,
    # when it trains, dQ, dK, dV) back to pinned host memory.  Two sets of device buffers and two
    # copy streams let the H2D of step s+1 and the D2H of step s-1 run while step s computes, as a
    # training or serving loop would; the serial figure (copy in, compute, copy out, one step at a
    # time) is reported beside it.
    host = {n: x[n].cpu().pin_memory() for n in x}
    # SHA-256 of each input's bytes as generated (this rank's replica), so a run's inputs can
    # be checked against another run's
    digests = {n: hashlib.sha256(host[n].view(torch.uint8).numpy()).hexdigest() for n in sorted(host)}

    def make_outs():
        out = {"o": torch.empty_like(q), "lse": torch.empty_like(lse)}
        if has_bwd:
            out.update(dq=torch.empty_like(q), dk=torch.empty_like(k), dv=torch.empty_like(v))
        return out

    dev_in = [x, {n: torch.empty_like(t_) for n, t_ in x.items()}]
    dev_out = [make_outs(), make_outs()]
    out_host = [{n: torch.empty(t_.shape, dtype=t_.dtype).pin_memory() for n, t_ in dev_out[0].items()}
                for _ in range(2)]
    h2d = sum(t_.numel() * t_.element_size() for t_ in host.values())
    d2h = sum(t_.numel() * t_.element_size() for t_ in out_host[0].values())
    s_in, s_out = torch.cuda.Stream(device=dev), torch.cuda.Stream(device=dev)

    def compute(b):
        xi, xo = dev_in[b], dev_out[b]
        attn.attn_fwd(xi["q"], xi["k"], xi["v"], xo["o"], xo["lse"], scale=w.scale, causal=w.causal)
        if has_bwd:
            attn.attn_bwd(xi["q"], xi["k"], xi["v"], xo["o"], xo["lse"], xi["do"], xo["dq"], xo["dk"], xo["dv"],
                          scale=w.scale, causal=w.causal, workspace=ws)

    def e2e_run(steps, pipelined):
        """Event-timed ms per step of `steps` end-to-end steps."""
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        in_ready = [torch.cuda.Event() for _ in range(2)]
        done = [torch.cuda.Event() for _ in range(2)]
        out_done = [torch.cuda.Event() for _ in range(2)]
        torch.cuda.synchronize()
        e0.record(stream)
        s_in.wait_event(e0)
        s_out.wait_event(e0)

        def copy_in(b):
            with torch.cuda.stream(s_in):
                for n in host:
                    dev_in[b][n].copy_(host[n], non_blocking=True)
                in_ready[b].record(s_in)

        if pipelined:
            copy_in(0)
        for st in range(steps):
            b = st % 2 if pipelined else 0
            if not pipelined:
                if st >= 1:
                    s_in.wait_event(out_done[0])       # the previous step has finished entirely
                copy_in(b)
            elif st + 1 < steps:
                nb = (st + 1) % 2
                if st >= 1:
                    s_in.wait_event(done[nb])          # buffer nb was read by step st - 1
                copy_in(nb)
            stream.wait_event(in_ready[b])
            if pipelined and st >= 2:
                stream.wait_event(out_done[b])        # step st - 2's results have left buffer b
            compute(b)
            done[b].record(stream)
            s_out.wait_event(done[b])
            with torch.cuda.stream(s_out):
                for n, t_ in dev_out[b].items():
                    out_host[b][n].copy_(t_, non_blocking=True)
                out_done[b].record(s_out)
            if not pipelined:
                stream.wait_event(out_done[b])
        stream.wait_event(out_done[(steps - 1) % 2 if pipelined else 0])
        if pipelined and steps >= 2:
            stream.wait_event(out_done[(steps - 2) % 2])
        e1.record(stream)
        torch.cuda.synchronize()
        return e0.elapsed_time(e1) / steps

    e2e_steps = args.e2e_steps or args.steps
    e2e_run(2, True)                                   # warm-up of the copy paths
    if dist:
        dist.barrier()
    e2e_ms = max_over_ranks([e2e_run(e2e_steps, True)], dist, dev)[0]
    if dist:
        dist.barrier()
    e2e_serial_ms = max_over_ranks([e2e_run(e2e_steps, False)], dist, dev)[0]
    e2e_value = job_flops / (e2e_ms * 1e-3) / 1e12
    e2e_serial = job_flops / (e2e_serial_ms * 1e-3) / 1e12

    # ---- roofline of the dominant kernel (backward when present)
    peaks, peaks_kind = load_peaks()
    peak = float(peaks["bf16_tflops"])
    if has_bwd and bwd_avg >= fwd_avg:
        kname, kflops, kms = "attn_bwd (prep + dK/dV + dQ kernels)", f_bwd, bwd_avg
        traffic = measured_traffic(w.name, "bwd")
    else:
        kname, kflops, kms = "attn_fwd_kernel", f_fwd, fwd_avg
        traffic = measured_traffic(w.name, "fwd")
    achieved = kflops / (kms * 1e-3) / 1e12
    roofline = {"kernel": kname, "bound": "tensor", "achieved": round(achieved, 1), "peak": peak,
                "unit": "TFLOP/s", "frac": round(achieved / peak, 4),
                "frac_of_sustained": round(achieved / float(peaks.get("bf16_tflops_sustained", peak)), 4),
                "peak_source": f"{peaks_kind} bf16 dense (burst)", "traffic": traffic}

    line = {"metric": "attention fwd+bwd TFLOPS" if has_bwd else "attention fwd TFLOPS",
            "value": round(value, 2), "unit": "TFLOPS", "n_gpus": world, "steps": args.steps,
            "warmup": args.warmup, "ms_per_step": round(ms_per_step, 4), "higher_is_better": True,
            "scaling": "strong" if args.shard else "weak", "vs_baseline": None, "dtype": "bf16", "data": "synthetic",
            "config": dict(config_dict(WORKLOADS[args.workload], world, shard=args.shard),
                           inputs={"generator": f"torch.Generator on {dev}, seed {rank_seed(w, rank)} (rank {rank})",
                                   "sha256": digests}),
            "fwd": {"ms": round(fwd_avg, 4), "tflops": round(f_fwd / (fwd_avg * 1e-3) / 1e12, 1),
                    "frac_of_peak": round(f_fwd / (fwd_avg * 1e-3) / 1e12 / peak, 4)},
            "roofline": roofline,
            "e2e": {"value": round(e2e_value, 3), "unit": "TFLOPS", "h2d_bytes_per_step": h2d,
                    "d2h_bytes_per_step": d2h, "ms_per_step": round(e2e_ms, 3),
                    "copies": "pinned host buffers; H2D of step s+1 and D2H of step s-1 overlap step s "
                              "(two device buffer sets, two copy streams); the first step's H2D and the "
                              "last step's D2H are not overlapped and count in the total",
                    "steps": e2e_steps,
                    "serial_value": round(e2e_serial, 3), "serial_ms_per_step": round(e2e_serial_ms, 3)},
            "gpu_launches": args.steps * (5 if has_bwd else 2),   # fwd = counter reset + kernel; bwd = prep + dK/dV + dQ
            "clocks": clocks}
    if has_bwd:
        line["bwd"] = {"ms": round(bwd_avg, 4), "tflops": round(f_bwd / (bwd_avg * 1e-3) / 1e12, 1),
                       "frac_of_peak": round(f_bwd / (bwd_avg * 1e-3) / 1e12 / peak, 4)}
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        r = time_oracle(w, args.cpu_budget)
        line["cpu_baseline"] = {"value": round(r["tflops"], 6), "unit": "TFLOPS", "cores": r["threads"],
                                "kind": "oracle", "extrapolated": True, "step_ms": round(r["step_ms"], 1),
                                "sample": oracle_sample_text(w, r), "host": cpu_info(),
                                "single_thread": single_thread_oracle()}
    if rank == 0:
        print(json.dumps(line), flush=True)
    if dist:
        dist.destroy_process_group()


if __name__ == "__main__":
    main()
