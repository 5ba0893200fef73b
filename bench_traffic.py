"""Launch lists and DRAM traffic of the benchmark workloads, from narrow ncu captures.

Two kinds of capture feed ``profiles/``; both run on one GPU, each only after the
same command line has exited 0 without ncu, always with ``--clock-control none``.

1. Launch list (time only, one pass per launch) of the full-size bench command:

       python bench.py --workload W --steps 2 --warmup 3 --no-cpu-baseline --e2e-steps 1 > plain.log 2>&1 && \\
       ncu --metrics gpu__time_duration.sum --clock-control none -c 60 --csv --log-file launches.csv \\
           python bench.py --workload W --steps 2 --warmup 3 --no-cpu-baseline --e2e-steps 1

   ``python bench_traffic.py launches --workload W launches.csv`` writes
   ``profiles/launches_<W>.md`` (per kernel: launches, time, share).

2. DRAM bytes, one kernel per capture (``-k``, ``-c 1``), on a reduced case of the
   same workload: B (or the head counts, keeping Hq/Hkv) divided by ``--div`` so the
   inputs stay a few hundred MB but larger than the 126 MB L2:

       python bench_traffic.py run --workload W --div 4 > plain.log 2>&1 && \\
       ncu --metrics dram__bytes_read.sum,dram__bytes_write.sum,gpu__time_duration.sum --clock-control none \\
           -k regex:attn_bwd_kv -s 1 -c 1 --csv --log-file dram_bwd_kv.csv \\
           python bench_traffic.py run --workload W --div 4

   (one such capture per kernel).  ``python bench_traffic.py dram --workload W --div 4
   dram_*.csv`` scales each kernel's bytes by ``div`` -- every kernel's traffic is a sum
   over independent (b, kv-head) units, so it grows in proportion to their number --
   and writes the workload's entry of ``profiles/dram_traffic.json`` and
   ``profiles/dram_<W>.md``.

Each traffic entry is stamped with ``bench.kernel_source_hash()`` of the tree it runs
on, so bench.py reports it only while the kernels are the ones that were captured.
ncu replays launches serially with cold caches: compare time SHARES with a live run,
not absolute times.
"""
from __future__ import annotations

import argparse
import collections
import csv
import dataclasses
import io
import json
import os
import subprocess
import sys

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

import bench  # noqa: E402
from attn_inputs import sweep_workloads  # noqa: E402

# The benchmark workloads and the sequence-length sweep's points (B*N = 16384, Hq*d = 2048)
ALL_WORKLOADS = {**bench.WORKLOADS, **{w.name: w for w in sweep_workloads()}}

DRAM_METRICS = "dram__bytes_read.sum,dram__bytes_write.sum,gpu__time_duration.sum"
# pipe utilisation read in the same one-kernel capture
PIPE_METRICS = ("sm__pipe_tensor_cycles_active.avg.pct_of_peak_sustained_active,"
                "sm__inst_executed_pipe_xu.avg.pct_of_peak_sustained_active,"
                "smsp__issue_active.avg.pct_of_peak_sustained_active,"
                "sm__cycles_elapsed.avg.per_second")
PIPE_LABELS = {"sm__pipe_tensor_cycles_active.avg.pct_of_peak_sustained_active": "tensor pipe active, % of active cycles",
               "sm__inst_executed_pipe_xu.avg.pct_of_peak_sustained_active": "XU (MUFU) instructions, % of peak",
               "smsp__issue_active.avg.pct_of_peak_sustained_active": "issue slots used, %",
               "sm__cycles_elapsed.avg.per_second": "SM clock during the capture (cycles/s)"}
# kernel name pattern for -k, per kernel of the path, and the pass it belongs to
KERNELS = {"fwd": ("attn_fwd_pp", "fwd"), "bwd_prep": ("attn_bwd_prep", "bwd"),
           "bwd_kv": ("attn_bwd_kv", "bwd"), "bwd_q": ("attn_bwd_q", "bwd")}
_MS = {"nsecond": 1e-6, "ns": 1e-6, "usecond": 1e-3, "us": 1e-3, "msecond": 1.0, "ms": 1.0, "second": 1e3, "s": 1e3}
_BYTES = {"byte": 1.0, "B": 1.0, "Kbyte": 1e3, "KB": 1e3, "Mbyte": 1e6, "MB": 1e6, "Gbyte": 1e9, "GB": 1e9}


def bench_run(workload: str) -> str:
    return f"python bench.py --workload {workload} --steps 2 --warmup 3 --no-cpu-baseline --e2e-steps 1"


def launches_command(workload: str) -> str:
    run = bench_run(workload)
    return (f"{run} > plain.log 2>&1 && \\\nncu --metrics gpu__time_duration.sum --clock-control none -c 60 --csv "
            f"--log-file launches.csv {run}")


def dram_command(workload: str, div: int, kernel: str) -> str:
    run = f"python bench_traffic.py run --workload {workload} --div {div}"
    pat = KERNELS[kernel][0]
    return (f"{run} > plain.log 2>&1 && \\\nncu --metrics {DRAM_METRICS},{PIPE_METRICS} --clock-control none "
            f"-k regex:{pat} -s 1 -c 1 --csv --log-file dram_{kernel}.csv {run}")


def reduced(w, div: int):
    """The workload with its independent (b, kv-head) units divided by ``div``."""
    if div == 1:
        return w
    if w.B % div == 0:
        return dataclasses.replace(w, B=w.B // div)
    if w.Hkv % div == 0:
        return dataclasses.replace(w, Hq=w.Hq // div, Hkv=w.Hkv // div)
    raise ValueError(f"cannot divide {w.name} by {div}")


def kernel_label(name: str) -> str:
    """Kernel name without its argument list and without ``void`` return types."""
    return name.split("(")[0].replace("void ", "").strip()


def parse_launches(text: str):
    """Per kernel (in first-seen order): launches, total ms, and DRAM bytes read and
    written when the capture has them (None otherwise)."""
    rows = list(csv.reader(io.StringIO("\n".join(l for l in text.splitlines() if l.startswith('"')))))
    if not rows:
        raise ValueError("no CSV rows in the ncu log")
    hdr = rows[0]
    ki, mi, ui, vi, idi = (hdr.index(k) for k in ("Kernel Name", "Metric Name", "Metric Unit", "Metric Value", "ID"))
    per_launch = collections.OrderedDict()
    for r in rows[1:]:
        per_launch.setdefault(r[idi], {"name": r[ki]})[r[mi]] = (float(r[vi].replace(",", "")), r[ui])
    agg = collections.OrderedDict()
    for launch in per_launch.values():
        a = agg.setdefault(kernel_label(launch["name"]), {"n": 0, "ms": 0.0, "rd": None, "wr": None, "pipes": {}})
        a["n"] += 1
        for m in PIPE_LABELS:
            if m in launch:
                a["pipes"][m] = launch[m][0]
        v, u = launch["gpu__time_duration.sum"]
        a["ms"] += v * _MS[u]
        for key, tag in (("dram__bytes_read.sum", "rd"), ("dram__bytes_write.sum", "wr")):
            if key in launch:
                v, u = launch[key]
                a[tag] = (a[tag] or 0.0) + v * _BYTES[u]
    return agg


def launch_table(workload: str, agg, note: str) -> str:
    ours = {k for k in agg if k.startswith("attn::")}
    total = sum(a["ms"] for a in agg.values())
    total_ours = sum(agg[k]["ms"] for k in ours) or 1.0
    out = [f"# Launch list: {workload}", "",
           "Command (time only, one pass per launch; ncu replays each launch serially with cold caches: "
           "compare shares, not absolute times):", "",
           "```", launches_command(workload), "```", "",
           f"Summarised by `python bench_traffic.py launches --workload {workload} launches.csv`.", "", note, "",
           "| kernel | launches | total ms | share of all | share of attention kernels | ms / launch |",
           "|---|---|---|---|---|---|"]
    for k, a in agg.items():
        share_ours = f"{100 * a['ms'] / total_ours:.1f}%" if k in ours else "-"
        out.append(f"| `{k}` | {a['n']} | {a['ms']:.3f} | {100 * a['ms'] / total:.1f}% | {share_ours} | "
                   f"{a['ms'] / a['n']:.3f} |")
    return "\n".join(out) + "\n"


def git_revision() -> str:
    try:
        return subprocess.check_output(["git", "-C", ROOT, "rev-parse", "--short", "HEAD"],
                                       stderr=subprocess.DEVNULL, text=True).strip()
    except (OSError, subprocess.CalledProcessError):
        return "unknown"


def write_launches(workload: str, csv_text: str, profiles_dir: str, revision: str | None = None) -> str:
    agg = parse_launches(csv_text)
    w = ALL_WORKLOADS[workload]
    passes = "one attn_fwd and one attn_bwd (prep + dK/dV + dQ kernels)" if "bwd" in w.passes else "one attn_fwd"
    note = (f"Kernel sources: git revision {revision or git_revision()} (source fingerprints: forward "
            f"{bench.kernel_source_hash('fwd')}, backward {bench.kernel_source_hash('bwd')}). The bench step is "
            f"{passes}; the run makes 6 of each (3 warm-up, "
            "2 timed, 1 end-to-end); the at:: kernels are torch's input generation and host-copy casts, "
            "outside the timed region.")
    os.makedirs(profiles_dir, exist_ok=True)
    path = os.path.join(profiles_dir, f"launches_{workload}.md")
    with open(path, "w") as f:
        f.write(launch_table(workload, agg, note))
    return path


def dram_entry(workload: str, div: int, csv_texts, revision: str | None = None, csrc: str | None = None):
    """Per kernel: DRAM bytes of one full-size launch (captured bytes x div); per pass: the
    sum over its kernels, stamped with the fingerprint of that pass's sources (of the
    tree in ``csrc``, default the working tree: pass the captured revision's sources
    when the tree has moved on)."""
    shash = {pas: bench.kernel_source_hash(pas, csrc) for pas in ("fwd", "bwd")}
    kernels = {}
    for text in csv_texts:
        for name, a in parse_launches(text).items():
            if a["rd"] is None:
                raise ValueError(f"{name}: capture has no DRAM metrics")
            key = next((k for k, (pat, _) in KERNELS.items() if pat in name), None)
            if key is None:
                continue
            kernels[key] = {"kernel": name, "captured_bytes": round((a["rd"] + a["wr"]) / a["n"]),
                            "captured_ms": a["ms"] / a["n"], "pipes": a["pipes"],
                            "read_bytes_per_launch": round(a["rd"] / a["n"] * div),
                            "write_bytes_per_launch": round(a["wr"] / a["n"] * div),
                            "bytes_per_launch": round((a["rd"] + a["wr"]) / a["n"] * div)}
    entry = {"div": div, "revision": revision or git_revision(), "kernels": kernels}
    for pas in ("fwd", "bwd"):
        ks = [k for k, (_, p) in KERNELS.items() if p == pas]
        if all(k in kernels for k in ks):
            entry[pas] = {"bytes_per_launch": sum(kernels[k]["bytes_per_launch"] for k in ks),
                          "source_hash": shash[pas]}
    return entry


def dram_table(workload: str, entry) -> str:
    from io_aware_exact_26_b200 import accounting as acc
    w = ALL_WORKLOADS[workload]
    alg = {"fwd": acc.min_bytes_fwd(w.B, w.Hq, w.Hkv, w.N, w.d), "bwd": acc.min_bytes_bwd(w.B, w.Hq, w.Hkv, w.N, w.d)}
    rw = reduced(w, entry["div"])
    out = [f"# DRAM traffic: {workload}", "",
           f"Captured per kernel on the reduced case B={rw.B}, Hq={rw.Hq}, Hkv={rw.Hkv}, N={rw.N}, d={rw.d} "
           f"(the workload's (b, kv-head) units divided by {entry['div']}), one launch each, and scaled by "
           f"{entry['div']} to a full-size launch.  Kernel sources: git revision {entry['revision']} "
           f"(source fingerprints: forward {entry.get('fwd', {}).get('source_hash')}, backward "
           f"{entry.get('bwd', {}).get('source_hash')}).", "", "Commands, one per kernel:", ""]
    for k in entry["kernels"]:
        out += ["```", dram_command(workload, entry["div"], k), "```"]
    out += ["", "| kernel | captured MB | read MB / full launch | write MB / full launch | total MB / full launch |",
            "|---|---|---|---|---|"]
    for k, e in entry["kernels"].items():
        out.append(f"| `{e['kernel']}` | {e['captured_bytes'] / 1e6:.1f} | {e['read_bytes_per_launch'] / 1e6:.1f} | "
                   f"{e['write_bytes_per_launch'] / 1e6:.1f} | {e['bytes_per_launch'] / 1e6:.1f} |")
    pipes = [m for m in PIPE_LABELS if any(m in e["pipes"] for e in entry["kernels"].values())]
    if pipes:
        out += ["", "Pipe counters of the same captures (reduced case, one launch, serialised):", "",
                "| metric | " + " | ".join(f"`{e['kernel']}`" for e in entry["kernels"].values()) + " |",
                "|---|" + "---|" * len(entry["kernels"])]
        out.append("| duration under ncu (ms) | " + " | ".join(f"{e['captured_ms']:.3f}"
                                                           for e in entry["kernels"].values()) + " |")
        for m in pipes:
            vals = []
            for e in entry["kernels"].values():
                v = e["pipes"].get(m)
                vals.append("-" if v is None else (f"{v / 1e9:.3f} GHz" if m.endswith("per_second") else f"{v:.1f}"))
            out.append(f"| {PIPE_LABELS[m]} | " + " | ".join(vals) + " |")
    out += ["", "| pass | DRAM MB / launch | algorithmic minimum MB | ratio |", "|---|---|---|---|"]
    for pas in ("fwd", "bwd"):
        if pas in entry:
            b = entry[pas]["bytes_per_launch"]
            out.append(f"| {pas} | {b / 1e6:.1f} | {alg[pas] / 1e6:.1f} | {b / alg[pas]:.2f} |")
    return "\n".join(out) + "\n"


def write_dram(workload: str, div: int, csv_texts, profiles_dir: str, revision: str | None = None,
               csrc: str | None = None):
    entry = dram_entry(workload, div, csv_texts, revision, csrc)
    path = os.path.join(profiles_dir, "dram_traffic.json")
    try:
        with open(path) as f:
            traffic = json.load(f)
    except (OSError, ValueError):
        traffic = {}
    traffic[workload] = entry
    os.makedirs(profiles_dir, exist_ok=True)
    with open(path, "w") as f:
        json.dump(traffic, f, indent=1)
    with open(os.path.join(profiles_dir, f"dram_{workload}.md"), "w") as f:
        f.write(dram_table(workload, entry))
    return entry


def write_sweep_dram(d: int, causal: bool, csv_dir: str, profiles_dir: str, revision: str | None = None):
    """DRAM bytes of every sweep point at head size ``d`` (causal or not) from per-kernel
    captures named ``dram_<workload>_<kernel>.csv`` in ``csv_dir`` (each point captured
    whole, div 1).  The sweep holds B*N fixed, so the algorithmic bytes are the same at
    every N: traffic that grew with N (re-reads, spilled score tiles) would show as a
    rising ratio.  Writes profiles/dram_sweep_<causal|full>_d<d>.md; returns the rows."""
    from io_aware_exact_26_b200 import accounting as acc
    rows = []
    for w in sweep_workloads():
        if w.d != d or w.causal != causal:
            continue
        texts = []
        for k in ("fwd_pp", "bwd_prep", "bwd_kv", "bwd_q"):
            with open(os.path.join(csv_dir, f"dram_{w.name}_{k}.csv")) as f:
                texts.append(f.read())
        e = dram_entry(w.name, 1, texts, revision)
        alg = {"fwd": acc.min_bytes_fwd(w.B, w.Hq, w.Hkv, w.N, w.d), "bwd": acc.min_bytes_bwd(w.B, w.Hq, w.Hkv, w.N, w.d)}
        rows.append({"workload": w.name, "N": w.N, "B": w.B, "H": w.Hq,
                     "fwd": e["fwd"]["bytes_per_launch"], "bwd": e["bwd"]["bytes_per_launch"],
                     "alg_fwd": alg["fwd"], "alg_bwd": alg["bwd"], "revision": e["revision"]})
    kind = "causal" if causal else "full"
    name = f"dram_sweep_{kind}_d{d}"
    w0 = rows[0]["workload"]
    out = [f"# DRAM traffic over the sequence-length sweep: {kind}, d = {d}", "",
           f"Each point of `bench.py --sweep` (B·N = 16384 tokens, Hq·d = 2048) captured whole, one launch per "
           f"kernel, kernel sources of revision {rows[0]['revision']}. With B·N fixed the algorithmic bytes are the "
           "same at every N (N = 32768 holds 32768 tokens, as B cannot go below 1), so the ratios to the "
           "algorithmic bytes should stay flat: traffic that grew like N² would double from one row to the "
           "next.", "", "Command per point and kernel (here the first point, dK/dV kernel):", "",
           "```", dram_command(w0, 1, "bwd_kv").replace("dram_bwd_kv.csv", f"dram_{w0}_bwd_kv.csv"), "```", "",
           "| N | B×H | fwd DRAM MB | fwd ÷ algorithmic | bwd DRAM MB | bwd ÷ algorithmic | bwd ÷ previous row |",
           "|---|---|---|---|---|---|---|"]
    prev = None
    for r in rows:
        step = "-" if prev is None else f"{r['bwd'] / prev:.2f}"
        out.append(f"| {r['N']} | {r['B']}×{r['H']} | {r['fwd'] / 1e6:.1f} | {r['fwd'] / r['alg_fwd']:.2f} | "
                   f"{r['bwd'] / 1e6:.1f} | {r['bwd'] / r['alg_bwd']:.2f} | {step} |")
        prev = r["bwd"]
    os.makedirs(profiles_dir, exist_ok=True)
    with open(os.path.join(profiles_dir, name + ".md"), "w") as f:
        f.write("\n".join(out) + "\n")
    return rows


def run_case(workload: str, div: int, reps: int):
    """The kernels of one bench step on the reduced case, ``reps`` times (for ncu -k/-s/-c)."""
    import torch
    import io_aware_exact_26_b200 as attn
    from attn_inputs import make_inputs
    w = reduced(ALL_WORKLOADS[workload], div)
    dev = torch.device("cuda", 0)
    x = make_inputs(w.B, w.Hq, w.Hkv, w.N, w.d, seed=w.seed, qk_std=w.qk_std, vo_std=w.vo_std,
                    boost_frac=w.boost_frac, boost=w.boost, device=dev, with_grad=True)
    ws = torch.empty(attn.attn_bwd_workspace_size(w.B, w.Hq, w.Hkv, w.N, w.d, w.causal), dtype=torch.uint8,
                     device=dev)
    for _ in range(reps):
        o, lse = attn.attn_fwd(x["q"], x["k"], x["v"], scale=w.scale, causal=w.causal)
        attn.attn_bwd(x["q"], x["k"], x["v"], o, lse, x["do"], scale=w.scale, causal=w.causal, workspace=ws)
    torch.cuda.synchronize()
    st = attn.attn_get_device_status()
    print(json.dumps({"case": dataclasses.asdict(w), "reps": reps, "status": st}))
    if st != 0:
        raise SystemExit(1)


def main():
    ap = argparse.ArgumentParser(description=__doc__.split("\n\n")[0])
    sub = ap.add_subparsers(dest="cmd", required=True)
    a = sub.add_parser("launches", help="launch table from a time-only ncu launch list")
    a.add_argument("--workload", required=True, choices=sorted(ALL_WORKLOADS))
    a.add_argument("--revision", default=None)
    a.add_argument("--profiles", default=os.path.join(ROOT, "profiles"))
    a.add_argument("csv")
    b = sub.add_parser("dram", help="DRAM bytes per full-size launch from per-kernel captures")
    b.add_argument("--workload", required=True, choices=sorted(ALL_WORKLOADS))
    b.add_argument("--div", type=int, required=True)
    b.add_argument("--revision", default=None)
    b.add_argument("--csrc", default=None, help="kernel sources of the captured revision (default: this tree)")
    b.add_argument("--profiles", default=os.path.join(ROOT, "profiles"))
    b.add_argument("csv", nargs="+")
    e = sub.add_parser("sweep-dram", help="DRAM bytes over the sequence-length sweep from per-kernel captures")
    e.add_argument("--d", type=int, required=True, choices=[64, 128])
    e.add_argument("--causal", action="store_true")
    e.add_argument("--revision", default=None)
    e.add_argument("--profiles", default=os.path.join(ROOT, "profiles"))
    e.add_argument("csv_dir")
    c = sub.add_parser("run", help="run one reduced case of the workload (the program ncu captures)")
    c.add_argument("--workload", required=True, choices=sorted(ALL_WORKLOADS))
    c.add_argument("--div", type=int, default=1)
    c.add_argument("--reps", type=int, default=3)
    args = ap.parse_args()
    if args.cmd == "launches":
        with open(args.csv) as f:
            print(write_launches(args.workload, f.read(), args.profiles, args.revision))
    elif args.cmd == "dram":
        texts = []
        for p in args.csv:
            with open(p) as f:
                texts.append(f.read())
        print(json.dumps({args.workload: write_dram(args.workload, args.div, texts, args.profiles, args.revision,
                                                    args.csrc)}))
    elif args.cmd == "sweep-dram":
        print(json.dumps(write_sweep_dram(args.d, args.causal, args.csv_dir, args.profiles, args.revision)))
    else:
        run_case(args.workload, args.div, args.reps)


if __name__ == "__main__":
    main()
