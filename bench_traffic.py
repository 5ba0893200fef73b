"""DRAM traffic of one bench.py run, from an ncu launch list.

Turns the CSV of an ncu launch list into ``profiles/launches_<workload>.md`` (per kernel:
launches, time, share, DRAM bytes per launch) and into the workload's entry in
``profiles/dram_traffic.json``, which bench.py reports as ``roofline.traffic``.

The capture runs on one GPU, after the same command has exited 0 without ncu:

    python bench.py --workload W --steps 1 --warmup 3 --no-cpu-baseline --e2e-steps 1 > plain.log 2>&1 && \\
    ncu --metrics gpu__time_duration.sum,dram__bytes_read.sum,dram__bytes_write.sum --clock-control none \\
        -c 200 --csv --log-file launches.csv \\
        python bench.py --workload W --steps 1 --warmup 3 --no-cpu-baseline --e2e-steps 1

and then, on the same source tree:

    python bench_traffic.py --workload W launches.csv

Each entry is stamped with ``bench.kernel_source_hash()`` of the tree it runs on, so
bench.py uses it only while the kernels are the ones that were captured.  ncu replays
every launch serially with cold caches: compare the time SHARES with a live run, not
the absolute times.
"""
from __future__ import annotations

import argparse
import collections
import csv
import io
import json
import os
import subprocess
import sys

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

import bench  # noqa: E402

METRICS = "gpu__time_duration.sum,dram__bytes_read.sum,dram__bytes_write.sum"
_MS = {"nsecond": 1e-6, "ns": 1e-6, "usecond": 1e-3, "us": 1e-3, "msecond": 1.0, "ms": 1.0, "second": 1e3, "s": 1e3}
_BYTES = {"byte": 1.0, "B": 1.0, "Kbyte": 1e3, "KB": 1e3, "Mbyte": 1e6, "MB": 1e6, "Gbyte": 1e9, "GB": 1e9}


def capture_command(workload: str) -> str:
    sel = "" if workload == bench.DEFAULT_WORKLOAD else f" --workload {workload}"
    run = f"python bench.py{sel} --steps 1 --warmup 3 --no-cpu-baseline --e2e-steps 1"
    return (f"{run} > plain.log 2>&1 && \\\nncu --metrics {METRICS} --clock-control none -c 200 --csv "
            f"--log-file launches.csv {run}")


def kernel_label(name: str) -> str:
    """Kernel name without its argument list and without ``void`` return types."""
    return name.split("(")[0].replace("void ", "").strip()


def parse_launches(text: str):
    """Per kernel (in first-seen order): launches, total ms, DRAM bytes read and written."""
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
        a = agg.setdefault(kernel_label(launch["name"]), {"n": 0, "ms": 0.0, "rd": 0.0, "wr": 0.0})
        a["n"] += 1
        v, u = launch["gpu__time_duration.sum"]
        a["ms"] += v * _MS[u]
        for key, tag in (("dram__bytes_read.sum", "rd"), ("dram__bytes_write.sum", "wr")):
            v, u = launch[key]
            a[tag] += v * _BYTES[u]
    return agg


def pass_bytes(agg):
    """DRAM bytes per call of each pass: the forward's kernels, the backward's kernels."""
    def per_call(pred):
        return round(sum((a["rd"] + a["wr"]) / a["n"] for k, a in agg.items() if pred(k)))
    return {"fwd": per_call(lambda k: "attn_fwd" in k or "sched_reset" in k),
            "bwd": per_call(lambda k: "attn_bwd" in k)}


def launch_table(workload: str, agg, note: str) -> str:
    ours = {k for k in agg if k.startswith("attn::")}
    total = sum(a["ms"] for a in agg.values())
    total_ours = sum(agg[k]["ms"] for k in ours) or 1.0
    out = [f"# Launch list: {workload}", "",
           "Command (ncu replays each launch serially with cold caches: compare shares, not absolute times):", "",
           "```", capture_command(workload), "```", "",
           f"Summarised by `python bench_traffic.py --workload {workload} launches.csv`.", "", note, "",
           "| kernel | launches | total ms | share of all | share of attention kernels | ms / launch | "
           "DRAM read MB / launch | DRAM write MB / launch |",
           "|---|---|---|---|---|---|---|---|"]
    for k, a in agg.items():
        share_ours = f"{100 * a['ms'] / total_ours:.1f}%" if k in ours else "-"
        out.append(f"| `{k}` | {a['n']} | {a['ms']:.3f} | {100 * a['ms'] / total:.1f}% | {share_ours} | "
                   f"{a['ms'] / a['n']:.3f} | {a['rd'] / a['n'] / 1e6:.1f} | {a['wr'] / a['n'] / 1e6:.1f} |")
    return "\n".join(out) + "\n"


def git_revision() -> str:
    try:
        return subprocess.check_output(["git", "-C", ROOT, "rev-parse", "--short", "HEAD"],
                                       stderr=subprocess.DEVNULL, text=True).strip()
    except (OSError, subprocess.CalledProcessError):
        return "unknown"


def update(workload: str, csv_text: str, profiles_dir: str, revision: str | None = None):
    """Write the launch table and merge this workload's entry into dram_traffic.json."""
    agg = parse_launches(csv_text)
    shash = bench.kernel_source_hash()
    rev = revision or git_revision()
    w = bench.WORKLOADS[workload]
    passes = "one attn_fwd and one attn_bwd (prep + dK/dV + dQ kernels)" if "bwd" in w.passes else "one attn_fwd"
    note = (f"Kernel sources: git revision {rev} (kernel source hash {shash}). The bench step is {passes}; "
            "the run makes 6 of each (3 warm-up, 1 timed, 2 end-to-end); the at:: kernels are torch's "
            "input generation and host-copy casts, outside the timed region.")
    os.makedirs(profiles_dir, exist_ok=True)
    with open(os.path.join(profiles_dir, f"launches_{workload}.md"), "w") as f:
        f.write(launch_table(workload, agg, note))
    path = os.path.join(profiles_dir, "dram_traffic.json")
    try:
        with open(path) as f:
            traffic = json.load(f)
    except (OSError, ValueError):
        traffic = {}
    per_pass = pass_bytes(agg)
    traffic[workload] = {p: {"bytes_per_launch": b, "source_hash": shash} for p, b in per_pass.items()
                         if b > 0 and (p == "fwd" or "bwd" in w.passes)}
    with open(path, "w") as f:
        json.dump(traffic, f, indent=1)
    return traffic[workload]


def main():
    ap = argparse.ArgumentParser(description=__doc__.split("\n\n")[0])
    ap.add_argument("--workload", required=True, choices=sorted(bench.WORKLOADS))
    ap.add_argument("--revision", default=None, help="git revision the capture was taken on (default: HEAD)")
    ap.add_argument("--profiles", default=os.path.join(ROOT, "profiles"))
    ap.add_argument("csv", help="the ncu --csv --log-file output")
    args = ap.parse_args()
    with open(args.csv) as f:
        entry = update(args.workload, f.read(), args.profiles, args.revision)
    print(json.dumps({args.workload: entry}))


if __name__ == "__main__":
    main()
