"""Measured issue cost of the tcgen05.mma shapes the attention kernels use, and of tcgen05.ld.

The attention kernels' tensor pipe is fed by M = 128, K = 16 bf16 instructions whose
operands come from shared memory (SS: S = Q K^T, S^T = K Q^T, dP = dO V^T) or
from tensor memory and shared memory (TS: O += P V, dV += P^T dO, dK += dS^T Q,
dQ += dS K).  The dense peak assumes 64 cycles per N = 128 instruction on one SM;
this probe (``bench_mma.cu``) measures what each shape really costs when issued
back to back, so each kernel's ceiling can be stated as the fraction of peak its
instruction mix allows:

    python bench_mma.py                 # JSON lines
    python bench_mma.py --profile       # also writes profiles/mma_issue_rates_b200.md

Needs a GPU; builds ``libbench_mma.so`` next to this file with nvcc on first use.
"""
from __future__ import annotations

import argparse
import ctypes
import json
import os
import subprocess
import sys

import numpy as np

ROOT = os.path.dirname(os.path.abspath(__file__))
SRC = os.path.join(ROOT, "bench_mma.cu")
LIB = os.path.join(ROOT, "libbench_mma.so")    # not bench_mma.so: that name would shadow this module

MODES = {0: ("SS", 128), 1: ("SS", 64), 2: ("TS", 128), 3: ("TS", 64), 4: ("SS", 256)}
SEQUENCES = {5: ("dK/dV step: 8 TS, 8 SS, 8 TS, 8 SS (N = 128)", 32),
             6: ("forward tile: 8 SS, 8 TS (N = 128)", 16)}
PEAK_CYCLES_PER_N = 0.5          # 2 * 128 * 16 flop per N column at 8192 dense bf16 flop/clk/SM


def build(force: bool = False) -> str:
    sys.path.insert(0, ROOT)
    from io_aware_exact_26_b200 import build as B
    if not force and os.path.exists(LIB) and os.path.getmtime(LIB) >= max(os.path.getmtime(SRC),
                                                                         os.path.getmtime(B.HEADERS[0])):
        return LIB
    cmd = [B.nvcc(), *B.NVCC_FLAGS, "-I", os.path.join(ROOT, "include"), "-I", B.CSRC, SRC, "-o", LIB + ".tmp"]
    subprocess.check_call(cmd)
    os.replace(LIB + ".tmp", LIB)
    return LIB


def load():
    L = ctypes.CDLL(build())
    L.probe_mma_rate.argtypes = [ctypes.c_int, ctypes.c_int, ctypes.c_int, ctypes.c_void_p]
    L.probe_tmem_ld_rate.argtypes = [ctypes.c_int, ctypes.c_int, ctypes.c_int, ctypes.c_int, ctypes.c_void_p]
    return L


def mma_rows(L, grid: int, reps: int):
    rows = []
    for mode in list(MODES) + list(SEQUENCES):
        out = np.zeros(2 * grid, dtype=np.uint64)
        if L.probe_mma_rate(mode, 8, grid, out.ctypes.data) != 0:          # warm-up
            raise RuntimeError(f"probe_mma_rate mode {mode} failed")
        if L.probe_mma_rate(mode, reps, grid, out.ctypes.data) != 0:
            raise RuntimeError(f"probe_mma_rate mode {mode} failed")
        if int(out[1::2].min()) != 1:
            raise RuntimeError(f"probe_mma_rate mode {mode}: a wait timed out")
        per_group = 8 if mode in MODES else SEQUENCES[mode][1]
        cyc = out[0::2].astype(np.float64) / (reps * per_group)
        if mode in MODES:
            kind, n = MODES[mode]
            row = {"shape": f"{kind} M=128 N={n} K=16", "cycles": round(float(np.median(cyc)), 2),
                   "math_cycles": n * PEAK_CYCLES_PER_N}
        else:
            row = {"shape": SEQUENCES[mode][0], "cycles": round(float(np.median(cyc)), 2), "math_cycles": 64.0}
        row["fraction_of_peak"] = round(row["math_cycles"] / row["cycles"], 3)
        row["max_over_sms"] = round(float(cyc.max()), 2)
        rows.append(row)
    return rows


def tmem_rows(L, grid: int, reps: int):
    rows = []
    for warps in (4, 8, 16):
        for store in (0, 1):
            out = np.zeros(16 * grid, dtype=np.uint64)
            if L.probe_tmem_ld_rate(8, warps, store, grid, out.ctypes.data) != 0 or \
                    L.probe_tmem_ld_rate(reps, warps, store, grid, out.ctypes.data) != 0:
                raise RuntimeError("probe_tmem_ld_rate failed")
            cyc = out.reshape(grid, 16)[:, :warps].astype(np.float64).max(axis=1) / reps
            it = float(np.median(cyc))
            rows.append({"warps": warps, "store_16_columns": bool(store), "cycles_per_iteration": round(it, 1),
                         "load_bytes_per_clk_per_sm": round(warps * 8192 / it, 1)})
    return rows


def write_profile(mma, tmem, grid, reps, path):
    lines = ["# tcgen05 issue cost on B200 (M = 128, K = 16, bf16 -> fp32)", "",
             "Command:", "", "```", "python bench_mma.py --profile", "```", "",
             f"One CTA per SM on {grid} SMs, {reps} groups of 8 instructions each, issued back to back by one "
             "thread; SM cycles per instruction (median over SMs; the maximum over SMs is beside it). "
             "`math cycles` is the instruction's flops at the dense bf16 rate of 8192 flop/clk/SM.", "",
             "| shape | cycles / instruction | math cycles | fraction of peak | max over SMs |", "|---|---|---|---|---|"]
    for r in mma:
        lines.append(f"| {r['shape']} | {r['cycles']} | {r['math_cycles']:g} | {r['fraction_of_peak']} | "
                     f"{r['max_over_sms']} |")
    lines += ["", "tcgen05.ld bandwidth (each warp loads 64 columns of its 32 lanes, 8 KB, per iteration):", "",
              "| warps | also store 16 columns | cycles / iteration | load bytes / clk / SM |", "|---|---|---|---|"]
    for r in tmem:
        lines.append(f"| {r['warps']} | {'yes' if r['store_16_columns'] else 'no'} | {r['cycles_per_iteration']} | "
                     f"{r['load_bytes_per_clk_per_sm']} |")
    with open(path, "w") as f:
        f.write("\n".join(lines) + "\n")


def main():
    ap = argparse.ArgumentParser(description=__doc__.split("\n\n")[0])
    ap.add_argument("--grid", type=int, default=148)
    ap.add_argument("--reps", type=int, default=2000)
    ap.add_argument("--profile", action="store_true")
    args = ap.parse_args()
    L = load()
    mma = mma_rows(L, args.grid, args.reps)
    tmem = tmem_rows(L, args.grid, args.reps)
    for r in mma + tmem:
        print(json.dumps(r))
    if args.profile:
        write_profile(mma, tmem, args.grid, args.reps, os.path.join(ROOT, "profiles", "mma_issue_rates_b200.md"))


if __name__ == "__main__":
    main()
