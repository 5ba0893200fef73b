"""Build libattn_b200.so in-tree with nvcc for sm_100a (no JIT cache, no torch extension)."""
from __future__ import annotations

import os
import subprocess

HERE = os.path.dirname(os.path.abspath(__file__))
ROOT = os.path.dirname(HERE)
CSRC = os.path.join(HERE, "csrc")
OUT = os.path.join(HERE, "libattn_b200.so")
SOURCES = [os.path.join(CSRC, "api.cu")]
HEADERS = [os.path.join(CSRC, f) for f in ("sm100.cuh", "fwd.cuh", "fwd_pp.cuh", "bwd.cuh", "decode.cuh")] + [
    os.path.join(ROOT, "include", "attn.h")]

NVCC_FLAGS = [
    "-gencode", "arch=compute_100a,code=sm_100a",
    "-O3", "-lineinfo", "-std=c++17",
    "-shared", "-Xcompiler", "-fPIC",
    "--expt-relaxed-constexpr",
]


def nvcc():
    for cand in (os.environ.get("NVCC"), "/usr/local/cuda/bin/nvcc", "nvcc"):
        if cand and (os.path.sep not in cand or os.path.exists(cand)):
            return cand
    return "nvcc"


# The checking build: the same sources with ATTN_CHECKS, whose kernels test every index
# they compute and record failures in the error word (see include/attn.h).
OUT_CHECKS = os.path.join(HERE, "libattn_b200_checks.so")


def _build_one(out, extra, force, verbose):
    newest = max(os.path.getmtime(f) for f in SOURCES + HEADERS + [__file__])
    if not force and os.path.exists(out) and os.path.getmtime(out) >= newest:
        return out
    cmd = [nvcc(), *NVCC_FLAGS, *extra, "-I", os.path.join(ROOT, "include"), "-I", CSRC, *SOURCES, "-o", out + ".tmp"]
    if verbose:
        cmd.insert(1, "-Xptxas=-v")
    subprocess.check_call(cmd)
    os.replace(out + ".tmp", out)
    return out


def build(force: bool = False, verbose: bool = False) -> str:
    return _build_one(OUT, [], force, verbose)


def build_checks(force: bool = False) -> str:
    return _build_one(OUT_CHECKS, ["-DATTN_CHECKS"], force, False)


if __name__ == "__main__":
    build(force=True, verbose=True)
