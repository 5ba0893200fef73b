"""Compile the C brute-force oracle (TEST INFRASTRUCTURE ONLY) and load it with ctypes."""
from __future__ import annotations

import ctypes
import os
import subprocess

import numpy as np

HERE = os.path.dirname(os.path.abspath(__file__))
SRC = os.path.join(HERE, "brute.c")
LIB = os.path.join(HERE, "_brute.so")


def build(force: bool = False) -> str:
    if force or not os.path.exists(LIB) or os.path.getmtime(LIB) < os.path.getmtime(SRC):
        subprocess.check_call(["gcc", "-O2", "-std=c99", "-shared", "-fPIC", SRC, "-o", LIB, "-lm"])
    return LIB


_lib = None


def _load():
    global _lib
    if _lib is None:
        _lib = ctypes.CDLL(build())
        dp = ctypes.POINTER(ctypes.c_double)
        ints = [ctypes.c_int] * 5
        _lib.brute_fwd.argtypes = [dp, dp, dp, dp, dp] + ints + [ctypes.c_double] + [ctypes.c_int] * 3
        _lib.brute_bwd.argtypes = [dp] * 7 + ints + [ctypes.c_double] + [ctypes.c_int] * 3
        _lib.brute_fwd.restype = ctypes.c_int
        _lib.brute_bwd.restype = ctypes.c_int
    return _lib


def _ptr(a):
    return a.ctypes.data_as(ctypes.POINTER(ctypes.c_double))


def _wlr(window):
    """(left, right) with None for no limit -> the C convention, -1 for no limit."""
    if window is None:
        return -1, -1
    return tuple(-1 if w is None else int(w) for w in window)


def brute_fwd(q, k, v, scale, causal, window=None):
    q, k, v = (np.ascontiguousarray(x, dtype=np.float64) for x in (q, k, v))
    B, Hq, N, d = q.shape
    o = np.empty_like(q)
    lse = np.empty((B, Hq, N))
    rc = _load().brute_fwd(_ptr(q), _ptr(k), _ptr(v), _ptr(o), _ptr(lse),
                           B, Hq, k.shape[1], N, d, float(scale), int(bool(causal)), *_wlr(window))
    if rc != 0:
        raise ValueError(f"brute_fwd rejected the arguments ({rc})")
    return o, lse


def brute_bwd(q, k, v, do, scale, causal, window=None):
    q, k, v, do = (np.ascontiguousarray(x, dtype=np.float64) for x in (q, k, v, do))
    B, Hq, N, d = q.shape
    dq = np.empty_like(q)
    dk = np.empty_like(k)
    dv = np.empty_like(v)
    rc = _load().brute_bwd(_ptr(q), _ptr(k), _ptr(v), _ptr(do), _ptr(dq), _ptr(dk), _ptr(dv),
                           B, Hq, k.shape[1], N, d, float(scale), int(bool(causal)), *_wlr(window))
    if rc != 0:
        raise ValueError(f"brute_bwd rejected the arguments ({rc})")
    return dq, dk, dv
