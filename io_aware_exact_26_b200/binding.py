"""Thin ctypes binding over the C ABI in ``include/attn.h``.

Argument marshalling only: shapes are read from the tensors, pointers and the
current CUDA stream are passed through, outputs are allocated with torch when
the caller gives none.  Every step of attention runs in the CUDA library; there
is no CPU or PyTorch fallback, and a missing or unloadable library raises.
"""
from __future__ import annotations

import ctypes
import os

import torch

_HERE = os.path.dirname(os.path.abspath(__file__))
library_path = os.path.join(_HERE, "libattn_b200.so")

ATTN_OK = 0
# Size of the fixed device scratch array behind attn_bwd_noalloc (see include/attn.h).
NOALLOC_SCRATCH_BYTES = 64 << 20
_lib = None


class AttnError(RuntimeError):
    def __init__(self, status: int, what: str):
        self.status = status
        super().__init__(f"{what}: {attn_status_string(status)} ({status})")


checks_library_path = os.path.join(_HERE, "libattn_b200_checks.so")


def lib():
    """Load libattn_b200.so (built by ``__graft_entry__.build()``); raise if it is missing."""
    global _lib
    if _lib is not None:
        return _lib
    _lib = load(library_path)
    return _lib


class use_library:
    """Context manager: route every call of this module through another build of the
    library (e.g. ``checks_library_path``), then restore the previous one."""

    def __init__(self, path):
        self.path = path

    def __enter__(self):
        global _lib
        self.prev = _lib
        _lib = load(self.path)
        return _lib

    def __exit__(self, *exc):
        global _lib
        _lib = self.prev
        return False


def load(path):
    """ctypes handle on a build of the library with every entry point's signature set."""
    if not os.path.exists(path):
        raise ImportError(f"{path} is not built; run __graft_entry__.build()")
    L = ctypes.CDLL(path)
    vp, i, f, sz = ctypes.c_void_p, ctypes.c_int, ctypes.c_float, ctypes.c_size_t
    L.attn_fwd.argtypes = [vp, vp, vp, vp, vp, i, i, i, i, i, f, i, vp]
    L.attn_fwd.restype = i
    L.attn_bwd_workspace_size.argtypes = [i, i, i, i, i, i]
    L.attn_bwd_workspace_size.restype = sz
    L.attn_bwd.argtypes = [vp, vp, vp, vp, vp, vp, vp, vp, vp, i, i, i, i, i, f, i, vp, sz, vp]
    L.attn_bwd.restype = i
    L.attn_fwd_window.argtypes = [vp, vp, vp, vp, vp, i, i, i, i, i, f, i, i, vp]
    L.attn_fwd_window.restype = i
    L.attn_bwd_window.argtypes = [vp, vp, vp, vp, vp, vp, vp, vp, vp, i, i, i, i, i, f, i, i, vp, sz, vp]
    L.attn_bwd_window.restype = i
    L.attn_decode_workspace_size.argtypes = [i, i, i, i, i, i, i]
    L.attn_decode_workspace_size.restype = sz
    L.attn_decode.argtypes = [vp, vp, vp, vp, vp, i, i, i, i, i, i, f, i, vp, sz, vp]
    L.attn_decode.restype = i
    L.attn_decode_splits.argtypes = [i, i, i, i, i, i, i]
    L.attn_decode_splits.restype = i
    L.attn_fwd_fp8.argtypes = [vp, vp, vp, vp, vp, i, i, i, i, i, f, f, f, f, i, vp]
    L.attn_fwd_fp8.restype = i
    L.attn_merge.argtypes = [vp, vp, vp, vp, ctypes.c_longlong, i, vp, vp]
    L.attn_merge.restype = i
    L.attn_accumulate.argtypes = [vp, vp, ctypes.c_longlong, vp]
    L.attn_accumulate.restype = i
    L.attn_bwd_noalloc.argtypes = [vp, vp, vp, vp, vp, vp, vp, vp, vp, i, i, i, i, i, f, i, vp]
    L.attn_bwd_noalloc.restype = i
    L.attn_get_device_status.argtypes = [vp]
    L.attn_get_device_status.restype = i
    L.attn_status_string.argtypes = [i]
    L.attn_status_string.restype = ctypes.c_char_p
    L.attn_selftest_timeout.argtypes = [ctypes.c_longlong, vp]
    L.attn_selftest_timeout.restype = i
    L.attn_checks_enabled.argtypes = []
    L.attn_checks_enabled.restype = i
    L.attn_selftest_bounds.argtypes = [vp]
    L.attn_selftest_bounds.restype = i
    L.attn_selftest_sched.argtypes = [vp, vp]
    L.attn_selftest_sched.restype = i
    return L


def attn_status_string(status: int) -> str:
    return lib().attn_status_string(int(status)).decode()


def _stream_ptr(stream):
    if stream is None:
        stream = torch.cuda.current_stream()
    return ctypes.c_void_p(stream.cuda_stream)


def _ptr(t):
    return ctypes.c_void_p(t.data_ptr()) if t is not None else ctypes.c_void_p(0)


def _check(t, name, dtype=torch.bfloat16):
    if not isinstance(t, torch.Tensor):
        raise TypeError(f"{name} must be a torch.Tensor")
    if t.dtype != dtype:
        raise TypeError(f"{name} must be {dtype}, got {t.dtype}")
    if not t.is_contiguous():
        raise ValueError(f"{name} must be contiguous")


def attn_fwd(q, k, v, o=None, lse=None, *, scale=None, causal=False, stream=None):
    """O = softmax(scale * Q K^T) V and the per-row log-sum-exp; returns (o, lse).

    q: [B, Hq, N, d] bf16; k, v: [B, Hkv, N, d] bf16; o: like q; lse: [B, Hq, N] fp32.
    """
    for t, n in ((q, "q"), (k, "k"), (v, "v")):
        _check(t, n)
    B, Hq, N, d = q.shape
    Hkv = k.shape[1]
    if o is None:
        o = torch.empty_like(q)
    if lse is None:
        lse = torch.empty((B, Hq, N), dtype=torch.float32, device=q.device)
    _check(o, "o")
    _check(lse, "lse", torch.float32)
    if scale is None:
        scale = d ** -0.5
    st = lib().attn_fwd(_ptr(q), _ptr(k), _ptr(v), _ptr(o), _ptr(lse), B, Hq, Hkv, N, d,
                        float(scale), int(bool(causal)), _stream_ptr(stream))
    if st != ATTN_OK:
        raise AttnError(st, "attn_fwd")
    return o, lse


def attn_fwd_fp8(q, k, v, o=None, lse=None, *, q_descale, k_descale, v_descale, scale=None, causal=False,
                 stream=None):
    """Forward with e4m3 Q, K, V (torch.float8_e4m3fn) and per-tensor descales; returns
    (o bf16, lse fp32).  The attended values are q * q_descale etc.; d is 64 or 128."""
    for t, n in ((q, "q"), (k, "k"), (v, "v")):
        _check(t, n, torch.float8_e4m3fn)
    B, Hq, N, d = q.shape
    Hkv = k.shape[1]
    o = torch.empty(q.shape, dtype=torch.bfloat16, device=q.device) if o is None else o
    lse = torch.empty((B, Hq, N), dtype=torch.float32, device=q.device) if lse is None else lse
    _check(o, "o")
    _check(lse, "lse", torch.float32)
    if scale is None:
        scale = d ** -0.5
    st = lib().attn_fwd_fp8(_ptr(q), _ptr(k), _ptr(v), _ptr(o), _ptr(lse), B, Hq, Hkv, N, d, float(scale),
                            float(q_descale), float(k_descale), float(v_descale), int(bool(causal)),
                            _stream_ptr(stream))
    if st != ATTN_OK:
        raise AttnError(st, "attn_fwd_fp8")
    return o, lse


def _window_args(window):
    # (left, right) with None for no limit -> the ABI's convention (negative = no limit)
    left, right = window
    return (-1 if left is None else int(left)), (-1 if right is None else int(right))


def attn_fwd_window(q, k, v, o=None, lse=None, *, window, scale=None, stream=None):
    """Local attention: query i sees keys i - left .. i + right, ``window = (left, right)``
    (None = no limit on that side); returns (o, lse)."""
    for t, n in ((q, "q"), (k, "k"), (v, "v")):
        _check(t, n)
    B, Hq, N, d = q.shape
    Hkv = k.shape[1]
    o = torch.empty_like(q) if o is None else o
    lse = torch.empty((B, Hq, N), dtype=torch.float32, device=q.device) if lse is None else lse
    _check(o, "o")
    _check(lse, "lse", torch.float32)
    if scale is None:
        scale = d ** -0.5
    wl, wr = _window_args(window)
    st = lib().attn_fwd_window(_ptr(q), _ptr(k), _ptr(v), _ptr(o), _ptr(lse), B, Hq, Hkv, N, d,
                               float(scale), wl, wr, _stream_ptr(stream))
    if st != ATTN_OK:
        raise AttnError(st, "attn_fwd_window")
    return o, lse


def attn_bwd_window(q, k, v, o, lse, do, dq=None, dk=None, dv=None, *, window, scale=None, workspace=None,
                    stream=None):
    """Backward of attn_fwd_window for the same ``window``; returns (dq, dk, dv)."""
    for t, n in ((q, "q"), (k, "k"), (v, "v"), (o, "o"), (do, "do")):
        _check(t, n)
    _check(lse, "lse", torch.float32)
    B, Hq, N, d = q.shape
    Hkv = k.shape[1]
    dq = torch.empty_like(q) if dq is None else dq
    dk = torch.empty_like(k) if dk is None else dk
    dv = torch.empty_like(v) if dv is None else dv
    for t, n in ((dq, "dq"), (dk, "dk"), (dv, "dv")):
        _check(t, n)
    if scale is None:
        scale = d ** -0.5
    wl, wr = _window_args(window)
    ws_bytes = 0 if workspace is None else workspace.numel() * workspace.element_size()
    st = lib().attn_bwd_window(_ptr(q), _ptr(k), _ptr(v), _ptr(o), _ptr(lse), _ptr(do), _ptr(dq), _ptr(dk),
                               _ptr(dv), B, Hq, Hkv, N, d, float(scale), wl, wr, _ptr(workspace),
                               ctypes.c_size_t(ws_bytes), _stream_ptr(stream))
    if st != ATTN_OK:
        raise AttnError(st, "attn_bwd_window")
    return dq, dk, dv


def attn_decode(q, k, v, o=None, lse=None, *, scale=None, causal=False, workspace=None, stream=None):
    """Nq query rows against Nk keys, split over the keys and merged by LSE; returns (o, lse).

    q: [B, Hq, Nq, d]; k, v: [B, Hkv, Nk, d] bf16.  causal: the queries are the last Nq
    positions (query i sees keys j <= Nk - Nq + i).  workspace=None lets the library
    allocate the split partials on the stream.
    """
    for t, n in ((q, "q"), (k, "k"), (v, "v")):
        _check(t, n)
    B, Hq, Nq, d = q.shape
    Hkv, Nk = k.shape[1], k.shape[2]
    o = torch.empty_like(q) if o is None else o
    lse = torch.empty((B, Hq, Nq), dtype=torch.float32, device=q.device) if lse is None else lse
    _check(o, "o")
    _check(lse, "lse", torch.float32)
    if scale is None:
        scale = d ** -0.5
    ws_bytes = 0 if workspace is None else workspace.numel() * workspace.element_size()
    st = lib().attn_decode(_ptr(q), _ptr(k), _ptr(v), _ptr(o), _ptr(lse), B, Hq, Hkv, Nq, Nk, d, float(scale),
                           int(bool(causal)), _ptr(workspace), ctypes.c_size_t(ws_bytes), _stream_ptr(stream))
    if st != ATTN_OK:
        raise AttnError(st, "attn_decode")
    return o, lse


def attn_merge(o_acc, lse_acc, o_part, lse_part, out=None, *, stream=None):
    """Merge a partial (o_part bf16, lse_part fp32) into the running (o_acc fp32, lse_acc fp32)
    in place; writes the merged O as bf16 into ``out`` when given."""
    _check(o_acc, "o_acc", torch.float32)
    _check(lse_acc, "lse_acc", torch.float32)
    _check(o_part, "o_part")
    _check(lse_part, "lse_part", torch.float32)
    if out is not None:
        _check(out, "out")
    d = o_acc.shape[-1]
    rows = o_acc.numel() // d
    if o_part.numel() != o_acc.numel() or lse_acc.numel() != rows or lse_part.numel() != rows:
        raise ValueError("attn_merge: shapes of the accumulator and the partial differ")
    st = lib().attn_merge(_ptr(o_acc), _ptr(lse_acc), _ptr(o_part), _ptr(lse_part), rows, d, _ptr(out),
                          _stream_ptr(stream))
    if st != ATTN_OK:
        raise AttnError(st, "attn_merge")
    return o_acc, lse_acc


def attn_accumulate(acc, part, *, stream=None):
    """acc += part in fp32, in place (acc fp32, part bf16, the same number of elements, a
    multiple of 8); returns acc."""
    _check(acc, "acc", torch.float32)
    _check(part, "part")
    if part.numel() != acc.numel():
        raise ValueError("attn_accumulate: the accumulator and the part differ in size")
    st = lib().attn_accumulate(_ptr(acc), _ptr(part), acc.numel(), _stream_ptr(stream))
    if st != ATTN_OK:
        raise AttnError(st, "attn_accumulate")
    return acc


def attn_decode_workspace_size(B, Hq, Hkv, Nq, Nk, d, causal=False) -> int:
    return int(lib().attn_decode_workspace_size(B, Hq, Hkv, Nq, Nk, d, int(bool(causal))))


def attn_decode_splits(B, Hq, Hkv, Nq, Nk, d, causal=False) -> int:
    return int(lib().attn_decode_splits(B, Hq, Hkv, Nq, Nk, d, int(bool(causal))))


def attn_bwd_workspace_size(B, Hq, Hkv, N, d, causal=False) -> int:
    return int(lib().attn_bwd_workspace_size(B, Hq, Hkv, N, d, int(bool(causal))))


def attn_bwd(q, k, v, o, lse, do, dq=None, dk=None, dv=None, *, scale=None, causal=False,
             workspace=None, stream=None):
    """Gradients of sum(O * dO) with respect to q, k, v; returns (dq, dk, dv).

    ``workspace``: a device tensor of at least attn_bwd_workspace_size(...) bytes, or
    None to let the library allocate it on the stream.
    """
    for t, n in ((q, "q"), (k, "k"), (v, "v"), (o, "o"), (do, "do")):
        _check(t, n)
    _check(lse, "lse", torch.float32)
    B, Hq, N, d = q.shape
    Hkv = k.shape[1]
    dq = torch.empty_like(q) if dq is None else dq
    dk = torch.empty_like(k) if dk is None else dk
    dv = torch.empty_like(v) if dv is None else dv
    for t, n in ((dq, "dq"), (dk, "dk"), (dv, "dv")):
        _check(t, n)
    if scale is None:
        scale = d ** -0.5
    # workspace=None passes NULL: the library then takes its workspace with a
    # stream-ordered allocation (cudaMallocAsync / cudaFreeAsync on the stream).
    ws_bytes = 0 if workspace is None else workspace.numel() * workspace.element_size()
    st = lib().attn_bwd(_ptr(q), _ptr(k), _ptr(v), _ptr(o), _ptr(lse), _ptr(do), _ptr(dq),
                        _ptr(dk), _ptr(dv), B, Hq, Hkv, N, d, float(scale), int(bool(causal)),
                        _ptr(workspace), ctypes.c_size_t(ws_bytes), _stream_ptr(stream))
    if st != ATTN_OK:
        raise AttnError(st, "attn_bwd")
    return dq, dk, dv


def attn_bwd_noalloc(q, k, v, o, lse, do, dq, dk, dv, *, scale=None, causal=False, stream=None):
    """attn_bwd for callers that cannot allocate device memory.

    The output tensors must be given (nothing is allocated here or in the
    library); the scratch is the library's fixed device array, so the shape's
    workspace must fit in NOALLOC_SCRATCH_BYTES (64 MiB).  Calls that overlap on
    the GPU race on that array.
    """
    for t, n in ((q, "q"), (k, "k"), (v, "v"), (o, "o"), (do, "do"), (dq, "dq"), (dk, "dk"), (dv, "dv")):
        _check(t, n)
    _check(lse, "lse", torch.float32)
    B, Hq, N, d = q.shape
    Hkv = k.shape[1]
    if scale is None:
        scale = d ** -0.5
    st = lib().attn_bwd_noalloc(_ptr(q), _ptr(k), _ptr(v), _ptr(o), _ptr(lse), _ptr(do), _ptr(dq), _ptr(dk),
                                _ptr(dv), B, Hq, Hkv, N, d, float(scale), int(bool(causal)),
                                _stream_ptr(stream))
    if st != ATTN_OK:
        raise AttnError(st, "attn_bwd_noalloc")
    return dq, dk, dv


def attn_selftest_timeout(limit_ns: int, stream=None) -> None:
    """Launch the bounded-wait self-test (one CTA waits on a barrier nothing arrives on)."""
    st = int(lib().attn_selftest_timeout(int(limit_ns), _stream_ptr(stream)))
    if st != 0:
        raise AttnError(st, "attn_selftest_timeout")


def attn_get_device_status(stream=None) -> int:
    """Synchronise the stream and return (and clear) the device-side error word."""
    return int(lib().attn_get_device_status(_stream_ptr(stream)))


def attn_selftest_bounds(stream=None) -> None:
    """Launch the index-check self-test (records a bounds failure in the checking build only)."""
    st = int(lib().attn_selftest_bounds(_stream_ptr(stream)))
    if st != 0:
        raise AttnError(st, "attn_selftest_bounds")


def attn_selftest_sched(stream=None) -> list:
    """Run the work-counter takeover self-test; returns its six claims (0 1 2 -1 -1 1 expected)."""
    out = torch.full((8,), -7, dtype=torch.int32, device="cuda")
    st = int(lib().attn_selftest_sched(_ptr(out), _stream_ptr(stream)))
    if st != 0:
        raise AttnError(st, "attn_selftest_sched")
    return out[:6].tolist()


def attn_checks_enabled() -> bool:
    return bool(lib().attn_checks_enabled())
