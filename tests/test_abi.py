"""The C ABI: the library loads, exports every symbol include/attn.h declares, and
rejects bad arguments on the host before any launch (no GPU needed for these)."""
import ctypes
import os
import re

import pytest

import __graft_entry__
from io_aware_exact_26_b200 import binding

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


@pytest.fixture(scope="module")
def L():
    __graft_entry__.build()
    return binding.lib()


def declared_functions():
    text = open(os.path.join(ROOT, "include", "attn.h")).read()
    text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
    return sorted(set(re.findall(r"\b(attn_[a-z0-9_]+)\s*\(", text)))


def test_header_declares_the_boundary():
    assert declared_functions() == sorted(
        ["attn_fwd", "attn_bwd", "attn_bwd_noalloc", "attn_bwd_workspace_size", "attn_get_device_status",
         "attn_status_string", "attn_selftest_timeout", "attn_fwd_window", "attn_bwd_window", "attn_decode",
         "attn_decode_workspace_size", "attn_decode_splits", "attn_merge", "attn_fwd_fp8", "attn_checks_enabled",
         "attn_selftest_bounds", "attn_selftest_sched", "attn_accumulate"])


def test_every_declared_symbol_is_exported(L):
    for name in declared_functions():
        assert hasattr(L, name), name


def test_status_strings(L):
    texts = {code: binding.attn_status_string(code) for code in range(-9, 1)}
    assert all(t and t != "unknown status" for t in texts.values())
    assert len(set(texts.values())) == len(texts)
    assert binding.attn_status_string(-99) == "unknown status"


def _have_gpu():
    try:
        import torch
        return torch.cuda.is_available()
    except Exception:
        return False


HAVE_GPU = _have_gpu()
FAKE = ctypes.c_void_p(0x10000)       # 16-byte aligned, never dereferenced on these paths
ODD = ctypes.c_void_p(0x10008)


def fwd(L, q=FAKE, k=FAKE, v=FAKE, o=FAKE, lse=FAKE, B=1, Hq=1, Hkv=1, N=128, d=64, scale=0.125, causal=0):
    return L.attn_fwd(q, k, v, o, lse, B, Hq, Hkv, N, d, scale, causal, None)


@pytest.mark.parametrize("kw,code", [
    (dict(d=96), -2), (dict(d=256), -2), (dict(N=0), -1), (dict(B=0), -1), (dict(Hq=3, Hkv=2), -1),
    (dict(Hkv=0), -1), (dict(scale=float("nan")), -1), (dict(scale=float("inf")), -1), (dict(scale=-1.0), -1),
    (dict(causal=2), -1), (dict(q=ctypes.c_void_p(0)), -1), (dict(lse=ctypes.c_void_p(0)), -1),
    (dict(q=ODD), -3), (dict(o=ODD), -3), (dict(lse=ODD), -3),
])
def test_fwd_rejects_bad_arguments(L, kw, code):
    assert fwd(L, **kw) == code


@pytest.mark.skipif(HAVE_GPU, reason="fake pointers would reach a launch on a GPU")
def test_null_workspace_passes_validation(L):
    # Without a device the call gets past every argument check and stops at the device
    # query; a NULL workspace is not rejected as missing (the library would allocate it).
    size = L.attn_bwd_workspace_size(1, 2, 1, 300, 128, 1)
    st = L.attn_bwd(FAKE, FAKE, FAKE, FAKE, FAKE, FAKE, FAKE, FAKE, FAKE, 1, 2, 1, 300, 128, 0.1, 1,
                    ctypes.c_void_p(0), ctypes.c_size_t(0), None)
    assert size > 0 and st == -2


def test_bwd_rejects_bad_arguments(L):
    size = L.attn_bwd_workspace_size(1, 2, 1, 300, 128, 1)
    assert size > 0
    assert L.attn_bwd_workspace_size(1, 3, 2, 300, 128, 1) == 0
    assert L.attn_bwd_workspace_size(1, 2, 1, 300, 96, 1) == 0

    def bwd(ws=FAKE, wsb=size, dq=FAKE, d=128, Hq=2, Hkv=1):
        return L.attn_bwd(FAKE, FAKE, FAKE, FAKE, FAKE, FAKE, dq, FAKE, FAKE, 1, Hq, Hkv, 300, d, 0.1, 1,
                          ws, ctypes.c_size_t(wsb), None)
    assert bwd(wsb=size - 1) == -6
    assert bwd(dq=ODD) == -3
    assert bwd(dq=ctypes.c_void_p(0)) == -1
    assert bwd(d=80) == -2
    assert bwd(Hq=3, Hkv=2) == -1
    assert bwd(Hq=3) == -6   # valid shape, but the workspace was sized for Hq=2


def test_workspace_size_grows_linearly_in_n(L):
    a = L.attn_bwd_workspace_size(2, 8, 2, 4096, 128, 1)
    b = L.attn_bwd_workspace_size(2, 8, 2, 8192, 128, 1)
    assert 1.9 < b / a < 2.1


def test_binding_fails_loudly_without_library(monkeypatch, tmp_path):
    monkeypatch.setattr(binding, "_lib", None)
    monkeypatch.setattr(binding, "library_path", str(tmp_path / "missing.so"))
    with pytest.raises(ImportError):
        binding.lib()


def test_selftest_sched_rejects_null_and_misaligned_output(L):
    assert L.attn_selftest_sched(None, None) == -1
    assert L.attn_selftest_sched(ctypes.c_void_p(0x1002), None) == -3


def test_selftest_timeout_rejects_out_of_range_limits(L):
    assert L.attn_selftest_timeout(0, None) == -1
    assert L.attn_selftest_timeout(-5, None) == -1
    assert L.attn_selftest_timeout(2_000_000_000, None) == -1


def test_window_entry_points_validate_like_the_plain_ones(L):
    def fwdw(q=FAKE, d=64, N=128, scale=0.125, wl=16, wr=0):
        return L.attn_fwd_window(q, FAKE, FAKE, FAKE, FAKE, 1, 1, 1, N, d, scale, wl, wr, None)
    assert fwdw(d=96) == -2
    assert fwdw(N=0) == -1
    assert fwdw(scale=-1.0) == -1
    assert fwdw(q=ODD) == -3
    assert fwdw(q=ctypes.c_void_p(0)) == -1
    size = L.attn_bwd_workspace_size(1, 2, 1, 300, 128, 0)

    def bwdw(wsb=size, dq=FAKE, d=128):
        return L.attn_bwd_window(FAKE, FAKE, FAKE, FAKE, FAKE, FAKE, dq, FAKE, FAKE, 1, 2, 1, 300, d, 0.1, 31, 0,
                                 FAKE, ctypes.c_size_t(wsb), None)
    assert bwdw(wsb=size - 1) == -6
    assert bwdw(dq=ODD) == -3
    assert bwdw(d=80) == -2


def test_decode_validates_before_any_launch(L):
    def dec(q=FAKE, Hq=8, Hkv=2, Nq=1, Nk=1000, d=128, scale=0.088, causal=1, ws=FAKE, wsb=1 << 30):
        return L.attn_decode(q, FAKE, FAKE, FAKE, FAKE, 2, Hq, Hkv, Nq, Nk, d, scale, causal, ws,
                             ctypes.c_size_t(wsb), None)
    assert dec(d=96) == -2
    assert dec(Nq=0) == -1
    assert dec(Nk=0) == -1
    assert dec(Nq=5, Nk=4) == -1                # causal needs Nq <= Nk
    assert dec(Hq=258, Hkv=1) == -1             # group larger than one 128-row tile
    assert dec(Hq=9) == -1
    assert dec(scale=float("nan")) == -1
    assert dec(q=ODD) == -3
    assert dec(ws=ODD) == -3
    assert dec(q=ctypes.c_void_p(0)) == -1
    assert L.attn_decode_workspace_size(2, 8, 2, 5, 4, 128, 1) == 0
    assert L.attn_decode_splits(2, 8, 2, 5, 4, 128, 1) == 0


def test_merge_validates_before_any_launch(L):
    assert L.attn_merge(FAKE, FAKE, FAKE, FAKE, 10, 96, None, None) == -2
    assert L.attn_merge(FAKE, FAKE, FAKE, FAKE, 0, 128, None, None) == -1
    assert L.attn_merge(ctypes.c_void_p(0), FAKE, FAKE, FAKE, 10, 128, None, None) == -1
    assert L.attn_merge(FAKE, FAKE, ODD, FAKE, 10, 128, None, None) == -3
    assert L.attn_merge(FAKE, FAKE, FAKE, FAKE, 10, 128, ODD, None) == -3


def test_accumulate_validates_before_any_launch(L):
    L.attn_accumulate.argtypes = [ctypes.c_void_p, ctypes.c_void_p, ctypes.c_longlong, ctypes.c_void_p]
    assert L.attn_accumulate(ctypes.c_void_p(0), FAKE, 64, None) == -1      # null accumulator
    assert L.attn_accumulate(FAKE, ctypes.c_void_p(0), 64, None) == -1      # null part
    assert L.attn_accumulate(FAKE, FAKE, 0, None) == -1                     # empty
    assert L.attn_accumulate(FAKE, FAKE, 100, None) == -1                   # not a multiple of 8
    assert L.attn_accumulate(ODD, FAKE, 64, None) == -3
    assert L.attn_accumulate(FAKE, ODD, 64, None) == -3


def test_fp8_forward_validates_before_any_launch(L):
    def f8(q=FAKE, d=128, dq=0.01, dk=0.01, dv=0.01, scale=0.088, N=256):
        return L.attn_fwd_fp8(q, FAKE, FAKE, FAKE, FAKE, 1, 2, 1, N, d, scale, dq, dk, dv, 1, None)
    assert f8(d=32) == -2                 # head dims 64 and 128 only
    assert f8(dq=0.0) == -1
    assert f8(dk=-1.0) == -1
    assert f8(dv=float("inf")) == -1
    assert f8(N=0) == -1
    assert f8(q=ODD) == -3
    assert f8(q=ctypes.c_void_p(0)) == -1


def test_checking_build_exports_the_same_boundary(L):
    import __graft_entry__  # noqa: F401  (build() made both libraries)
    C = binding.load(binding.checks_library_path)
    for name in declared_functions():
        assert hasattr(C, name), name
    assert C.attn_checks_enabled() == 1 and L.attn_checks_enabled() == 0
