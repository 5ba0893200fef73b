"""The checking build (libattn_b200_checks.so, compiled with ATTN_CHECKS) on the GPU.

Its kernels test every tile coordinate, head index and global row they compute
against the tensor it addresses and record a failure in the error word instead of
accessing memory outside it -- no trap, no assert.  This runs the small parity
shapes of every entry point through that build: no check may fire, and the results
must still match the fp64 oracle.  The self-test hands the check an index outside
its range (nothing is accessed with it) to show that a failure is reported.
"""
import numpy as np
import pytest
import torch

from attn_inputs import make_fp8_inputs, make_inputs, to_f64
from oracle import reference as ref
from tests.parity import check_grad, check_lse, check_o, f64

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def attn():
    import __graft_entry__
    __graft_entry__.build()
    import io_aware_exact_26_b200 as a
    return a


def test_bounds_selftest_reports_only_in_the_checking_build(attn):
    attn.attn_selftest_bounds()
    assert attn.attn_get_device_status() == 0 and not attn.attn_checks_enabled()
    with attn.use_library(attn.checks_library_path):
        assert attn.attn_checks_enabled()
        attn.attn_selftest_bounds()
        assert attn.attn_get_device_status() == -8          # ATTN_ERR_DEVICE_BOUNDS, word cleared
        assert attn.attn_get_device_status() == 0


SHAPES = [(1, 2, 2, 257, 128, True), (2, 4, 2, 1000, 64, True), (1, 2, 1, 384, 128, False), (1, 1, 1, 17, 64, False)]


@pytest.mark.parametrize("B,Hq,Hkv,N,d,causal", SHAPES)
def test_forward_and_backward_under_index_checks(attn, B, Hq, Hkv, N, d, causal):
    x = make_inputs(B, Hq, Hkv, N, d, seed=N + d)
    q, k, v, do = (x[n].cuda() for n in ("q", "k", "v", "do"))
    with attn.use_library(attn.checks_library_path):
        o, lse = attn.attn_fwd(q, k, v, causal=causal)
        grads = attn.attn_bwd(q, k, v, o, lse, do, causal=causal)
        ow, lw = attn.attn_fwd_window(q, k, v, window=(100, 3))
        gw = attn.attn_bwd_window(q, k, v, ow, lw, do, window=(100, 3))
        torch.cuda.synchronize()
        assert attn.attn_get_device_status() == 0
    qf, kf, vf, dof = (to_f64(x[n]) for n in ("q", "k", "v", "do"))
    o_ref, lse_ref = ref.ref_fwd(qf, kf, vf, d ** -0.5, causal)
    check_o(f64(o), o_ref, "checks O")
    check_lse(f64(lse), lse_ref, "checks LSE")
    for g, r, name in zip(grads, ref.ref_bwd(qf, kf, vf, dof, d ** -0.5, causal), ("dQ", "dK", "dV")):
        check_grad(f64(g), r, f"checks {name}")
    ow_ref, _ = ref.ref_fwd(qf, kf, vf, d ** -0.5, False, window=(100, 3))
    check_o(f64(ow), ow_ref, "checks window O")
    for g, r, name in zip(gw, ref.ref_bwd(qf, kf, vf, dof, d ** -0.5, False, window=(100, 3)), ("dQ", "dK", "dV")):
        check_grad(f64(g), r, f"checks window {name}")


def test_decode_fp8_and_merge_under_index_checks(attn):
    g = torch.Generator().manual_seed(8)
    q = torch.randn(2, 8, 5, 128, generator=g).to(torch.bfloat16)
    k = torch.randn(2, 2, 3000, 128, generator=g).to(torch.bfloat16)
    v = torch.randn(2, 2, 3000, 128, generator=g).to(torch.bfloat16)
    x8 = make_fp8_inputs(1, 2, 1, 300, 128, seed=4)
    with attn.use_library(attn.checks_library_path):
        o, lse = attn.attn_decode(q.cuda(), k.cuda(), v.cuda(), causal=True)
        o8, l8 = attn.attn_fwd_fp8(x8["q"].cuda(), x8["k"].cuda(), x8["v"].cuda(), q_descale=x8["q_descale"],
                                   k_descale=x8["k_descale"], v_descale=x8["v_descale"], causal=True)
        acc = torch.zeros((2, 8, 5, 128), device="cuda")
        lacc = torch.full((2, 8, 5), float("-inf"), device="cuda")
        attn.attn_merge(acc, lacc, o, lse)
        torch.cuda.synchronize()
        assert attn.attn_get_device_status() == 0
    o_ref, lse_ref = ref.ref_decode(to_f64(q), to_f64(k), to_f64(v), 128 ** -0.5, True)
    check_o(f64(o), o_ref, "checks decode O")
    check_lse(f64(lse), lse_ref, "checks decode LSE")
    assert np.abs(f64(acc) - f64(o)).max() < 1e-6
    q8, k8, v8 = (x8[n].view(torch.uint8).numpy() for n in ("q", "k", "v"))
    _, l8_ref = ref.ref_fwd_fp8(q8, k8, v8, x8["q_descale"], x8["k_descale"], x8["v_descale"], 128 ** -0.5, True)
    check_lse(f64(l8), l8_ref, "checks fp8 LSE")
