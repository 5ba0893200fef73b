"""Backward parity: dQ, dK, dV from the CUDA path vs the fp64 oracle; determinism."""
import numpy as np
import pytest
import torch

from attn_inputs import make_inputs, to_f64
from oracle import reference as ref
from tests.parity import check_grad, f64

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def attn():
    import __graft_entry__
    __graft_entry__.build()
    import io_aware_exact_26_b200 as a
    return a


def run_fwd_bwd(attn, x, d, causal, scale=None):
    q, k, v, do = (x[n].cuda() for n in ("q", "k", "v", "do"))
    scale = d ** -0.5 if scale is None else scale
    o, lse = attn.attn_fwd(q, k, v, scale=scale, causal=causal)
    dq, dk, dv = attn.attn_bwd(q, k, v, o, lse, do, scale=scale, causal=causal)
    torch.cuda.synchronize()
    assert attn.attn_get_device_status() == 0
    return (q, k, v, do, o, lse), (dq, dk, dv), scale


SMALL = [
    (1, 1, 1, 128, 64, False),
    (1, 1, 1, 128, 128, False),
    (1, 1, 1, 256, 128, True),
    (1, 2, 2, 256, 64, True),
    (1, 2, 2, 512, 128, False),
    (1, 4, 2, 384, 128, True),
    (1, 4, 1, 256, 64, False),
    (1, 1, 1, 17, 128, True),
    (1, 2, 1, 130, 64, True),
    (1, 2, 2, 257, 128, False),
    (2, 2, 2, 1000, 64, True),
    (1, 2, 2, 1024, 128, True),
]


@pytest.mark.parametrize("B,Hq,Hkv,N,d,causal", SMALL)
def test_bwd_matches_oracle(attn, B, Hq, Hkv, N, d, causal):
    x = make_inputs(B, Hq, Hkv, N, d, seed=N * 3 + d + causal)
    _, grads, scale = run_fwd_bwd(attn, x, d, causal)
    g_ref = ref.ref_bwd(to_f64(x["q"]), to_f64(x["k"]), to_f64(x["v"]), to_f64(x["do"]), scale, causal)
    for g, r, name in zip(grads, g_ref, ("dQ", "dK", "dV")):
        check_grad(f64(g), r, f"B{B} Hq{Hq} Hkv{Hkv} N{N} d{d} {'causal' if causal else 'full'} {name}")


def test_bwd_is_bitwise_deterministic(attn):
    x = make_inputs(2, 4, 2, 1024, 128, seed=5)
    ins, g1, scale = run_fwd_bwd(attn, x, 128, True)
    q, k, v, do, o, lse = ins
    for _ in range(2):
        g2 = attn.attn_bwd(q, k, v, o, lse, do, scale=scale, causal=True)
        torch.cuda.synchronize()
        for a, b in zip(g1, g2):
            assert torch.equal(a, b)


@pytest.mark.parametrize("B,H,N,d,causal,window", [(4, 32, 4096, 64, True, None), (2, 8, 2048, 64, False, None),
                                                    (2, 8, 1000, 64, True, None), (1, 16, 4096, 128, True, None),
                                                    (1, 16, 8192, 64, False, (256, 256))])
def test_bwd_is_bitwise_deterministic_across_memory_states(attn, B, H, N, d, causal, window):
    """The same backward, repeated with fresh outputs and workspace after other device
    memory was overwritten with noise, gives the same bits every time (masked tiles make
    the warps' times differ, which is where barrier races would show)."""
    x = make_inputs(B, H, H, N, d, seed=11)
    if window is None:
        ins, g1, scale = run_fwd_bwd(attn, x, d, causal)
        q, k, v, do, o, lse = ins
    else:
        q, k, v, do = (x[n].cuda() for n in ("q", "k", "v", "do"))
        scale = d ** -0.5
        o, lse = attn.attn_fwd_window(q, k, v, window=window)
        g1 = attn.attn_bwd_window(q, k, v, o, lse, do, window=window)
    for rep in range(3):
        noise = torch.randn(64 << 20, device="cuda")           # 256 MB of other data in the allocator's pool
        del noise
        ws = torch.empty(attn.attn_bwd_workspace_size(B, H, H, N, d, bool(causal)), dtype=torch.uint8,
                         device="cuda")
        ws.random_()
        if window is None:
            g2 = attn.attn_bwd(q, k, v, o, lse, do, scale=scale, causal=causal, workspace=ws)
        else:
            g2 = attn.attn_bwd_window(q, k, v, o, lse, do, window=window, workspace=ws)
        torch.cuda.synchronize()
        assert attn.attn_get_device_status() == 0
        for a, b, name in zip(g1, g2, ("dQ", "dK", "dV")):
            assert torch.equal(a, b), (rep, name, (a.float() - b.float()).abs().max().item())


def test_bwd_null_workspace_through_c_abi(attn):
    """workspace = NULL: the library allocates on the stream; same bits as a caller workspace."""
    import ctypes
    B, Hq, Hkv, N, d = 1, 4, 2, 700, 128
    x = make_inputs(B, Hq, Hkv, N, d, seed=77)
    ins, ref_g, scale = run_fwd_bwd(attn, x, d, True)
    q, k, v, do, o, lse = ins
    outs = [torch.full_like(t, float("nan")) for t in (q, k, v)]
    P = lambda t: ctypes.c_void_p(t.data_ptr())
    st = attn.lib().attn_bwd(P(q), P(k), P(v), P(o), P(lse), P(do), P(outs[0]), P(outs[1]), P(outs[2]),
                             B, Hq, Hkv, N, d, scale, 1, ctypes.c_void_p(0), ctypes.c_size_t(0),
                             ctypes.c_void_p(torch.cuda.current_stream().cuda_stream))
    assert st == 0
    torch.cuda.synchronize()
    assert attn.attn_get_device_status() == 0
    for a, b in zip(outs, ref_g):
        assert torch.equal(a, b)


@pytest.mark.parametrize("causal", [True, False])
def test_scale_zero_is_uniform_attention(attn, causal):
    """scale = 0: every visible key gets the same weight (no NaN from masked scores)."""
    B, Hq, Hkv, N, d = 1, 2, 1, 200, 64
    x = make_inputs(B, Hq, Hkv, N, d, seed=91)
    (q, k, v, do, o, lse), grads, _ = run_fwd_bwd(attn, x, d, causal, scale=0.0)
    from tests.parity import check_lse, check_o
    o_ref, lse_ref = ref.ref_fwd(to_f64(x["q"]), to_f64(x["k"]), to_f64(x["v"]), 0.0, causal)
    check_o(f64(o), o_ref)
    check_lse(f64(lse), lse_ref)
    g_ref = ref.ref_bwd(to_f64(x["q"]), to_f64(x["k"]), to_f64(x["v"]), to_f64(x["do"]), 0.0, causal)
    for g, r, name in zip(grads, g_ref, ("dQ", "dK", "dV")):
        check_grad(f64(g), r, name)
