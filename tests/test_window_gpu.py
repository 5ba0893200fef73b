"""Local (sliding-window) attention on the CUDA path vs the fp64 oracle.

Page "attn-efficient", efficient-attention family table, sliding-window row: each
position attends only to the w positions nearest it.  The library's window is
(left, right): query i sees keys i - left .. i + right; a negative side (None
here) has no limit.  Cases cover windows that are not multiples of the 128-key
tile, ragged N, both head sizes, GQA, one-sided and symmetric bands, a band of
one key, and bands wider than N.
"""
import numpy as np
import pytest
import torch

from attn_inputs import make_inputs, to_f64
from oracle import reference as ref
from tests.parity import check_grad, check_lse, check_o, f64

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def attn():
    import __graft_entry__
    __graft_entry__.build()
    import io_aware_exact_26_b200 as a
    return a


CASES = [
    # B, Hq, Hkv, N, d, (left, right)
    (1, 2, 2, 1000, 128, (255, 0)),
    (1, 2, 1, 777, 64, (100, 100)),
    (2, 4, 2, 1024, 128, (0, 0)),
    (1, 2, 2, 513, 128, (None, 130)),
    (1, 4, 4, 384, 64, (1, None)),
    (1, 1, 1, 300, 128, (127, 0)),
    (1, 2, 2, 2048, 128, (511, 0)),
    (1, 2, 2, 256, 64, (300, 300)),
    (1, 3, 1, 1100, 128, (200, 37)),
]


def _ids(c):
    return f"B{c[0]}-Hq{c[1]}-Hkv{c[2]}-N{c[3]}-d{c[4]}-w{c[5][0]}_{c[5][1]}"


@pytest.mark.parametrize("case", CASES, ids=_ids)
def test_window_forward_and_backward_match_oracle(attn, case):
    B, Hq, Hkv, N, d, window = case
    x = make_inputs(B, Hq, Hkv, N, d, seed=N + 13 * d + (window[0] or 0))
    q, k, v, do = (x[n].cuda() for n in ("q", "k", "v", "do"))
    o, lse = attn.attn_fwd_window(q, k, v, window=window)
    dq, dk, dv = attn.attn_bwd_window(q, k, v, o, lse, do, window=window)
    torch.cuda.synchronize()
    assert attn.attn_get_device_status() == 0
    scale = d ** -0.5
    qf, kf, vf, dof = (to_f64(x[n]) for n in ("q", "k", "v", "do"))
    o_ref, lse_ref = ref.ref_fwd(qf, kf, vf, scale, False, window=window)
    check_o(f64(o), o_ref, f"window {window} O")
    check_lse(f64(lse), lse_ref, f"window {window} LSE")
    for g, r, name in zip((dq, dk, dv), ref.ref_bwd(qf, kf, vf, dof, scale, False, window=window),
                          ("dQ", "dK", "dV")):
        check_grad(f64(g), r, f"window {window} {name}")


@pytest.mark.parametrize("d", [64, 128])
def test_unbounded_windows_are_the_plain_entry_points_bit_for_bit(attn, d):
    """(None, 0) is causal and (None, None) is full attention: same kernels, same bits."""
    B, Hq, Hkv, N = 1, 4, 2, 700
    x = make_inputs(B, Hq, Hkv, N, d, seed=5 + d)
    q, k, v, do = (x[n].cuda() for n in ("q", "k", "v", "do"))
    for causal, window in ((True, (None, 0)), (False, (None, None))):
        o1, l1 = attn.attn_fwd(q, k, v, causal=causal)
        o2, l2 = attn.attn_fwd_window(q, k, v, window=window)
        g1 = attn.attn_bwd(q, k, v, o1, l1, do, causal=causal)
        g2 = attn.attn_bwd_window(q, k, v, o2, l2, do, window=window)
        torch.cuda.synchronize()
        assert torch.equal(o1, o2) and torch.equal(l1, l2)
        for a, b in zip(g1, g2):
            assert torch.equal(a, b)


def test_window_of_one_key_returns_v(attn):
    """window (0, 0): every row sees only its own key, so O = V exactly and LSE = scale q.k."""
    B, H, N, d = 1, 2, 300, 128
    x = make_inputs(B, H, H, N, d, seed=3, with_grad=False)
    q, k, v = (x[n].cuda() for n in ("q", "k", "v"))
    o, lse = attn.attn_fwd_window(q, k, v, window=(0, 0))
    torch.cuda.synchronize()
    assert torch.equal(o, v)
    want = d ** -0.5 * np.einsum("bhnd,bhnd->bhn", f64(q), f64(k))
    assert np.abs(f64(lse) - want).max() < 1e-3


def test_window_backward_is_bitwise_deterministic(attn):
    B, Hq, Hkv, N, d = 1, 4, 2, 1500, 128
    x = make_inputs(B, Hq, Hkv, N, d, seed=17)
    q, k, v, do = (x[n].cuda() for n in ("q", "k", "v", "do"))
    o, lse = attn.attn_fwd_window(q, k, v, window=(300, 40))
    g1 = attn.attn_bwd_window(q, k, v, o, lse, do, window=(300, 40))
    g2 = attn.attn_bwd_window(q, k, v, o, lse, do, window=(300, 40))
    torch.cuda.synchronize()
    for a, b in zip(g1, g2):
        assert torch.equal(a, b)
