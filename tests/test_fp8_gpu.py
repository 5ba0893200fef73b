"""FP8 forward (e4m3 Q, K, V with per-tensor descales) vs the fp64 oracle.

The oracle attends over the values the e4m3 codes stand for (code * descale), so
input quantisation is not an error here.  The kernel's only extra rounding is P:
the probabilities are rounded to e4m3 for the P V product (row sums and LSE use
the unrounded values).  Tolerance, per output element, derived from that rounding:
  - e4m3 keeps 3 mantissa bits, so a rounded p is off by at most 2^-4 p (half the
    2^-3 spacing) in the normal range, and by at most 2^-10 below 2^-6 (spacing 2^-9);
  - O_i = sum_j fl(p_j) v_j / l with l >= l_true = sum_j exp(s_j - max s) (the
    kernel's exponent base never exceeds the row max), so each term's error is at
    most max(2^-4 w_j, 2^-10 / l_true) |v_j| with w_j the exact softmax weights;
  - the roundings are independent and of either sign: their sum is held to 6 sigma
    (uniform errors, variance bound^2 / 3), plus half a bf16 ulp of the output and
    2e-3 for fp32 accumulation and the exp2 approximation.
LSE keeps the plain 1e-3 gate.
"""
import numpy as np
import pytest
import torch

from attn_inputs import make_fp8_inputs
from oracle import reference as ref
from tests.parity import check_lse, f64, half_ulp_bf16, _record

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def attn():
    import __graft_entry__
    __graft_entry__.build()
    import io_aware_exact_26_b200 as a
    return a


def fp8_bound(qf, kf, vf, scale, causal, o_ref):
    B, Hq, N, d = qf.shape
    G = Hq // kf.shape[1]
    bound = np.empty_like(o_ref)
    for b in range(B):
        for h in range(Hq):
            s = scale * qf[b, h] @ kf[b, h // G].T
            if causal:
                s = np.where(np.tril(np.ones((N, N), bool)), s, -np.inf)
            e = np.exp(s - s.max(axis=1, keepdims=True))
            l_true = e.sum(axis=1, keepdims=True)
            w = e / l_true
            per = np.maximum(2.0 ** -4 * w, 2.0 ** -10 / l_true)          # [N, N]
            var = (per ** 2) @ (vf[b, h // G] ** 2) / 3                     # [N, d]
            bound[b, h] = 6 * np.sqrt(var)
    return bound + half_ulp_bf16(o_ref) + 2e-3


CASES = [
    # B, Hq, Hkv, N, causal, d
    (1, 2, 2, 256, False, 128),
    (1, 4, 2, 1000, True, 128),
    (2, 2, 2, 1024, False, 128),
    (1, 2, 1, 130, True, 128),
    (1, 1, 1, 17, False, 128),
    (1, 8, 2, 512, True, 128),
    # d = 64: 64-byte e4m3 rows, zero-padded to the 128-byte swizzle row on chip
    (1, 2, 2, 256, False, 64),
    (1, 4, 2, 1000, True, 64),
    (2, 2, 1, 1024, False, 64),
    (1, 1, 1, 17, True, 64),
]


@pytest.mark.parametrize("B,Hq,Hkv,N,causal,d", CASES)
def test_fp8_forward_matches_oracle_within_e4m3_rounding_of_p(attn, B, Hq, Hkv, N, causal, d):
    x = make_fp8_inputs(B, Hq, Hkv, N, d, seed=N + Hq + causal + d)
    ds = {n: x[n + "_descale"] for n in ("q", "k", "v")}
    o, lse = attn.attn_fwd_fp8(x["q"].cuda(), x["k"].cuda(), x["v"].cuda(), q_descale=ds["q"], k_descale=ds["k"],
                               v_descale=ds["v"], causal=causal)
    torch.cuda.synchronize()
    assert attn.attn_get_device_status() == 0
    q8, k8, v8 = (x[n].view(torch.uint8).numpy() for n in ("q", "k", "v"))
    o_ref, lse_ref = ref.ref_fwd_fp8(q8, k8, v8, ds["q"], ds["k"], ds["v"], d ** -0.5, causal)
    tag = f"fp8 B{B} Hq{Hq} Hkv{Hkv} N{N} d{d} {'causal' if causal else 'full'}"
    check_lse(f64(lse), lse_ref, f"{tag} LSE")
    qf, kf, vf = (ref.decode_e4m3(a) * ds[n] for a, n in ((q8, "q"), (k8, "k"), (v8, "v")))
    bound = fp8_bound(qf, kf, vf, d ** -0.5, causal, o_ref)
    err = np.abs(f64(o) - o_ref)
    _record("O (fp8)", f"{tag} O", err, f"e4m3 rounding of P, 6 sigma (max {bound.max():.3g})",
            float(np.sqrt(np.mean(err ** 2)) / np.sqrt(np.mean(o_ref ** 2))), o_ref)
    worst = np.unravel_index(np.argmax(err - bound), err.shape)
    assert np.all(err <= bound), f"{tag}: |err| {err[worst]:.3g} > bound {bound[worst]:.3g} at {worst}"


def test_fp8_forward_is_deterministic_and_rejects_other_head_sizes(attn):
    """Two calls give the same bits at d = 128 and d = 64; d = 32 is refused."""
    x = make_fp8_inputs(1, 2, 2, 300, 128, seed=1)
    args = dict(q_descale=x["q_descale"], k_descale=x["k_descale"], v_descale=x["v_descale"], causal=True)
    q, k, v = (x[n].cuda() for n in ("q", "k", "v"))
    o1, l1 = attn.attn_fwd_fp8(q, k, v, **args)
    o2, l2 = attn.attn_fwd_fp8(q, k, v, **args)
    torch.cuda.synchronize()
    assert torch.equal(o1, o2) and torch.equal(l1, l2)
    y = make_fp8_inputs(1, 2, 1, 300, 64, seed=2)
    q6, k6, v6 = (y[n].cuda() for n in ("q", "k", "v"))
    o3, l3 = attn.attn_fwd_fp8(q6, k6, v6, q_descale=1.0, k_descale=1.0, v_descale=1.0, causal=True)
    o4, l4 = attn.attn_fwd_fp8(q6, k6, v6, q_descale=1.0, k_descale=1.0, v_descale=1.0, causal=True)
    torch.cuda.synchronize()
    assert torch.equal(o3, o4) and torch.equal(l3, l4)
    z = make_fp8_inputs(1, 1, 1, 128, 32, seed=2)
    with pytest.raises(attn.AttnError):
        attn.attn_fwd_fp8(z["q"].cuda(), z["k"].cuda(), z["v"].cuda(), q_descale=1.0, k_descale=1.0, v_descale=1.0)
    with pytest.raises(attn.AttnError):
        attn.attn_fwd_fp8(q, k, v, q_descale=0.0, k_descale=1.0, v_descale=1.0)
