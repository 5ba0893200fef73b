"""Invariants of exact attention checked on the CUDA path directly (no oracle call).

Inputs are chosen so that the statement is exact in bf16 where that matters:
  * constant V rows: every output row equals that row (softmax rows sum to one);
  * Q = 0: uniform attention, O = column mean of V (causal: prefix mean),
    LSE = ln(number of visible keys);
  * shift invariance (page "attn-efficient", online-softmax section: the same
    number subtracted from a whole score row leaves softmax unchanged): K + u
    adds q_i . u to every score of row i, so O is unchanged and LSE moves by
    scale * q_i . u; Q, K, u are on a grid where K + u is exact in bf16;
  * V = I (N = d): O equals the probability rows, which sum to one;
  * a dominant score: q_i = t * e_j with orthonormal keys selects V_j;
  * gradients: sum_j dK_j = 0 and sum_j dV_j = sum_i dO_i (over the group).
"""
import numpy as np
import pytest
import torch

from tests.parity import check_o, f64, half_ulp_bf16

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def attn():
    import __graft_entry__
    __graft_entry__.build()
    import io_aware_exact_26_b200 as a
    return a


def bf(x):
    return torch.as_tensor(x, dtype=torch.float32).to(torch.bfloat16).cuda().contiguous()


@pytest.mark.parametrize("d,causal", [(64, False), (128, True), (128, False)])
def test_constant_v_rows_return_v(attn, d, causal):
    g = torch.Generator().manual_seed(1)
    B, H, N = 1, 2, 300
    q = bf(torch.randn(B, H, N, d, generator=g) * 2)
    k = bf(torch.randn(B, H, N, d, generator=g) * 2)
    row = torch.randn(d, generator=g)
    v = bf(row.expand(B, H, N, d))
    o, _ = attn.attn_fwd(q, k, v, causal=causal)
    torch.cuda.synchronize()
    want = np.broadcast_to(f64(v[0, 0, 0]), (B, H, N, d))
    check_o(f64(o), want, "O for constant V")


@pytest.mark.parametrize("d,causal", [(64, True), (128, False)])
def test_zero_q_gives_mean_of_v(attn, d, causal):
    g = torch.Generator().manual_seed(2)
    B, H, N = 2, 1, 257
    q = bf(torch.zeros(B, H, N, d))
    k = bf(torch.randn(B, H, N, d, generator=g))
    v = bf(torch.randn(B, H, N, d, generator=g))
    o, lse = attn.attn_fwd(q, k, v, causal=causal)
    torch.cuda.synchronize()
    vf = f64(v)
    if causal:
        cnt = np.arange(1, N + 1)
        want = np.cumsum(vf, axis=2) / cnt[None, None, :, None]
        lse_want = np.broadcast_to(np.log(cnt), (B, H, N))
    else:
        want = np.broadcast_to(vf.mean(axis=2, keepdims=True), vf.shape)
        lse_want = np.full((B, H, N), np.log(N))
    check_o(f64(o), want, "O for Q = 0")
    assert np.abs(f64(lse) - lse_want).max() < 1e-4


@pytest.mark.parametrize("causal", [False, True])
def test_shift_invariance(attn, causal):
    g = torch.Generator().manual_seed(3)
    B, H, N, d = 1, 2, 384, 128
    # values on a 1/8 grid with small magnitude: K + u stays exact in bf16
    q = bf(torch.randint(-8, 9, (B, H, N, d), generator=g) / 8)
    k = bf(torch.randint(-8, 9, (B, H, N, d), generator=g) / 8)
    u = torch.randint(-8, 9, (d,), generator=g) / 8
    k2 = bf(k.float().cpu() + u)
    assert torch.equal(k2.float(), k.float() + u.cuda())
    v = bf(torch.randn(B, H, N, d, generator=g))
    o1, l1 = attn.attn_fwd(q, k, v, causal=causal)
    o2, l2 = attn.attn_fwd(q, k2, v, causal=causal)
    torch.cuda.synchronize()
    check_o(f64(o2), f64(o1), "O after shifting K")
    shift = d ** -0.5 * (f64(q) @ u.double().numpy())
    assert np.abs(f64(l2) - f64(l1) - shift).max() < 2e-3


@pytest.mark.parametrize("d", [64, 128])
def test_identity_v_exposes_probability_rows(attn, d):
    g = torch.Generator().manual_seed(4)
    N = d
    q = bf(torch.randn(1, 1, N, d, generator=g) * 3)
    k = bf(torch.randn(1, 1, N, d, generator=g) * 3)
    v = bf(torch.eye(N).reshape(1, 1, N, d))
    o, lse = attn.attn_fwd(q, k, v, causal=False)
    torch.cuda.synchronize()
    p = f64(o)[0, 0]
    assert p.min() >= 0
    np.testing.assert_allclose(p.sum(axis=1), 1.0, atol=2e-2)
    # against the softmax of the bf16 scores computed in fp64
    s = d ** -0.5 * f64(q)[0, 0] @ f64(k)[0, 0].T
    want = np.exp(s - s.max(axis=1, keepdims=True))
    want /= want.sum(axis=1, keepdims=True)
    assert np.abs(p - want).max() <= 1e-2 + half_ulp_bf16(want).max()


def test_dominant_score_selects_its_v_row(attn):
    d = N = 128
    j_of = [(i * 37 + 5) % N for i in range(N)]
    q = torch.zeros(1, 1, N, d)
    for i, j in enumerate(j_of):
        q[0, 0, i, j] = 64.0
    k = torch.eye(N).reshape(1, 1, N, d)
    g = torch.Generator().manual_seed(5)
    v = torch.randn(1, 1, N, d, generator=g)
    o, _ = attn.attn_fwd(bf(q), bf(k), bf(v), scale=1.0, causal=False)
    torch.cuda.synchronize()
    want = f64(bf(v))[0, 0][j_of]
    check_o(f64(o)[0, 0], want, "O for a dominant score")


@pytest.mark.parametrize("causal", [False, True])
def test_gradient_sum_identities(attn, causal):
    g = torch.Generator().manual_seed(6)
    B, Hq, Hkv, N, d = 1, 4, 2, 512, 128
    q, k, v, do = (bf(torch.randn(B, h, N, d, generator=g)) for h in (Hq, Hkv, Hkv, Hq))
    o, lse = attn.attn_fwd(q, k, v, causal=causal)
    dq, dk, dv = attn.attn_bwd(q, k, v, o, lse, do, causal=causal)
    torch.cuda.synchronize()
    dkf, dvf = f64(dk), f64(dv)
    G = Hq // Hkv
    dv_want = f64(do).reshape(B, Hkv, G, N, d).sum(axis=(2, 3))
    # sums of N bf16-rounded rows: allow the rounding of each row
    tol_v = 2e-2 * max(1.0, np.abs(dv_want).max())
    assert np.abs(dvf.sum(axis=2) - dv_want).max() <= tol_v
    # sum_j dK_j = scale * sum_i (sum_j dS_ij) q_i = 0, since each row of dS sums to zero.
    # What the kernels may leave: bf16 rounding of every dK row (half an ulp each) and,
    # inside, bf16 rounding of every dS element and of O (which feeds D_i).  Those
    # errors are independent and of either sign, so their sum is bounded at 6 sigma,
    # with each rounding error uniform in +-half ulp (variance hulp^2 / 3).
    scale = d ** -0.5
    qf, kf, vf, dof, of = f64(q), f64(k), f64(v), f64(do), f64(o)
    for b in range(B):
        for g in range(Hkv):
            var = (half_ulp_bf16(dkf[b, g]) ** 2).sum(axis=0) / 3          # [d]
            for h in range(g * G, (g + 1) * G):
                s = scale * qf[b, h] @ kf[b, g].T
                if causal:
                    s = np.where(np.tril(np.ones((N, N), bool)), s, -np.inf)
                p = np.exp(s - s.max(axis=1, keepdims=True))
                p /= p.sum(axis=1, keepdims=True)
                dp = dof[b, h] @ vf[b, g].T
                dd = (dof[b, h] * of[b, h]).sum(axis=1)
                ds = p * (dp - dd[:, None])
                e_row = (half_ulp_bf16(ds) ** 2).sum(axis=1) / 3 \
                    + ((dof[b, h] * half_ulp_bf16(of[b, h])) ** 2).sum(axis=1) / 3
                var += scale ** 2 * (e_row[:, None] * qf[b, h] ** 2).sum(axis=0)
            bound = 6 * np.sqrt(var)
            got = np.abs(dkf[b, g].sum(axis=0))
            assert np.all(got <= bound), f"sum_j dK_j: {got.max():.3g} vs bound {bound[np.argmax(got)]:.3g}"
