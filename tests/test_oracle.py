"""Pins for the fp64 oracle (CPU only).

Each check ties the oracle to something other than itself, chosen so that a
dropped term, a wrong sign or index, or a transposed operand fails at least one:
  * an independent brute-force implementation in C (long double, no BLAS);
  * torch's fp64 CPU scaled-dot-product attention and its autograd (a library
    routine the whole operation reduces to);
  * central finite differences of sum(O * dO) for the backward;
  * closed forms: constant V, Q = 0 (column / prefix means), a dominant score,
    N = 1, V = I (O equals the probability rows), orthonormal keys (textbook softmax);
  * shift invariance (page "attn-efficient", online-softmax section: subtracting
    one constant from a whole score row leaves softmax unchanged);
  * blockwise online softmax equals full softmax over random partitions
    (page "attn-efficient": blockwise and full results are identical; page
    "attention 的显存线性化" §二: mathematically the same result);
  * gradient invariants that follow from softmax rows summing to one.
"""
import numpy as np
import pytest
import torch

from attn_inputs import make_inputs, to_f64
from oracle import build as obuild
from oracle import reference as ref

RNG = np.random.default_rng(12345)


def rand(*shape, scale=1.0):
    return RNG.standard_normal(shape) * scale


TINY = [
    # B, Hq, Hkv, N, d, causal
    (1, 1, 1, 1, 3, False),
    (1, 1, 1, 5, 4, True),
    (2, 2, 2, 7, 3, False),
    (1, 4, 2, 9, 5, True),
    (1, 4, 1, 16, 8, False),
    (2, 3, 3, 6, 2, True),
]


@pytest.mark.parametrize("B,Hq,Hkv,N,d,causal", TINY)
def test_fwd_matches_c_brute_force(B, Hq, Hkv, N, d, causal):
    q, k, v = rand(B, Hq, N, d), rand(B, Hkv, N, d), rand(B, Hkv, N, d)
    scale = 1 / np.sqrt(d)
    o, lse = ref.ref_fwd(q, k, v, scale, causal)
    ob, lseb = obuild.brute_fwd(q, k, v, scale, causal)
    np.testing.assert_allclose(o, ob, rtol=1e-12, atol=1e-13)
    np.testing.assert_allclose(lse, lseb, rtol=1e-12, atol=1e-13)


@pytest.mark.parametrize("B,Hq,Hkv,N,d,causal", TINY)
def test_bwd_matches_c_brute_force(B, Hq, Hkv, N, d, causal):
    q, k, v, do = rand(B, Hq, N, d), rand(B, Hkv, N, d), rand(B, Hkv, N, d), rand(B, Hq, N, d)
    scale = 0.7
    got = ref.ref_bwd(q, k, v, do, scale, causal)
    exp = obuild.brute_bwd(q, k, v, do, scale, causal)
    for g, e in zip(got, exp):
        np.testing.assert_allclose(g, e, rtol=1e-11, atol=1e-12)


def _torch_sdpa(q, k, v, scale, causal):
    G = q.shape[1] // k.shape[1]
    tq, tk, tv = (torch.tensor(x, dtype=torch.float64, requires_grad=True) for x in (q, k, v))
    o = torch.nn.functional.scaled_dot_product_attention(
        tq, tk.repeat_interleave(G, dim=1), tv.repeat_interleave(G, dim=1),
        is_causal=causal, scale=scale)
    return tq, tk, tv, o


@pytest.mark.parametrize("B,Hq,Hkv,N,d,causal", TINY + [(1, 2, 1, 64, 16, True), (2, 2, 2, 33, 8, False)])
def test_fwd_bwd_match_torch_fp64_sdpa(B, Hq, Hkv, N, d, causal):
    q, k, v, do = rand(B, Hq, N, d), rand(B, Hkv, N, d), rand(B, Hkv, N, d), rand(B, Hq, N, d)
    scale = 1 / np.sqrt(d)
    tq, tk, tv, to = _torch_sdpa(q, k, v, scale, causal)
    o, lse = ref.ref_fwd(q, k, v, scale, causal)
    np.testing.assert_allclose(o, to.detach().numpy(), rtol=1e-10, atol=1e-12)
    (to * torch.tensor(do)).sum().backward()
    dq, dk, dv = ref.ref_bwd(q, k, v, do, scale, causal)
    np.testing.assert_allclose(dq, tq.grad.numpy(), rtol=1e-9, atol=1e-11)
    np.testing.assert_allclose(dk, tk.grad.numpy(), rtol=1e-9, atol=1e-11)
    np.testing.assert_allclose(dv, tv.grad.numpy(), rtol=1e-9, atol=1e-11)
    # LSE against its definition through torch's logsumexp of the masked scores
    s = scale * torch.einsum("bhnd,bhmd->bhnm", torch.tensor(q),
                             torch.tensor(k).repeat_interleave(Hq // Hkv, dim=1))
    if causal:
        s = s.masked_fill(torch.triu(torch.ones(N, N, dtype=torch.bool), 1), float("-inf"))
    np.testing.assert_allclose(lse, torch.logsumexp(s, dim=-1).numpy(), rtol=1e-12, atol=1e-12)


def _fd_grads(fwd, q, k, v, do, scale, causal, h=1e-6):
    """Central differences of L = sum(O * dO) with respect to every entry of q, k, v."""
    def loss(qq, kk, vv):
        return float((fwd(qq, kk, vv, scale, causal)[0] * do).sum())
    grads = []
    for which in range(3):
        args = [q.copy(), k.copy(), v.copy()]
        g = np.zeros_like(args[which])
        it = np.nditer(g, flags=["multi_index"])
        for _ in it:
            idx = it.multi_index
            plus = [a.copy() for a in args]
            minus = [a.copy() for a in args]
            plus[which][idx] += h
            minus[which][idx] -= h
            g[idx] = (loss(*plus) - loss(*minus)) / (2 * h)
        grads.append(g)
    return grads


@pytest.mark.parametrize("B,Hq,Hkv,N,d,causal", [(1, 1, 1, 4, 3, False), (1, 2, 1, 6, 2, True),
                                                 (1, 2, 2, 5, 4, True), (1, 4, 2, 3, 2, False)])
def test_bwd_matches_finite_differences(B, Hq, Hkv, N, d, causal):
    q, k, v, do = rand(B, Hq, N, d), rand(B, Hkv, N, d), rand(B, Hkv, N, d), rand(B, Hq, N, d)
    scale = 0.6
    fd = _fd_grads(ref.ref_fwd, q, k, v, do, scale, causal)
    got = ref.ref_bwd(q, k, v, do, scale, causal)
    for g, e in zip(got, fd):
        np.testing.assert_allclose(g, e, rtol=1e-7, atol=1e-8)


def test_finite_differences_catch_a_planted_sign_error(monkeypatch):
    """A mistake planted in the oracle (dS = P (dP + D)) must fail the FD pin."""
    q, k, v, do = rand(1, 1, 4, 3), rand(1, 1, 4, 3), rand(1, 1, 4, 3), rand(1, 1, 4, 3)
    fd = _fd_grads(ref.ref_fwd, q, k, v, do, 0.6, False)

    def bad_grad_head(qh, kh, vh, doh, scale, causal, block=1024, window=None):
        p, _, _ = ref._softmax_rows(ref._scores(qh, kh, scale, causal, np.arange(qh.shape[0])))
        o = p @ vh
        dd = (doh * o).sum(axis=1)
        ds = p * (doh @ vh.T + dd[:, None])
        return scale * ds @ kh, scale * ds.T @ qh, p.T @ doh

    monkeypatch.setattr(ref, "grad_head", bad_grad_head)
    bad = ref.ref_bwd(q, k, v, do, 0.6, False)
    assert not np.allclose(bad[0], fd[0], rtol=1e-5, atol=1e-6)
    np.testing.assert_allclose(bad[2], fd[2], rtol=1e-7, atol=1e-8)  # dV does not involve dS


@pytest.mark.parametrize("causal", [False, True])
@pytest.mark.parametrize("parts", [[1], [4], [1, 2, 3], [5, 1, 1, 9], "ones", "random"])
def test_blockwise_online_softmax_equals_full(parts, causal):
    n, d = 23, 6
    qh, kh, vh = rand(n, d, scale=2.0), rand(n, d, scale=2.0), rand(n, d)
    if parts == "ones":
        bounds = list(range(n + 1))
    elif parts == "random":
        cuts = sorted(RNG.choice(np.arange(1, n), size=7, replace=False).tolist())
        bounds = [0] + cuts + [n]
    else:
        bounds, x = [0], 0
        while x < n:
            for p in parts:
                x = min(n, x + p)
                bounds.append(x)
                if x == n:
                    break
    o_full, lse_full = ref.attend_head(qh, kh, vh, 0.4, causal)
    o_on, lse_on = ref.online_fwd_head(qh, kh, vh, 0.4, causal, bounds)
    np.testing.assert_allclose(o_on, o_full, rtol=1e-13, atol=1e-14)
    np.testing.assert_allclose(lse_on, lse_full, rtol=1e-13, atol=1e-14)


def test_online_recurrence_tracks_running_max_and_sum():
    """After each block, m and l equal the max and the shifted exp-sum of the prefix."""
    n, d = 12, 4
    qh, kh, vh = rand(n, d), rand(n, d), rand(n, d)
    for cut in range(1, n + 1):
        o, lse = ref.online_fwd_head(qh, kh[:cut], vh[:cut], 1.0, False, sorted({0, cut // 2, cut}))
        s = qh @ kh[:cut].T
        np.testing.assert_allclose(lse, np.log(np.exp(s).sum(axis=1)), rtol=1e-13)
        p = np.exp(s) / np.exp(s).sum(axis=1, keepdims=True)
        np.testing.assert_allclose(o, p @ vh[:cut], rtol=1e-12, atol=1e-13)


@pytest.mark.parametrize("causal", [False, True])
def test_constant_v_rows_return_v(causal):
    B, H, N, d = 1, 2, 37, 8
    q, k = rand(B, H, N, d, scale=3.0), rand(B, H, N, d, scale=3.0)
    row = rand(d)
    v = np.broadcast_to(row, (B, H, N, d)).copy()
    o, _ = ref.ref_fwd(q, k, v, 0.3, causal)
    np.testing.assert_allclose(o, v, rtol=1e-13, atol=1e-14)


@pytest.mark.parametrize("causal", [False, True])
def test_zero_q_gives_mean_of_v(causal):
    B, H, N, d = 2, 1, 19, 5
    q = np.zeros((B, H, N, d))
    k, v = rand(B, H, N, d), rand(B, H, N, d)
    o, lse = ref.ref_fwd(q, k, v, 0.5, causal)
    if causal:
        cnt = np.arange(1, N + 1)
        expect = np.cumsum(v, axis=2) / cnt[None, None, :, None]
        lse_exp = np.log(cnt)[None, None, :]
    else:
        expect = np.broadcast_to(v.mean(axis=2, keepdims=True), v.shape)
        lse_exp = np.full((B, H, N), np.log(N))
    np.testing.assert_allclose(o, expect, rtol=1e-13, atol=1e-14)
    np.testing.assert_allclose(lse, np.broadcast_to(lse_exp, lse.shape), rtol=1e-13)


def test_dominant_score_selects_its_v_row_closed_form():
    """Orthonormal keys: S_i = scale * T on key j, 0 elsewhere; P_ij = e^a / (e^a + N - 1)."""
    N, d = 6, 8
    k = np.eye(d)[:N][None, None]
    v = rand(1, 1, N, d)
    T = 60.0
    scale = 0.5
    q = np.zeros((1, 1, N, d))
    for i in range(N):
        q[0, 0, i, (i + 2) % N] = T
    o, lse = ref.ref_fwd(q, k, v, scale, False)
    a = scale * T
    p_hit = np.exp(a) / (np.exp(a) + N - 1)
    p_miss = 1.0 / (np.exp(a) + N - 1)
    for i in range(N):
        j = (i + 2) % N
        expect = p_hit * v[0, 0, j] + p_miss * (v[0, 0].sum(axis=0) - v[0, 0, j])
        np.testing.assert_allclose(o[0, 0, i], expect, rtol=1e-12, atol=1e-14)
        np.testing.assert_allclose(o[0, 0, i], v[0, 0, j], atol=1e-11)
        np.testing.assert_allclose(lse[0, 0, i], a + np.log1p((N - 1) * np.exp(-a)), rtol=1e-14)


def test_single_key_returns_v0_and_lse_is_the_score():
    d = 7
    q, k, v = rand(3, 2, 1, d), rand(3, 2, 1, d), rand(3, 2, 1, d)
    for causal in (False, True):
        o, lse = ref.ref_fwd(q, k, v, 0.25, causal)
        np.testing.assert_allclose(o, v, rtol=1e-14)
        np.testing.assert_allclose(lse, 0.25 * (q * k).sum(-1), rtol=1e-13)


def test_identity_v_and_orthonormal_keys_expose_textbook_softmax():
    """With K = V = I (N = d), O_i = softmax(scale * q_i): compare with scipy's softmax."""
    from scipy.special import softmax
    N = d = 16
    q = rand(1, 1, N, d, scale=2.0)
    eye = np.eye(N)[None, None]
    o, _ = ref.ref_fwd(q, eye, eye, 0.7, False)
    np.testing.assert_allclose(o[0, 0], softmax(0.7 * q[0, 0], axis=1), rtol=1e-13, atol=1e-15)
    oc, _ = ref.ref_fwd(q, eye, eye, 0.7, True)
    for i in range(N):
        expect = np.zeros(N)
        expect[:i + 1] = softmax(0.7 * q[0, 0, i, :i + 1])
        np.testing.assert_allclose(oc[0, 0, i], expect, rtol=1e-13, atol=1e-15)


@pytest.mark.parametrize("causal", [False, True])
def test_shift_invariance(causal):
    """K + u (one vector for all keys) adds q_i . u to every score of row i: O unchanged."""
    B, H, N, d = 1, 2, 21, 6
    q, k, v = rand(B, H, N, d), rand(B, H, N, d), rand(B, H, N, d)
    u = rand(d, scale=4.0)
    o1, l1 = ref.ref_fwd(q, k, v, 0.5, causal)
    o2, l2 = ref.ref_fwd(q, k + u, v, 0.5, causal)
    np.testing.assert_allclose(o2, o1, rtol=1e-11, atol=1e-12)
    np.testing.assert_allclose(l2, l1 + 0.5 * (q @ u), rtol=1e-11, atol=1e-12)


@pytest.mark.parametrize("causal", [False, True])
def test_gradient_invariants(causal):
    B, Hq, Hkv, N, d = 2, 4, 2, 17, 5
    q, k, v, do = rand(B, Hq, N, d), rand(B, Hkv, N, d), rand(B, Hkv, N, d), rand(B, Hq, N, d)
    dq, dk, dv = ref.ref_bwd(q, k, v, do, 0.4, causal)
    G = Hq // Hkv
    # sum_j dK_j = scale * sum_i (sum_j dS_ij) q_i = 0, per kv head
    np.testing.assert_allclose(dk.sum(axis=2), 0.0, atol=1e-12)
    # sum_j dV_j = sum_i (sum_j P_ij) dO_i = sum of dO over the group's q heads
    expect = do.reshape(B, Hkv, G, N, d).sum(axis=(2, 3))
    np.testing.assert_allclose(dv.sum(axis=2), expect, rtol=1e-12, atol=1e-12)


def test_row_blocks_equal_whole_matrix():
    q, k, v, do = rand(1, 2, 50, 4), rand(1, 1, 50, 4), rand(1, 1, 50, 4), rand(1, 2, 50, 4)
    o1, l1 = ref.ref_fwd(q, k, v, 0.5, True, block=7)
    o2, l2 = ref.ref_fwd(q, k, v, 0.5, True, block=4096)
    np.testing.assert_allclose(o1, o2, rtol=1e-14, atol=1e-15)
    np.testing.assert_allclose(l1, l2, rtol=1e-14)
    g1 = ref.ref_bwd(q, k, v, do, 0.5, True, block=7)
    g2 = ref.ref_bwd(q, k, v, do, 0.5, True, block=4096)
    for a, b in zip(g1, g2):
        np.testing.assert_allclose(a, b, rtol=1e-12, atol=1e-13)


def test_attend_head_on_sampled_rows_matches_full():
    qh, kh, vh = rand(40, 8), rand(40, 8), rand(40, 8)
    rows = np.array([0, 3, 17, 39])
    o, lse = ref.attend_head(qh, kh, vh, 0.3, True)
    os_, ls = ref.attend_head(qh, kh, vh, 0.3, True, rows=rows)
    np.testing.assert_allclose(os_, o[rows], rtol=1e-14)
    np.testing.assert_allclose(ls, lse[rows], rtol=1e-14)


def test_seeded_inputs_are_bf16_and_reproducible():
    a = make_inputs(1, 4, 2, 64, 16, seed=5, qk_std=3.0, boost_frac=0.05, boost=8.0)
    b = make_inputs(1, 4, 2, 64, 16, seed=5, qk_std=3.0, boost_frac=0.05, boost=8.0)
    for key in a:
        assert a[key].dtype == torch.bfloat16
        assert torch.equal(a[key], b[key])
    # boosted rows are exact multiples of 8 of an unboosted draw
    c = make_inputs(1, 4, 2, 64, 16, seed=5, qk_std=3.0)
    ratio = to_f64(a["k"]) / np.where(to_f64(c["k"]) == 0, 1, to_f64(c["k"]))
    per_row = np.isclose(ratio, 8.0).all(axis=-1)
    assert per_row.sum(axis=-1).tolist() == [[3, 3]]


@pytest.mark.parametrize("causal", [False, True])
def test_sampled_gradient_rows_match_full_backward(causal):
    B, Hq, Hkv, N, d = 1, 4, 2, 45, 6
    q, k, v, do = rand(B, Hq, N, d), rand(B, Hkv, N, d), rand(B, Hkv, N, d), rand(B, Hq, N, d)
    dq, dk, dv = ref.ref_bwd(q, k, v, do, 0.45, causal)
    rows = np.array([0, 7, 44])
    np.testing.assert_allclose(ref.grad_q_rows(q[0, 3], k[0, 1], v[0, 1], do[0, 3], 0.45, causal, rows),
                               dq[0, 3, rows], rtol=1e-12, atol=1e-13)
    gk, gv = ref.grad_kv_rows([q[0, 2], q[0, 3]], k[0, 1], v[0, 1], [do[0, 2], do[0, 3]], 0.45, causal,
                              rows, block=16)
    np.testing.assert_allclose(gk, dk[0, 1, rows], rtol=1e-11, atol=1e-12)
    np.testing.assert_allclose(gv, dv[0, 1, rows], rtol=1e-11, atol=1e-12)


# ---------------------------------------------------------------- local (sliding-window) attention
# Page "attn-efficient", efficient-attention family table, sliding-window row: each
# position attends only to the w positions nearest it.  window = (left, right):
# query i sees keys j with i - left <= j <= i + right (None = no limit).
WINDOWS = [(2, 0), (0, 3), (3, 2), (None, 1), (1, None), (5, 5)]


@pytest.mark.parametrize("window", WINDOWS)
@pytest.mark.parametrize("causal", [False, True])
def test_window_fwd_bwd_match_c_brute_force(window, causal):
    B, Hq, Hkv, N, d = 1, 4, 2, 11, 3
    q, k, v, do = rand(B, Hq, N, d), rand(B, Hkv, N, d), rand(B, Hkv, N, d), rand(B, Hq, N, d)
    o, lse = ref.ref_fwd(q, k, v, 0.8, causal, window=window)
    ob, lseb = obuild.brute_fwd(q, k, v, 0.8, causal, window=window)
    np.testing.assert_allclose(o, ob, rtol=1e-12, atol=1e-13)
    np.testing.assert_allclose(lse, lseb, rtol=1e-12, atol=1e-13)
    for g, e in zip(ref.ref_bwd(q, k, v, do, 0.8, causal, window=window),
                    obuild.brute_bwd(q, k, v, do, 0.8, causal, window=window)):
        np.testing.assert_allclose(g, e, rtol=1e-11, atol=1e-12)


@pytest.mark.parametrize("window", WINDOWS)
def test_window_matches_torch_sdpa_with_a_band_mask(window):
    """torch's fp64 SDPA with an explicit boolean band mask (a library routine), and autograd."""
    B, Hq, Hkv, N, d = 2, 2, 1, 13, 4
    q, k, v, do = rand(B, Hq, N, d), rand(B, Hkv, N, d), rand(B, Hkv, N, d), rand(B, Hq, N, d)
    i = torch.arange(N)[:, None]
    j = torch.arange(N)[None, :]
    band = torch.ones(N, N, dtype=torch.bool)
    if window[0] is not None:
        band &= j >= i - window[0]
    if window[1] is not None:
        band &= j <= i + window[1]
    tq, tk, tv = (torch.tensor(x, dtype=torch.float64, requires_grad=True) for x in (q, k, v))
    to = torch.nn.functional.scaled_dot_product_attention(
        tq, tk.repeat_interleave(Hq // Hkv, dim=1), tv.repeat_interleave(Hq // Hkv, dim=1), attn_mask=band, scale=0.5)
    o, lse = ref.ref_fwd(q, k, v, 0.5, False, window=window)
    np.testing.assert_allclose(o, to.detach().numpy(), rtol=1e-10, atol=1e-12)
    (to * torch.tensor(do)).sum().backward()
    for g, e in zip(ref.ref_bwd(q, k, v, do, 0.5, False, window=window), (tq.grad, tk.grad, tv.grad)):
        np.testing.assert_allclose(g, e.numpy(), rtol=1e-9, atol=1e-11)


def test_window_special_cases():
    B, H, N, d = 1, 2, 17, 5
    q, k, v = rand(B, H, N, d, scale=2.0), rand(B, H, N, d, scale=2.0), rand(B, H, N, d)
    full = ref.ref_fwd(q, k, v, 0.7, False)
    causal = ref.ref_fwd(q, k, v, 0.7, True)
    for a, b in zip(ref.ref_fwd(q, k, v, 0.7, False, window=(N, N)), full):        # wider than N: no mask
        np.testing.assert_array_equal(a, b)
    for a, b in zip(ref.ref_fwd(q, k, v, 0.7, False, window=(None, 0)), causal):   # (None, 0) is causal
        np.testing.assert_array_equal(a, b)
    o, lse = ref.ref_fwd(q, k, v, 0.7, False, window=(0, 0))                      # only itself: O_i = V_i
    np.testing.assert_allclose(o, v, rtol=1e-14, atol=1e-15)
    np.testing.assert_allclose(lse, 0.7 * np.einsum("bhnd,bhnd->bhn", q, k), rtol=1e-13, atol=1e-14)
    # left window 1, causal: row i averages V_{i-1}, V_i with weights from the two scores
    o, _ = ref.ref_fwd(q, k, v, 0.7, True, window=(1, None))
    s1 = 0.7 * np.einsum("bhnd,bhnd->bhn", q[:, :, 1:], k[:, :, :-1])
    s0 = 0.7 * np.einsum("bhnd,bhnd->bhn", q[:, :, 1:], k[:, :, 1:])
    w1 = 1 / (1 + np.exp(s0 - s1))
    want = w1[..., None] * v[:, :, :-1] + (1 - w1[..., None]) * v[:, :, 1:]
    np.testing.assert_allclose(o[:, :, 1:], want, rtol=1e-12, atol=1e-13)
    np.testing.assert_allclose(o[:, :, 0], v[:, :, 0], rtol=1e-14)


@pytest.mark.parametrize("window", [(3, 0), (2, 4)])
def test_window_bwd_matches_finite_differences(window):
    q, k, v, do = rand(1, 2, 7, 2), rand(1, 1, 7, 2), rand(1, 1, 7, 2), rand(1, 2, 7, 2)

    def fwd(qq, kk, vv, scale, causal):
        return ref.ref_fwd(qq, kk, vv, scale, causal, window=window)
    fd = _fd_grads(fwd, q, k, v, do, 0.6, False)
    for g, e in zip(ref.ref_bwd(q, k, v, do, 0.6, False, window=window), fd):
        np.testing.assert_allclose(g, e, rtol=1e-7, atol=1e-8)


@pytest.mark.parametrize("window", [(4, 0), (2, 3)])
def test_window_blockwise_online_softmax_equals_full(window):
    n, d = 19, 4
    qh, kh, vh = rand(n, d, scale=2.0), rand(n, d, scale=2.0), rand(n, d)
    o_full, lse_full = ref.attend_head(qh, kh, vh, 0.4, False, window=window)
    o_on, lse_on = ref.online_fwd_head(qh, kh, vh, 0.4, False, [0, 3, 4, 10, 12, n], window=window)
    np.testing.assert_allclose(o_on, o_full, rtol=1e-13, atol=1e-14)
    np.testing.assert_allclose(lse_on, lse_full, rtol=1e-13, atol=1e-14)


# ---------------------------------------------------------------- decoding: Nq query rows against Nk keys
@pytest.mark.parametrize("nq,nk", [(1, 1), (1, 9), (3, 9), (9, 9), (4, 17)])
def test_causal_decode_is_the_tail_of_full_causal_attention(nq, nk):
    """The reading puts the Nq queries at the last positions: their rows of square
    causal attention over all Nk positions (itself pinned to the C brute force)."""
    B, Hq, Hkv, d = 2, 4, 2, 3
    qfull, k, v = rand(B, Hq, nk, d), rand(B, Hkv, nk, d), rand(B, Hkv, nk, d)
    o_full, lse_full = ref.ref_fwd(qfull, k, v, 0.7, True)
    o, lse = ref.ref_decode(qfull[:, :, nk - nq:], k, v, 0.7, True)
    np.testing.assert_allclose(o, o_full[:, :, nk - nq:], rtol=1e-13, atol=1e-14)
    np.testing.assert_allclose(lse, lse_full[:, :, nk - nq:], rtol=1e-13, atol=1e-14)
    ob, lseb = obuild.brute_fwd(qfull, k, v, 0.7, True)
    np.testing.assert_allclose(o, ob[:, :, nk - nq:], rtol=1e-12, atol=1e-13)


@pytest.mark.parametrize("causal", [False, True])
def test_decode_matches_torch_sdpa_rectangular(causal):
    B, Hq, Hkv, nq, nk, d = 2, 6, 3, 5, 23, 4
    q, k, v = rand(B, Hq, nq, d), rand(B, Hkv, nk, d), rand(B, Hkv, nk, d)
    mask = None
    if causal:   # bottom-right aligned: query i sees keys j <= nk - nq + i
        mask = torch.arange(nk)[None, :] <= torch.arange(nq)[:, None] + (nk - nq)
    to = torch.nn.functional.scaled_dot_product_attention(
        torch.tensor(q), torch.tensor(k).repeat_interleave(2, dim=1), torch.tensor(v).repeat_interleave(2, dim=1),
        attn_mask=mask, scale=0.3)
    o, lse = ref.ref_decode(q, k, v, 0.3, causal)
    np.testing.assert_allclose(o, to.numpy(), rtol=1e-10, atol=1e-12)
    s = 0.3 * np.einsum("bhqd,bhkd->bhqk", q, np.repeat(k, 2, axis=1))
    if causal:
        s = np.where(mask.numpy(), s, -np.inf)
    np.testing.assert_allclose(lse, np.log(np.exp(s).sum(axis=-1)), rtol=1e-12)


def test_decode_partials_merge_by_lse():
    """The merge rule the split-KV path relies on: attention over disjoint key ranges,
    combined with weights exp(LSE_s - LSE), equals attention over all keys."""
    nq, nk, d = 3, 40, 5
    qh, kh, vh = rand(nq, d), rand(nk, d), rand(nk, d)
    o, lse = ref.attend_head(qh, kh, vh, 0.9, False)
    parts = [ref.attend_head(qh, kh[a:b], vh[a:b], 0.9, False) for a, b in ((0, 7), (7, 8), (8, 40))]
    m = np.max([p[1] for p in parts], axis=0)
    w = [np.exp(p[1] - m) for p in parts]
    lse_m = m + np.log(sum(w))
    o_m = sum(wi[:, None] * p[0] for wi, p in zip(w, parts)) / sum(w)[:, None]
    np.testing.assert_allclose(o_m, o, rtol=1e-13, atol=1e-14)
    np.testing.assert_allclose(lse_m, lse, rtol=1e-13)


# ---------------------------------------------------------------- e4m3 inputs
def test_e4m3_decoding_matches_torch_on_every_code():
    codes = np.arange(256, dtype=np.uint8)
    ours = ref.decode_e4m3(codes)
    theirs = torch.from_numpy(codes).view(torch.float8_e4m3fn).to(torch.float64).numpy()
    nan = np.isnan(theirs)
    assert nan.sum() == 2 and np.array_equal(np.isnan(ours), nan)          # 0x7f, 0xff
    np.testing.assert_array_equal(ours[~nan], theirs[~nan])
    assert ours[0x7e] == 448.0 and ours[0x01] == 2.0 ** -9 and ours[0x38] == 1.0 and ours[0xb8] == -1.0


def test_fp8_oracle_is_the_definition_on_the_dequantised_values():
    from attn_inputs import make_fp8_inputs
    x = make_fp8_inputs(1, 2, 1, 9, 4, seed=5)
    q8, k8, v8 = (x[n].view(torch.uint8).numpy() for n in ("q", "k", "v"))
    o, lse = ref.ref_fwd_fp8(q8, k8, v8, x["q_descale"], x["k_descale"], x["v_descale"], 0.5, True)
    qf, kf, vf = (x[n].to(torch.float64).numpy() * x[n + "_descale"] for n in ("q", "k", "v"))
    ob, lseb = obuild.brute_fwd(qf, kf, vf, 0.5, True)
    np.testing.assert_allclose(o, ob, rtol=1e-12, atol=1e-13)
    np.testing.assert_allclose(lse, lseb, rtol=1e-12, atol=1e-13)
