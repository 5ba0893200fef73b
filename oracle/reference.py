"""numpy fp64 oracle for exact attention (TEST INFRASTRUCTURE ONLY, see package docstring).

Definition followed (page "attention 的显存线性化", §一, and page "注意力计算的计算与
显存瓶颈", §1.1.1): S = Q K^T / sqrt(d_k), P = softmax(S) row by row, O = P V.
The row softmax subtracts the row maximum first (same page 1, §1.1.8 formula):
P_ij = exp(S_ij - m_i) / sum_j exp(S_ij - m_i).

Readings where the pages are silent:
* ``scale`` is an explicit argument; the intended value is 1/sqrt(d).
* causal: query i sees keys j <= i (equal query and key lengths).
* local (sliding-window) attention, page "attn-efficient", efficient-attention
  family table, sliding-window row (Longformer / Mistral: each position attends
  only to the w positions nearest it, O(n*w)): the pages give no convention for
  "nearest", so ``window = (left, right)`` lets query i see keys j with
  i - left <= j <= i + right (None = no limit on that side).  Mistral's causal
  window of w positions is (w - 1, 0); a symmetric window is (w/2, w/2).  With
  causal=True the window is intersected with j <= i.
* GQA (page "attn-efficient", table of the three families, row ③): q-head h uses
  kv-head h // (Hq // Hkv), contiguous groups.
* LSE_i = m_i + ln sum_j exp(S_ij - m_i), natural log over the scaled scores,
  masked keys excluded.
* Backward (the pages only say it recomputes local blocks, page
  "attention 的显存线性化" §五): exact gradient of L = sum(O * dO):
  dV = P^T dO, dP = dO V^T, D_i = sum_k dO_ik O_ik, dS = P * (dP - D),
  dQ = scale dS K, dK = scale dS^T Q; GQA sums dK, dV over the group.

Rows are independent (page 1 §1.1.8), so computing S and P for a block of rows
at a time gives the same values as the whole matrix; this is the only
restructuring here and it exists only to bound memory at N = 32768.
"""
from __future__ import annotations

import numpy as np


def visible(rows, nkeys, causal, window=None):
    """[len(rows), nkeys] booleans: may query row i see key j (the mask of the definition)."""
    i = np.asarray(rows)[:, None]
    j = np.arange(nkeys)[None, :]
    vis = np.ones((i.shape[0], nkeys), dtype=bool)
    if causal:
        vis &= j <= i
    if window is not None:
        left, right = window
        if left is not None:
            vis &= j >= i - left
        if right is not None:
            vis &= j <= i + right
    return vis


def _scores(qh, kh, scale, causal, rows, window=None):
    """S for the query rows ``rows`` (array of indices) of one head, fp64, masked with -inf."""
    s = scale * (qh[rows] @ kh.T)
    if causal or window is not None:
        s = np.where(visible(rows, kh.shape[0], causal, window), s, -np.inf)
    return s


def _softmax_rows(s):
    """Row softmax with max subtraction; returns (P, m, LSE)."""
    m = s.max(axis=1)
    e = np.exp(s - m[:, None])
    l = e.sum(axis=1)
    return e / l[:, None], m, m + np.log(l)


def attend_head(qh, kh, vh, scale, causal, rows=None, block=1024, window=None):
    """O and LSE for the given query rows of one head (all rows when ``rows`` is None).

    qh: [N, d]; kh, vh: [N, d]; fp64.  Returns (O[len(rows), d], LSE[len(rows)]).
    """
    n = qh.shape[0]
    rows = np.arange(n) if rows is None else np.asarray(rows, dtype=np.int64)
    o = np.empty((rows.shape[0], vh.shape[1]))
    lse = np.empty(rows.shape[0])
    for a in range(0, rows.shape[0], block):
        r = rows[a:a + block]
        p, _, lse[a:a + block] = _softmax_rows(_scores(qh, kh, scale, causal, r, window))
        o[a:a + block] = p @ vh
    return o, lse


def ref_fwd(q, k, v, scale, causal, block=1024, window=None):
    """Forward oracle.  q [B,Hq,N,d], k/v [B,Hkv,N,d] fp64 -> O [B,Hq,N,d], LSE [B,Hq,N]."""
    B, Hq, N, d = q.shape
    G = Hq // k.shape[1]
    o = np.empty((B, Hq, N, v.shape[3]))
    lse = np.empty((B, Hq, N))
    for b in range(B):
        for h in range(Hq):
            o[b, h], lse[b, h] = attend_head(q[b, h], k[b, h // G], v[b, h // G], scale, causal,
                                             block=block, window=window)
    return o, lse


def grad_rows(qh, kh, vh, doh, scale, causal, r, window=None):
    """The part of the one-head gradient that comes from the query rows ``r``:
    (dQ[r], that block's terms of dK, that block's terms of dV), fp64."""
    p, _, _ = _softmax_rows(_scores(qh, kh, scale, causal, r, window))
    o = p @ vh
    dd = (doh[r] * o).sum(axis=1)              # D_i = sum_k dO_ik O_ik
    dp = doh[r] @ vh.T                          # dP = dO V^T
    ds = p * (dp - dd[:, None])                 # dS = P * (dP - D)
    return scale * (ds @ kh), scale * (ds.T @ qh[r]), p.T @ doh[r]


def grad_head(qh, kh, vh, doh, scale, causal, block=1024, window=None):
    """Gradients of sum(O * dO) for one q-head against its kv-head: (dQ, dK, dV), fp64.
    dK and dV are sums over query rows, taken one row block at a time."""
    n = qh.shape[0]
    dq = np.empty_like(qh)
    dk = np.zeros_like(kh)
    dv = np.zeros_like(vh)
    for a in range(0, n, block):
        r = np.arange(a, min(n, a + block))
        dq[r], dkr, dvr = grad_rows(qh, kh, vh, doh, scale, causal, r, window)
        dk += dkr
        dv += dvr
    return dq, dk, dv


def ref_bwd(q, k, v, do, scale, causal, block=1024, window=None):
    """Backward oracle: (dQ [B,Hq,N,d], dK [B,Hkv,N,d], dV [B,Hkv,N,d]) in fp64."""
    B, Hq, N, d = q.shape
    Hkv = k.shape[1]
    G = Hq // Hkv
    dq = np.empty_like(q)
    dk = np.zeros_like(k)
    dv = np.zeros_like(v)
    for b in range(B):
        for h in range(Hq):
            g = h // G
            dq[b, h], dkh, dvh = grad_head(q[b, h], k[b, g], v[b, g], do[b, h], scale, causal,
                                           block=block, window=window)
            dk[b, g] += dkh
            dv[b, g] += dvh
    return dq, dk, dv


def ref_decode(q, k, v, scale, causal):
    """Attention of Nq new query rows against Nk cached keys (split-KV decoding; page
    "attention 的显存线性化", reading list on FlashDecoding, and the online-softmax
    part of page "attn-efficient", whose rescale merges the per-split partials).

    q [B,Hq,Nq,d], k/v [B,Hkv,Nk,d], fp64.  The result is the plain definition over
    all Nk keys; how the keys are split never shows.  Causal reading (the pages give
    none for Nq != Nk): the query rows are the LAST Nq positions of the sequence, so
    query i sits at position Nk - Nq + i and sees keys j <= Nk - Nq + i -- the window
    (None, Nk - Nq) of ``visible``.  Returns (O [B,Hq,Nq,d], LSE [B,Hq,Nq]).
    """
    nq, nk = q.shape[2], k.shape[2]
    if causal and nq > nk:
        raise ValueError("causal decoding needs Nq <= Nk")
    return ref_fwd(q, k, v, scale, False, window=(None, nk - nq) if causal else None)


def decode_e4m3(codes):
    """Values of e4m3 bytes (OCP FP8 E4M3: sign bit, 4 exponent bits with bias 7, 3
    mantissa bits; exponent 0 is subnormal, m/8 * 2^-6; the all-ones pattern
    S.1111.111 is NaN; there are no infinities), as float64."""
    c = np.asarray(codes, dtype=np.uint8).astype(np.int64)
    sign = np.where(c & 0x80, -1.0, 1.0)
    e = (c >> 3) & 0xF
    m = c & 0x7
    val = np.where(e == 0, m / 8.0 * 2.0 ** -6, (1.0 + m / 8.0) * 2.0 ** (e - 7.0))
    val = np.where((e == 15) & (m == 7), np.nan, val)
    return sign * val


def ref_fwd_fp8(q8, k8, v8, q_descale, k_descale, v_descale, scale, causal):
    """Forward oracle for e4m3 inputs: the plain definition on the values they stand
    for, q = decode(q8) * q_descale (likewise k, v), in fp64.  q8/k8/v8 are the raw
    bytes (uint8 arrays)."""
    return ref_fwd(decode_e4m3(q8) * q_descale, decode_e4m3(k8) * k_descale, decode_e4m3(v8) * v_descale,
                   scale, causal)


def online_fwd_head(qh, kh, vh, scale, causal, bounds, window=None):
    """The pages' blockwise online softmax for one head (used only in self-tests).

    Page "attention 的显存线性化" §三: for each key block j, with S_ij = Q_i K_j^T,
      m^(j) = max(m^(j-1), rowmax S_ij)
      l^(j) = exp(m^(j-1) - m^(j)) l^(j-1) + rowsum exp(S_ij - m^(j)).
    The output update printed there is incomplete; page "attn-efficient"
    (online-softmax section) completes it: whenever the max grows, the partial
    output is multiplied by exp(m_old - m_new).  Reading used:
      O_acc^(j) = exp(m^(j-1) - m^(j)) O_acc^(j-1) + exp(S_ij - m^(j)) V_j,
      O = O_acc / l,  LSE = m + ln l.
    ``bounds`` are the key-block edges, e.g. [0, 3, 4, 10, N].
    """
    n, dv = qh.shape[0], vh.shape[1]
    rows = np.arange(n)
    m = np.full(n, -np.inf)
    l = np.zeros(n)
    acc = np.zeros((n, dv))
    for a, b in zip(bounds[:-1], bounds[1:]):
        s = scale * (qh @ kh[a:b].T)
        if causal or window is not None:
            s = np.where(visible(rows, kh.shape[0], causal, window)[:, a:b], s, -np.inf)
        m_new = np.maximum(m, s.max(axis=1))
        live = np.isfinite(m_new)   # rows that have seen at least one unmasked key
        alpha = np.where(live, np.exp(np.where(live, m, 0.0) - np.where(live, m_new, 0.0)), 1.0)
        pt = np.where(live[:, None], np.exp(s - np.where(live, m_new, 0.0)[:, None]), 0.0)
        l = alpha * l + pt.sum(axis=1)
        acc = alpha[:, None] * acc + pt @ vh[a:b]
        m = m_new
    return acc / l[:, None], m + np.log(l)


def grad_q_rows(qh, kh, vh, doh, scale, causal, rows, window=None):
    """dQ for the given query rows of one head (full key range), from the same formulas as
    ``grad_head``; used to check sampled rows of full-size problems."""
    rows = np.asarray(rows, dtype=np.int64)
    p, _, _ = _softmax_rows(_scores(qh, kh, scale, causal, rows, window))
    o = p @ vh
    dd = (doh[rows] * o).sum(axis=1)
    ds = p * (doh[rows] @ vh.T - dd[:, None])
    return scale * (ds @ kh)


def grad_kv_rows(qhs, kh, vh, dohs, scale, causal, keys, block=1024, window=None):
    """dK and dV for the given key rows of one kv-head, summed over the q-heads in
    ``qhs`` / ``dohs`` (the GQA group).  Needs LSE and D of every query row, so it
    costs one full forward per q-head."""
    keys = np.asarray(keys, dtype=np.int64)
    dk = np.zeros((keys.shape[0], kh.shape[1]))
    dv = np.zeros((keys.shape[0], vh.shape[1]))
    n = kh.shape[0]
    for qh, doh in zip(qhs, dohs):
        for a in range(0, n, block):
            r = np.arange(a, min(n, a + block))
            p_full, m, lse = _softmax_rows(_scores(qh, kh, scale, causal, r, window))
            o = p_full @ vh
            dd = (doh[r] * o).sum(axis=1)
            p = p_full[:, keys]                          # P[r, keys]
            dp = doh[r] @ vh[keys].T
            ds = p * (dp - dd[:, None])
            dk += scale * (ds.T @ qh[r])
            dv += p.T @ doh[r]
    return dk, dv
