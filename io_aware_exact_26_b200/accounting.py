"""FLOP and byte accounting for exact attention (host-side arithmetic, no GPU).

Used by the benchmark to turn a measured time into TFLOPS and into achieved
algorithmic bandwidth, and by the tests to check the byte model against the
numbers the attention pages print.

Counting rules
--------------
* Forward FLOPs: two contractions S = Q K^T and O = P V, each 2*N*N*d per head
  (page "注意力计算的计算与显存瓶颈" §1.1.3: both are n*n*d multiply-adds), so
  4*B*Hq*N^2*d.  Backward: five contractions (S recomputed, dP, dV, dK, dQ), so
  10*B*Hq*N^2*d.  Causal masking halves both (the usual convention for the
  triangular half of S).
* Algorithmic bytes are the tensors the method must move through HBM once:
  the forward reads Q, K, V and writes O and LSE; the backward reads Q, K, V, O,
  dO, LSE and writes dQ, dK, dV.  K and V count once per kv-head (GQA).
  Page "性能模型：用 Roofline 与算术强度算清为什么快" §3.1.3: only the necessary
  Q/K/V/O traffic is left once S and P stay on chip.
* The materialising ("standard") attention's intermediate S and P, each an
  [n, n] matrix, for the byte figures on page 1 §1.1.2 and page 4's
  parameter-ledger row.
"""
from __future__ import annotations

BF16 = 2
FP32 = 4


def flops_fwd(B, Hq, N, d, causal):
    f = 4.0 * B * Hq * N * N * d
    return f / 2 if causal else f


def flops_bwd(B, Hq, N, d, causal):
    f = 10.0 * B * Hq * N * N * d
    return f / 2 if causal else f


def min_bytes_fwd(B, Hq, Hkv, N, d):
    qo = 2 * B * Hq * N * d * BF16
    kv = 2 * B * Hkv * N * d * BF16
    return qo + kv + B * Hq * N * FP32


def min_bytes_bwd(B, Hq, Hkv, N, d):
    q_side = 4 * B * Hq * N * d * BF16        # read Q, O, dO; write dQ
    kv_side = 4 * B * Hkv * N * d * BF16      # read K, V; write dK, dV
    return q_side + kv_side + B * Hq * N * FP32   # read LSE


def score_matrix_bytes(n, elem_bytes=BF16):
    """One [n, n] score (or probability) matrix."""
    return n * n * elem_bytes


def naive_sp_bytes(n, elem_bytes=BF16):
    """S and P together, as the materialising implementation keeps both."""
    return 2 * score_matrix_bytes(n, elem_bytes)


def qk_flops(n, d):
    return 2.0 * n * n * d


def qk_bytes(n, d, elem_bytes=BF16):
    """Read Q and K, write S."""
    return 2 * n * d * elem_bytes + n * n * elem_bytes


def softmax_flops(n):
    """About three operations per score: subtract the max, exponentiate, divide."""
    return 3.0 * n * n


def softmax_bytes(n, elem_bytes=BF16):
    """Read S, write P."""
    return 2 * n * n * elem_bytes


def balance_point(flops_per_s, bytes_per_s):
    """Roofline ridge: arithmetic intensity above which a kernel is compute bound."""
    return flops_per_s / bytes_per_s


def tflops(flops, ms):
    return flops / (ms * 1e-3) / 1e12


def min_bytes_decode(B, Hq, Hkv, Nq, Nk, d):
    """Decoding reads Q, K, V once and writes O and LSE: K and V dominate, O(Nk * d)."""
    return 2 * B * Hq * Nq * d * BF16 + 2 * B * Hkv * Nk * d * BF16 + B * Hq * Nq * FP32


def flops_decode(B, Hq, Nq, Nk, d, causal):
    """4*d FLOPs per visible (query, key) pair; causal queries are the last Nq positions."""
    if causal:
        pairs = sum(Nk - Nq + 1 + i for i in range(Nq))
    else:
        pairs = Nq * Nk
    return 4.0 * B * Hq * pairs * d


def visible_pairs(N, left, right):
    """Number of (query, key) pairs with i - left <= j <= i + right (None = no limit),
    0 <= i, j < N."""
    wl = N if left is None else min(left, N)
    wr = N if right is None else min(right, N)
    total = 0
    for i in range(N):
        total += min(N - 1, i + wr) - max(0, i - wl) + 1
    return total


def flops_window(B, Hq, N, d, left, right, bwd=False):
    """4*d FLOPs per visible pair forward, 10*d backward (the dense counts restricted to
    the band; causal, (None, 0), gives exactly the halved-plus-diagonal count)."""
    return (10.0 if bwd else 4.0) * B * Hq * visible_pairs(N, left, right) * d
