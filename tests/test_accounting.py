"""The byte / FLOP model the benchmark uses, pinned to numbers the attention pages print."""
import os

import pytest

from io_aware_exact_26_b200 import accounting as acc

GOLDEN = os.path.join(os.path.dirname(__file__), "golden", "page_numbers.txt")


def _golden():
    out = {}
    with open(GOLDEN, encoding="utf-8") as f:
        for line in f:
            if not line.strip() or line.startswith("#"):
                continue
            key, val, tol, cite = (x.strip() for x in line.split("|"))
            out[key] = (float(val), float(tol), cite)
    return out


G = _golden()

COMPUTED = {
    "sp_fp16_bytes_per_n2": lambda: acc.naive_sp_bytes(1000) / 1000 ** 2,
    "sp_growth_8k_to_64k": lambda: acc.naive_sp_bytes(65536) / acc.naive_sp_bytes(8192),
    "qk_flops_n4096_d4096": lambda: acc.qk_flops(4096, 4096),
    "softmax_flops_n4096": lambda: acc.softmax_flops(4096),
    "softmax_bytes_n4096": lambda: acc.softmax_bytes(4096),
    "softmax_ai": lambda: acc.softmax_flops(4096) / acc.softmax_bytes(4096),
    "a100_balance_point": lambda: acc.balance_point(312e12, 2.0e12),
    "qk_ai_n8192_order": lambda: 8192 / 4,
    "s_mb_d128_n4096": lambda: acc.score_matrix_bytes(4096) / 1e6,
    "sp_mb_d128_n4096": lambda: acc.naive_sp_bytes(4096) / 1e6,
    "o_mb_d128_n4096": lambda: 4096 * 128 * acc.BF16 / 1e6,
    "sp_mb_d128_n8192": lambda: acc.naive_sp_bytes(8192) / 1e6,
    "s_fp32_mib_n4096": lambda: acc.score_matrix_bytes(4096, acc.FP32) / 2 ** 20,
    "score_mb_n4096": lambda: acc.score_matrix_bytes(4096) / 1e6,
    "score_gb_n131072": lambda: acc.score_matrix_bytes(131072) / 1e9,
    "score_elems_n131072": lambda: 131072 ** 2,
    "a100_std_bw_gbs": lambda: 40.3 / 41.7e-3,
    "a100_fa_bw_gbs": lambda: 4.4 / 7.3e-3,
    "a100_speedup": lambda: 41.7 / 7.3,
}


@pytest.mark.parametrize("key", sorted(G))
def test_page_number(key):
    val, tol, cite = G[key]
    got = COMPUTED[key]()
    assert got == pytest.approx(val, rel=max(tol, 1e-12)), cite


def test_every_golden_number_is_checked():
    assert set(G) == set(COMPUTED)


def test_page_script_table_quadruples_per_doubling():
    """The S+P table the page's NumPy script prints (page 1, second §1.1.8): MiB = 4 n^2 / 2^20."""
    mib = [acc.naive_sp_bytes(n) / 2 ** 20 for n in (1024, 2048, 4096, 8192, 16384, 32768)]
    assert mib == [4, 16, 64, 256, 1024, 4096]


def test_worked_example_byte_terms():
    """Page 1 §1.1.5 prints 1.3e8 B for Q K^T, but its own terms sum to about 1.0e8."""
    assert acc.qk_bytes(4096, 4096) == pytest.approx(1.0e8, rel=0.01)
    assert acc.qk_flops(4096, 4096) / acc.qk_bytes(4096, 4096) == pytest.approx(1370, rel=0.01)


def test_attention_flops_and_min_bytes():
    # GPT-2-medium shape, non-causal
    assert acc.flops_fwd(64, 16, 1024, 64, False) == pytest.approx(274.9e9, rel=1e-3)
    assert acc.flops_bwd(64, 16, 1024, 64, False) == pytest.approx(687.2e9, rel=1e-3)
    assert acc.flops_fwd(8, 16, 4096, 128, True) == pytest.approx(549.8e9, rel=1e-3)
    assert acc.flops_fwd(1, 32, 32768, 128, True) == pytest.approx(8.796e12, rel=1e-3)
    # forward minimum: Q, K, V, O in bf16 plus LSE in fp32
    assert acc.min_bytes_fwd(1, 1, 1, 256, 64) == 4 * 256 * 64 * 2 + 256 * 4
    assert acc.min_bytes_fwd(64, 16, 16, 1024, 64) == pytest.approx(541e6, rel=2e-3)
    # GQA counts K, V once per kv head
    assert acc.min_bytes_fwd(4, 32, 8, 8192, 128) == pytest.approx(675e6, rel=2e-3)
    assert acc.min_bytes_bwd(64, 16, 16, 1024, 64) == 8 * 64 * 16 * 1024 * 64 * 2 + 64 * 16 * 1024 * 4
    assert acc.tflops(1e12, 1000.0) == pytest.approx(1.0)


def test_visible_pair_counts_of_bands():
    N = 777
    assert acc.visible_pairs(N, None, None) == N * N
    assert acc.visible_pairs(N, None, 0) == N * (N + 1) // 2              # causal
    assert acc.visible_pairs(N, 0, 0) == N                                 # each row sees itself
    assert acc.visible_pairs(N, 10, 0) == sum(min(i, 10) + 1 for i in range(N))
    assert acc.visible_pairs(N, 3, 5) == sum(min(N - 1, i + 5) - max(0, i - 3) + 1 for i in range(N))
    assert acc.flops_window(1, 1, N, 64, None, 0) == 4 * 64 * N * (N + 1) / 2


def test_decode_bytes_and_flops():
    assert acc.min_bytes_decode(2, 8, 2, 1, 1000, 128) == 2 * 2 * 8 * 128 * 2 + 2 * 2 * 2 * 1000 * 128 * 2 + 2 * 8 * 4
    assert acc.flops_decode(1, 1, 1, 10, 4, True) == 4 * 10 * 4          # the last query sees all keys
    assert acc.flops_decode(1, 1, 3, 10, 4, True) == 4 * 4 * (8 + 9 + 10)
    assert acc.flops_decode(1, 1, 3, 10, 4, False) == 4 * 4 * 30
