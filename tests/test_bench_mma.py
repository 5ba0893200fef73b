"""The tensor-core issue-rate probe (bench_mma.py): it builds for sm_100a without a GPU,
exports its two entry points, rejects bad arguments before launching, and its profile
table has one row per shape."""
import ctypes
import os
import sys

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
sys.path.insert(0, ROOT)

import bench_mma  # noqa: E402


def test_probe_builds_and_exports_its_entry_points():
    L = ctypes.CDLL(bench_mma.build())
    assert hasattr(L, "probe_mma_rate") and hasattr(L, "probe_tmem_ld_rate")


def test_probe_rejects_bad_arguments_without_a_launch():
    L = bench_mma.load()
    buf = (ctypes.c_ulonglong * 32)()
    assert L.probe_mma_rate(7, 10, 1, buf) == -1          # no such mode
    assert L.probe_mma_rate(0, 0, 1, buf) == -1           # no repetitions
    assert L.probe_mma_rate(0, 10, 1, None) == -1         # no output
    assert L.probe_tmem_ld_rate(10, 17, 0, 1, buf) == -1  # more warps than lane quarters x 4
    assert L.probe_tmem_ld_rate(10, 4, 0, 0, buf) == -1   # empty grid


def test_profile_table_has_a_row_per_shape(tmp_path):
    mma = [{"shape": "SS M=128 N=128 K=16", "cycles": 64.0, "math_cycles": 64.0, "fraction_of_peak": 1.0,
            "max_over_sms": 64.1}]
    tmem = [{"warps": 8, "store_16_columns": False, "cycles_per_iteration": 190.0, "load_bytes_per_clk_per_sm": 344.9}]
    path = tmp_path / "p.md"
    bench_mma.write_profile(mma, tmem, 148, 2000, path)
    text = path.read_text()
    assert "| SS M=128 N=128 K=16 | 64.0 | 64 | 1.0 | 64.1 |" in text
    assert "| 8 | no | 190.0 | 344.9 |" in text
    assert "python bench_mma.py --profile" in text
