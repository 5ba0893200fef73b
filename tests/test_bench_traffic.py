"""Host logic of bench_traffic (no GPU): an ncu launch list becomes the DRAM bytes bench.py reports."""
import json
import os
import sys

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
sys.path.insert(0, ROOT)

import bench  # noqa: E402
import bench_traffic  # noqa: E402

HDR = ('"ID","Process ID","Process Name","Host Name","Kernel Name","Context","Stream","Block Size","Grid Size",'
       '"Device","CC","Section Name","Metric Name","Metric Unit","Metric Value"')


def row(i, name, metric, unit, value):
    return (f'"{i}","1","python3","h","{name}","1","7","(32, 1, 1)","(1, 1, 1)","0","10.0","Command line profiler metrics",'
            f'"{metric}","{unit}","{value}"')


def launch(i, name, ms_ns, rd, rd_unit, wr, wr_unit):
    return [row(i, name, "dram__bytes_read.sum", rd_unit, rd), row(i, name, "dram__bytes_write.sum", wr_unit, wr),
            row(i, name, "gpu__time_duration.sum", "nsecond", ms_ns)]


def sample_csv():
    lines = ["==PROF== Connected to process 1", HDR]
    lines += launch(0, "void at::vectorized_elementwise_kernel<4>(int)", "1,000", "2", "Mbyte", "1", "Mbyte")
    lines += launch(1, "attn::sched_reset_kernel(int)", "2,000", "0", "byte", "0", "byte")
    lines += launch(2, "void attn::attn_fwd_pp_kernel<64>(CUtensorMap, attn::FwdParams)", "500,000", "400", "Mbyte",
                    "100", "Mbyte")
    lines += launch(3, "attn::sched_reset_kernel(int)", "2,000", "0", "byte", "0", "byte")
    lines += launch(4, "void attn::attn_fwd_pp_kernel<64>(CUtensorMap, attn::FwdParams)", "520,000", "0.6", "Gbyte",
                    "100", "Mbyte")
    lines += launch(5, "void attn::attn_bwd_prep_kernel<64>(int)", "40,000", "270", "Mbyte", "5", "Mbyte")
    lines += launch(6, "void attn::attn_bwd_kv_kernel<64>(CUtensorMap)", "800,000", "550", "Mbyte", "220", "Mbyte")
    lines += launch(7, "void attn::attn_bwd_q_kernel<64>(CUtensorMap)", "600,000", "540", "Mbyte", "110", "Mbyte")
    lines.append("==PROF== Disconnected from process 1")
    return "\n".join(lines)


def test_launches_are_grouped_per_kernel_with_units_converted():
    agg = bench_traffic.parse_launches(sample_csv())
    assert list(agg) == ["at::vectorized_elementwise_kernel<4>", "attn::sched_reset_kernel",
                         "attn::attn_fwd_pp_kernel<64>", "attn::attn_bwd_prep_kernel<64>",
                         "attn::attn_bwd_kv_kernel<64>", "attn::attn_bwd_q_kernel<64>"]
    fwd = agg["attn::attn_fwd_pp_kernel<64>"]
    assert fwd["n"] == 2 and abs(fwd["ms"] - 1.02) < 1e-12
    assert fwd["rd"] == 400e6 + 0.6e9 and fwd["wr"] == 200e6


def test_per_pass_bytes_are_per_call_sums_of_the_pass_kernels():
    b = bench_traffic.pass_bytes(bench_traffic.parse_launches(sample_csv()))
    assert b["fwd"] == round((400e6 + 600e6 + 200e6) / 2)          # reset kernels move nothing
    assert b["bwd"] == round(275e6 + 770e6 + 650e6)


def test_entries_are_stamped_and_read_back_only_for_the_same_sources(tmp_path, monkeypatch):
    entry = bench_traffic.update("gpt2_medium_b64_h16_n1024_d64", sample_csv(), str(tmp_path), revision="abc1234")
    assert entry["fwd"]["source_hash"] == bench.kernel_source_hash()
    md = (tmp_path / "launches_gpt2_medium_b64_h16_n1024_d64.md").read_text()
    assert "abc1234" in md and "--clock-control none" in md and "`attn::attn_bwd_kv_kernel<64>`" in md
    monkeypatch.setattr(bench, "TRAFFIC_FILE", str(tmp_path / "dram_traffic.json"))
    assert bench.measured_traffic("gpt2_medium_b64_h16_n1024_d64", "bwd") == entry["bwd"]["bytes_per_launch"]
    data = json.loads((tmp_path / "dram_traffic.json").read_text())
    data["gpt2_medium_b64_h16_n1024_d64"]["bwd"]["source_hash"] = "0" * 16    # kernels changed since
    (tmp_path / "dram_traffic.json").write_text(json.dumps(data))
    assert bench.measured_traffic("gpt2_medium_b64_h16_n1024_d64", "bwd") is None


def test_forward_only_workloads_get_no_backward_entry(tmp_path):
    entry = bench_traffic.update("causal_b8_h16_n4096_d128", sample_csv(), str(tmp_path), revision="abc1234")
    assert set(entry) == {"fwd"}


def test_source_fingerprint_ignores_comments_and_layout_but_not_code():
    src = "int f(int x) {\n  // scale\n  return 2 * x; /* twice */\n}\n"
    same = "int f(int x) { return 2 * x; }  // reformatted\n"
    other = "int f(int x) {\n  return 3 * x;\n}\n"
    assert bench.code_text(src) == bench.code_text(same)
    assert bench.code_text(src) != bench.code_text(other)
    assert "scale" not in bench.code_text(src) and "twice" not in bench.code_text(src)
