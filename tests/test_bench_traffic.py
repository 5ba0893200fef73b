"""Host logic of bench_traffic (no GPU): an ncu launch list becomes the DRAM bytes bench.py reports."""
import json
import os
import sys

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
sys.path.insert(0, ROOT)

import pytest  # noqa: E402

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


def time_only_csv():
    lines = ["==PROF== Connected to process 1", HDR]
    for i, (name, ns) in enumerate([("attn::sched_reset_kernel(int)", "2,000"),
                                    ("void attn::attn_fwd_pp_kernel<128>(CUtensorMap, attn::FwdParams)", "7,000,000"),
                                    ("void attn::attn_bwd_kv_kernel<128>(CUtensorMap)", "12,000,000")]):
        lines.append(row(i, name, "gpu__time_duration.sum", "nsecond", ns))
    return "\n".join(lines)


def test_launches_are_grouped_per_kernel_with_units_converted():
    agg = bench_traffic.parse_launches(sample_csv())
    assert list(agg) == ["at::vectorized_elementwise_kernel<4>", "attn::sched_reset_kernel",
                         "attn::attn_fwd_pp_kernel<64>", "attn::attn_bwd_prep_kernel<64>",
                         "attn::attn_bwd_kv_kernel<64>", "attn::attn_bwd_q_kernel<64>"]
    fwd = agg["attn::attn_fwd_pp_kernel<64>"]
    assert fwd["n"] == 2 and abs(fwd["ms"] - 1.02) < 1e-12
    assert fwd["rd"] == 400e6 + 0.6e9 and fwd["wr"] == 200e6


def test_time_only_launch_lists_have_no_dram_figures(tmp_path):
    agg = bench_traffic.parse_launches(time_only_csv())
    assert all(a["rd"] is None and a["wr"] is None for a in agg.values())
    path = bench_traffic.write_launches("long_causal_b1_h32_n32768_d128", time_only_csv(), str(tmp_path), "abc1234")
    md = open(path).read()
    assert "abc1234" in md and "--clock-control none" in md and "gpu__time_duration.sum --clock" in md
    assert "dram__" not in md    # the full-size capture collects time only


def test_dram_commands_capture_one_kernel_one_launch():
    for k in bench_traffic.KERNELS:
        cmd = bench_traffic.dram_command("long_causal_b1_h32_n32768_d128", 4, k)
        assert " -k regex:" in cmd and " -c 1 " in cmd and "--clock-control none" in cmd and "--div 4" in cmd


def test_reduced_cases_divide_the_independent_units():
    w = bench.WORKLOADS["long_causal_b1_h32_n32768_d128"]
    r = bench_traffic.reduced(w, 4)
    assert (r.B, r.Hq, r.Hkv, r.N, r.d) == (1, 8, 8, 32768, 128)
    g = bench_traffic.reduced(bench.WORKLOADS["gqa_causal_b4_hq32_hkv8_n8192_d128"], 4)
    assert (g.B, g.Hq, g.Hkv) == (1, 32, 8)
    # still larger than L2 per input tensor set
    assert 3 * r.B * r.Hq * r.N * r.d * 2 > 126e6


def test_dram_entries_scale_to_full_launches_and_are_stamped(tmp_path, monkeypatch):
    texts = [sample_csv()]
    entry = bench_traffic.write_dram("long_causal_b1_h32_n32768_d128", 4, texts, str(tmp_path), revision="abc1234")
    k = entry["kernels"]
    assert k["fwd"]["bytes_per_launch"] == round((400e6 + 600e6 + 200e6) / 2 * 4)
    assert k["bwd_kv"]["bytes_per_launch"] == round(770e6 * 4)
    assert entry["bwd"]["bytes_per_launch"] == sum(k[x]["bytes_per_launch"] for x in ("bwd_prep", "bwd_kv", "bwd_q"))
    assert entry["fwd"]["source_hash"] == bench.kernel_source_hash("fwd")
    assert entry["bwd"]["source_hash"] == bench.kernel_source_hash("bwd")
    md = (tmp_path / "dram_long_causal_b1_h32_n32768_d128.md").read_text()
    assert "abc1234" in md and "-k regex:attn_bwd_kv" in md
    monkeypatch.setattr(bench, "TRAFFIC_FILE", str(tmp_path / "dram_traffic.json"))
    assert bench.measured_traffic("long_causal_b1_h32_n32768_d128", "bwd") == entry["bwd"]["bytes_per_launch"]
    data = json.loads((tmp_path / "dram_traffic.json").read_text())
    data["long_causal_b1_h32_n32768_d128"]["bwd"]["source_hash"] = "0" * 16    # kernels changed since
    (tmp_path / "dram_traffic.json").write_text(json.dumps(data))
    assert bench.measured_traffic("long_causal_b1_h32_n32768_d128", "bwd") is None


def test_time_only_captures_are_refused_as_dram_evidence():
    with pytest.raises(ValueError):
        bench_traffic.dram_entry("long_causal_b1_h32_n32768_d128", 4, [time_only_csv()])


def test_pass_fingerprints_cover_only_their_own_sources(tmp_path):
    import shutil
    src = os.path.join(ROOT, "io_aware_exact_26_b200", "csrc")
    for name in os.listdir(src):
        shutil.copy(os.path.join(src, name), tmp_path / name)
    f0, b0 = bench.kernel_source_hash("fwd", str(tmp_path)), bench.kernel_source_hash("bwd", str(tmp_path))
    (tmp_path / "fwd_pp.cuh").write_text((tmp_path / "fwd_pp.cuh").read_text() + "\nint changed;\n")
    assert bench.kernel_source_hash("fwd", str(tmp_path)) != f0          # the forward's stamp moves
    assert bench.kernel_source_hash("bwd", str(tmp_path)) == b0          # the backward's does not


def test_source_fingerprint_ignores_comments_and_layout_but_not_code():
    src = "int f(int x) {\n  // scale\n  return 2 * x; /* twice */\n}\n"
    same = "int f(int x) { return 2 * x; }  // reformatted\n"
    other = "int f(int x) {\n  return 3 * x;\n}\n"
    assert bench.code_text(src) == bench.code_text(same)
    assert bench.code_text(src) != bench.code_text(other)
    assert "scale" not in bench.code_text(src) and "twice" not in bench.code_text(src)


def test_sweep_dram_summarises_every_point_of_one_head_size(tmp_path):
    """Per-kernel captures of every causal d = 128 sweep point become one table, with the
    ratio to the algorithmic bytes (the same at every N but the last) and row to row."""
    from attn_inputs import sweep_workloads
    pts = [w for w in sweep_workloads() if w.d == 128 and w.causal]
    for i, w in enumerate(pts):
        for k, name in (("fwd_pp", "attn::attn_fwd_pp_kernel<128>(x)"), ("bwd_prep", "attn::attn_bwd_prep_kernel<128>(x)"),
                        ("bwd_kv", "attn::attn_bwd_kv_kernel<128>(x)"), ("bwd_q", "attn::attn_bwd_q_kernel<128>(x)")):
            mb = str(100 + i)                                     # traffic that grows a little with N
            text = "\n".join([HDR] + launch(0, name, "1,000", mb, "Mbyte", "10", "Mbyte"))
            (tmp_path / f"dram_{w.name}_{k}.csv").write_text(text)
    rows = bench_traffic.write_sweep_dram(128, True, str(tmp_path), str(tmp_path), revision="abc1234")
    assert [r["N"] for r in rows] == [w.N for w in pts]
    assert rows[0]["fwd"] == 110e6 and rows[0]["bwd"] == 3 * 110e6
    md = (tmp_path / "dram_sweep_causal_d128.md").read_text()
    assert "abc1234" in md and md.count("\n| ") == len(pts) + 1    # header + one row per point
