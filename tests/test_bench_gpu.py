"""bench.py end to end on one GPU: the JSON line keeps its contract.

Runs the benchmark as a user would (a subprocess, small workload, few steps) and checks
the keys and their internal consistency: throughput against the step time, the roofline
object against the backward's own timing, the end-to-end block with its copied bytes,
the kernel-launch count, the clock record and the oracle baseline; and that the
reference arm prints the same metric with its labels.
"""
import json
import os
import subprocess
import sys

import pytest

pytestmark = pytest.mark.gpu

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
WORKLOAD = "gpt2_medium_b64_h16_n1024_d64"   # forward + backward


def run_bench(*extra):
    out = subprocess.run([sys.executable, "bench.py", "--workload", WORKLOAD, *extra], cwd=ROOT,
                         capture_output=True, text=True, timeout=900)
    assert out.returncode == 0, out.stderr[-2000:]
    lines = [ln for ln in out.stdout.splitlines() if ln.startswith("{")]
    assert len(lines) == 1, out.stdout
    return json.loads(lines[0])


def test_bench_line_keeps_its_contract():
    sys.path.insert(0, ROOT)
    import bench
    steps, warmup = 4, 3
    d = run_bench("--steps", str(steps), "--warmup", str(warmup), "--cpu-budget", "1.0")
    for key in ("metric", "value", "unit", "n_gpus", "steps", "warmup", "ms_per_step", "higher_is_better",
                "scaling", "vs_baseline", "dtype", "data", "config", "roofline", "e2e", "gpu_launches",
                "clocks", "fwd", "bwd", "cpu_baseline"):
        assert key in d, key
    assert d["steps"] == steps and d["warmup"] == warmup and d["n_gpus"] == 1
    assert d["config"]["workload"] == WORKLOAD and d["higher_is_better"] is True
    sha = d["config"]["inputs"]["sha256"]
    assert set(sha) == {"q", "k", "v", "do"} and all(len(h) == 64 for h in sha.values())
    f, fb = bench.step_flops(bench.WORKLOADS[WORKLOAD])
    # value is the step's FLOPs over the timed step time
    assert abs(d["value"] - (f + fb) / (d["ms_per_step"] * 1e-3) / 1e12) <= 0.01 * d["value"] + 1e-3
    r = d["roofline"]
    assert r["bound"] == "tensor" and r["unit"] == "TFLOP/s" and r["peak"] > 0
    assert abs(r["achieved"] - d["bwd"]["tflops"]) <= 0.1 + 1e-3 * r["achieved"]
    assert abs(r["frac"] - r["achieved"] / r["peak"]) <= 1e-3
    e = d["e2e"]
    assert e["unit"] == d["unit"] and e["value"] > 0
    assert e["h2d_bytes_per_step"] > 0 and e["d2h_bytes_per_step"] > 0
    assert d["gpu_launches"] == steps * 5             # counter reset + forward, prep + dK/dV + dQ
    assert "sm_mhz" in d["clocks"] and "reasons" in d["clocks"]
    c = d["cpu_baseline"]
    assert c["kind"] == "oracle" and c["value"] > 0 and c["cores"] >= 1 and c["extrapolated"] is True


def test_reference_arm_prints_the_same_metric():
    d = run_bench("--impl", "reference", "--steps", "1", "--warmup", "0")
    assert d["impl"] == "reference" and d["metric"] == "attention fwd+bwd TFLOPS" and d["unit"] == "TFLOPS"
    assert d["cpu_baseline"]["kind"] == "oracle" and d["e2e"]["h2d_bytes_per_step"] == 0
