"""The benchmark's JSON line: the keys and units the result contract asks for, for the
CUDA arm (on a GPU) and for the reference arm (the CPU oracle), on the tiny workload."""
import json
import os
import subprocess
import sys

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def run_bench(*args):
    r = subprocess.run([sys.executable, os.path.join(ROOT, "bench.py"), *args],
                       capture_output=True, text=True, timeout=900, cwd=ROOT)
    assert r.returncode == 0, r.stderr[-2000:]
    lines = [ln for ln in r.stdout.strip().splitlines() if ln.startswith("{")]
    assert len(lines) == 1, r.stdout[-2000:]
    return json.loads(lines[0])


def check_common(line, steps, warmup):
    assert line["metric"].startswith("MoE-layer tokens/s")
    assert line["unit"] == "tokens/s" and line["value"] > 0
    assert line["n_gpus"] == 1 and line["steps"] == steps and line["warmup"] == warmup
    assert line["higher_is_better"] is True and line["scaling"] == "weak"
    assert line["data"] == "synthetic" and line["vs_baseline"] is None
    # value is tokens per second of the whole job: T tokens per step
    cfg = line["config"]
    assert cfg["workload"].startswith("tiny: T=256 ")
    assert abs(line["value"] - cfg["T"] / (line["ms_per_step"] * 1e-3)) <= 1e-6 * line["value"]
    e2e = line["e2e"]
    assert e2e["unit"] == "tokens/s" and e2e["value"] > 0
    assert "h2d_bytes_per_step" in e2e and "d2h_bytes_per_step" in e2e


def test_reference_arm_line():
    line = run_bench("--impl", "reference", "--config", "tiny", "--steps", "1", "--warmup", "3")
    check_common(line, 1, 3)
    assert line["impl"] == "reference" and line["dtype"] == "f64"
    cb = line["cpu_baseline"]
    assert cb["kind"] == "oracle" and cb["cores"] >= 1 and cb["value"] == line["value"]
    assert line["e2e"]["h2d_bytes_per_step"] == 0 and line["e2e"]["d2h_bytes_per_step"] == 0


@pytest.mark.gpu
def test_cuda_arm_line():
    line = run_bench("--config", "tiny", "--steps", "3", "--warmup", "3", "--no-cpu-baseline")
    check_common(line, 3, 3)
    assert "impl" not in line and line["dtype"] == "bf16"
    ref = run_bench("--impl", "reference", "--config", "tiny", "--steps", "1", "--warmup", "3")
    assert line["config"] == ref["config"]  # both arms name the same workload object
    roof = line["roofline"]
    assert roof["bound"] in ("tensor", "hbm", "alu") and roof["peak"] > 0
    assert abs(roof["frac"] - roof["achieved"] / roof["peak"]) < 1e-9
    assert roof["unit"] in ("TFLOP/s", "GB/s") and "traffic" in roof
    # the copies of the end-to-end run are counted from the tensors it moves
    assert line["e2e"]["h2d_bytes_per_step"] > 0 and line["e2e"]["d2h_bytes_per_step"] > 0
    clocks = line["clocks"]
    assert "sm_mhz" in clocks and "sm_max_mhz" in clocks and isinstance(clocks["reasons"], list)
    assert line["gpu_launches"] > 0
    assert 0 < line["index_ms"] < line["ms_per_step"] and 0 < line["ffn_ms"] < line["ms_per_step"]
