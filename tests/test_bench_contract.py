"""bench.py's JSON line: the keys and types the benchmark contract asks for, for the reference arm
(the oracle on the host cores: runs on the CPU) and for the CUDA arm (on a GPU), on the tiny
workload so that each run takes seconds."""
import json
import pathlib
import subprocess
import sys

import pytest

ROOT = pathlib.Path(__file__).resolve().parents[1]


def run_bench(*args, timeout=600):
    res = subprocess.run([sys.executable, str(ROOT / "bench.py"), *args], cwd=ROOT,
                         capture_output=True, text=True, timeout=timeout)
    assert res.returncode == 0, res.stderr[-2000:]
    lines = [ln for ln in res.stdout.splitlines() if ln.startswith("{")]
    assert len(lines) == 1, res.stdout[-2000:]
    return json.loads(lines[0])


def check_common(d, steps, warmup):
    for key in ("metric", "value", "unit", "n_gpus", "steps", "warmup", "ms_per_step",
                "higher_is_better", "scaling", "vs_baseline", "dtype", "data", "config", "e2e"):
        assert key in d, key
    assert d["steps"] == steps and d["warmup"] == warmup and d["n_gpus"] == 1
    assert d["value"] > 0 and d["ms_per_step"] > 0 and d["higher_is_better"] is True
    assert d["scaling"] == "weak" and d["vs_baseline"] is None
    assert d["config"]["workload"] == "tiny_mlra4_f32" and d["config"]["parallelism"] == "dp1"
    e2e = d["e2e"]
    assert e2e["value"] > 0 and e2e["unit"] == d["unit"]
    assert "h2d_bytes_per_step" in e2e and "d2h_bytes_per_step" in e2e


def test_reference_arm_line():
    d = run_bench("--impl", "reference", "--steps", "2", "--warmup", "3",
                  "--workload", "tiny_mlra4_f32")
    check_common(d, 2, 3)
    assert d["impl"] == "reference" and d["dtype"] == "f64"
    cb = d["cpu_baseline"]
    assert cb["kind"] == "oracle" and cb["cores"] >= 1 and cb["value"] == d["value"] and cb["sample"]
    assert d["e2e"]["value"] == d["value"]
    assert d["e2e"]["h2d_bytes_per_step"] == 0 and d["e2e"]["d2h_bytes_per_step"] == 0


@pytest.mark.gpu
def test_cuda_arm_line():
    d = run_bench("--steps", "3", "--warmup", "3", "--workload", "tiny_mlra4_f32", "--no-side",
                  "--no-cpu-baseline")
    check_common(d, 3, 3)
    assert "impl" not in d and d["dtype"] == "bf16" and d["data"] == "synthetic"
    r = d["roofline"]
    for key in ("bound", "achieved", "peak", "unit", "frac", "traffic"):
        assert key in r, key
    assert r["bound"] == "hbm" and r["unit"] == "GB/s" and r["peak"] > 0
    assert abs(r["frac"] - r["achieved"] / r["peak"]) < 1e-9
    assert d["gpu_launches"] > 0
    assert d["e2e"]["h2d_bytes_per_step"] > 0 and d["e2e"]["d2h_bytes_per_step"] > 0
    clk = d["clocks"]
    assert "sm_mhz" in clk and "sm_max_mhz" in clk and isinstance(clk["reasons"], list)
    assert d["warmup_run"] >= 3
