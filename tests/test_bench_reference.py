"""The reference arm of bench.py (the CPU oracle on a bounded sample) prints one JSON line with the
benchmark contract's keys; it runs without a GPU."""
import json
import os
import subprocess
import sys

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
KEYS = {"impl", "metric", "value", "unit", "n_gpus", "steps", "warmup", "ms_per_step", "higher_is_better",
        "scaling", "vs_baseline", "dtype", "data", "config", "cpu_baseline", "e2e"}


def _run(*extra):
    out = subprocess.run([sys.executable, os.path.join(ROOT, "bench.py"), "--impl", "reference", "--steps", "1",
                          "--warmup", "0", *extra], capture_output=True, text=True, timeout=600, cwd=ROOT)
    assert out.returncode == 0, out.stderr[-2000:]
    lines = [l for l in out.stdout.splitlines() if l.startswith("{")]
    assert len(lines) == 1, out.stdout
    return json.loads(lines[0])


def test_attention_reference_line():
    d = _run("--workload", "tiny", "--cpu-rows", "512")
    assert KEYS <= set(d), KEYS - set(d)
    assert d["impl"] == "reference" and d["value"] > 0 and d["unit"] == "TFLOPS"
    assert d["config"]["workload"] == "tiny"
    assert d["cpu_baseline"]["kind"] == "oracle" and d["cpu_baseline"]["cores"] >= 1
    assert d["e2e"]["h2d_bytes_per_step"] == 0 and d["e2e"]["value"] == d["value"]


def test_linear_reference_line():
    d = _run("--op", "linear", "--linear-workload", "lin_tiny")
    assert KEYS <= set(d), KEYS - set(d)
    assert d["impl"] == "reference" and d["unit"] == "TOPS" and d["value"] > 0
    assert d["config"]["M"] == 333 and d["config"]["K"] == 512


def test_sfu_cap_arithmetic():
    """4*d FLOPs per exponential at 16 results/clk/SM: 2.38 PFLOP/s at d = 128, 148 SMs, 1965 MHz."""
    sys.path.insert(0, ROOT)
    import bench
    assert abs(bench.sfu_cap_tflops(128, 148, 1965.0) - 4 * 128 * 16 * 148 * 1965e6 / 1e12) < 1e-9
    assert 2380 < bench.sfu_cap_tflops(128, 148, 1965.0) < 2385
    assert bench.sfu_cap_tflops(64, 148, 1965.0) * 2 == bench.sfu_cap_tflops(128, 148, 1965.0)
    assert bench.sfu_cap_tflops(128, 148, None) is None
    c = bench.sfu_cap(128, 148, 1965.0, 1416.2)
    assert abs(c["frac"] - 1416.2 / c["tflops"]) < 1e-12
    assert bench.sfu_cap(128, 148, None, 1416.2)["frac"] is None
