"""bench.py's JSON line on a short run of the 4 x 16 x 2048 x 64 workload: every key the
measurement contract names is present and consistent (the headline, the end-to-end pass
through host buffers, the roofline of the dominant kernel, the launch count, the clock
samples), and the reference arm (the float64 oracle) prints its own line."""
import json
import os
import subprocess
import sys

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))

pytestmark = pytest.mark.gpu


def run_bench(*args):
    out = subprocess.run([sys.executable, os.path.join(ROOT, "bench.py"), *args], cwd=ROOT,
                         capture_output=True, text=True, timeout=600)
    assert out.returncode == 0, out.stderr[-2000:]
    return json.loads(out.stdout.strip().splitlines()[-1])


def test_bench_line_has_the_contract_keys():
    d = run_bench("--config", "2", "--steps", "3", "--warmup", "3", "--no-cpu-baseline")
    assert d["metric"] and d["unit"] == "TFLOP/s" and d["value"] > 0
    assert d["n_gpus"] == 1 and d["steps"] == 3 and d["warmup"] == 3
    assert d["ms_per_step"] > 0 and d["higher_is_better"] is True and d["scaling"] == "weak"
    assert d["dtype"] == "bf16" and d["data"] == "synthetic"
    assert "4x16x2048x64" in d["config"]["workload"]
    r = d["roofline"]
    assert r["bound"] == "tensor" and r["unit"] == "TFLOP/s" and r["peak"] > 0
    assert abs(r["frac"] - r["achieved"] / r["peak"]) < 1e-9
    e = d["e2e"]
    assert e["value"] > 0 and e["unit"] == d["unit"]
    # every step's inputs up and every result down: Q, K, V, E and O, dQ, dK, dV at least
    assert e["h2d_bytes_per_step"] >= 4 * 4 * 16 * 2048 * 64 * 2
    assert e["d2h_bytes_per_step"] >= 4 * 4 * 16 * 2048 * 64 * 2
    assert e["value"] < d["value"]  # the copies cost time
    # nine kernels per step (table, rotation, forward, loss x2, preprocess, dK/dV, dQ, dalpha)
    assert d["gpu_launches"] == 9 * 3
    assert set(d["kernels"]) >= {"fwd_sm100", "bwd_dkdv_sm100", "bwd_dq_sm100"}
    assert "sm_mhz" in d["clocks"] and "reasons" in d["clocks"]


def test_reference_arm_line():
    d = run_bench("--impl", "reference", "--config", "2", "--steps", "1", "--warmup", "0")
    assert d["impl"] == "reference" and d["value"] > 0 and d["dtype"] == "f64"
    assert d["cpu_baseline"]["kind"] == "oracle" and d["cpu_baseline"]["cores"] >= 1
    assert d["e2e"]["h2d_bytes_per_step"] == 0 and d["e2e"]["d2h_bytes_per_step"] == 0
