"""The bench line's contract, on a short run of the default problem.

The line is what the measurement is judged by, so every key it must carry is
checked: metric and unit, the whole-job value, the roofline with its measured
peak and DRAM traffic, the end-to-end figure with its copied bytes, the
launch count, the clock record and the CPU baseline slot.
"""

import json
import os
import subprocess
import sys

import pytest
import torch

pytestmark = pytest.mark.gpu

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


@pytest.fixture(scope="module", autouse=True)
def cuda_ready():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")


def test_default_bench_line_carries_every_key():
    r = subprocess.run([sys.executable, os.path.join(ROOT, "bench.py"), "--steps", "5", "--warmup", "3",
                        "--no-cpu-baseline"], capture_output=True, text=True, timeout=600, cwd=ROOT)
    assert r.returncode == 0, r.stderr[-2000:]
    lines = [l for l in r.stdout.splitlines() if l.startswith("{")]
    assert len(lines) == 1
    d = json.loads(lines[0])
    assert d["metric"].startswith("attention fwd TFLOP/s") and d["unit"] == "TFLOP/s"
    assert d["n_gpus"] == 1 and d["steps"] == 5 and d["warmup"] == 3
    assert d["higher_is_better"] is True and d["scaling"] == "weak" and d["dtype"] == "bf16"
    assert d["vs_baseline"] is None and d["value"] > 0 and d["ms_per_step"] > 0
    assert d["config"]["workload"] == "b2h16n8192d128_causal"
    rf = d["roofline"]
    assert rf["bound"] == "tensor" and rf["unit"] == "TFLOP/s" and rf["peak"] > 0
    assert abs(rf["frac"] - rf["achieved"] / rf["peak"]) < 1e-9
    assert "traffic" in rf
    e2e = d["e2e"]
    assert e2e["value"] > 0 and e2e["unit"] == "TFLOP/s"
    assert e2e["h2d_bytes_per_step"] == 3 * 2 * 16 * 8192 * 128 * 2
    assert e2e["d2h_bytes_per_step"] == 2 * 16 * 8192 * 128 * 2 + 2 * 16 * 8192 * 4
    assert d["gpu_launches"] == 5
    assert {"sm_mhz", "sm_max_mhz", "reasons"} <= set(d["clocks"])
    assert "cpu_baseline" in d and d["cpu_baseline"] is None  # skipped by --no-cpu-baseline
