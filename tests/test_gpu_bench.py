"""bench.py's own arm on the GPU keeps the JSON line contract on a short 1K run: one line with
the metric, a positive whole-step value, the roofline of the attention kernel against a measured
peak, the clocks seen during the timed steps (with the kernel's own clock record), the count of
the library's launches, and an e2e entry through the host-buffer runner with its copied bytes."""
import json
import os
import subprocess
import sys

import pytest

pytestmark = pytest.mark.gpu

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def run_bench(*args):
    out = subprocess.run([sys.executable, os.path.join(ROOT, "bench.py"), *args],
                         capture_output=True, text=True, timeout=900, cwd=ROOT)
    assert out.returncode == 0, out.stderr[-2000:]
    lines = [l for l in out.stdout.splitlines() if l.strip()]
    assert len(lines) == 1, out.stdout
    return json.loads(lines[0])


def test_gpu_arm_line(gpu_required):
    d = run_bench("--workload", "1k", "--steps", "3", "--warmup", "3", "--extra-workloads", "none",
                  "--no-cpu-baseline")
    for key in ("metric", "value", "unit", "n_gpus", "steps", "warmup", "ms_per_step",
                "higher_is_better", "scaling", "dtype", "data", "config", "roofline", "e2e",
                "gpu_launches", "clocks", "ms_per_kernel"):
        assert key in d, key
    assert d["value"] > 0 and d["steps"] == 3 and d["warmup"] == 3 and d["n_gpus"] == 1
    assert d["config"]["workload"] == "1k" and d["dtype"] == "bf16"
    r = d["roofline"]
    assert r["bound"] == "tensor" and r["unit"] == "TFLOP/s" and r["peak"] > 0
    assert 0 < r["frac"] == pytest.approx(r["achieved"] / r["peak"])
    assert r["kernel_sm_mhz"] and 200 < r["kernel_sm_mhz"] < 3000
    # two launches per step (permute_rope, the attention with the unpermute in its epilogue;
    # the 1K plan splits nothing, so there is no merge launch)
    assert d["gpu_launches"] == 2 * 3
    c = d["clocks"]
    assert "reasons" in c and c.get("kernel_sm_mhz")
    e = d["e2e"]
    assert e["value"] > 0 and e["h2d_bytes_per_step"] > 0 and e["d2h_bytes_per_step"] > 0
