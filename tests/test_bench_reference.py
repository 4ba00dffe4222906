"""The reference arm of bench.py (the oracle timed on the host cores) keeps the JSON line
contract: one line, impl "reference", the metric and unit of the GPU arm, a cpu_baseline
describing the run and an e2e entry with no host-device bytes.  It needs no GPU."""
import json
import os
import subprocess
import sys

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def run_bench(*args):
    out = subprocess.run([sys.executable, os.path.join(ROOT, "bench.py"), *args],
                         capture_output=True, text=True, timeout=600, cwd=ROOT)
    assert out.returncode == 0, out.stderr[-2000:]
    lines = [l for l in out.stdout.splitlines() if l.strip()]
    assert len(lines) == 1, out.stdout
    return json.loads(lines[0])


@pytest.mark.parametrize("args,unit", [(("--workload", "1k"), "useful TFLOP/s"),
                                       (("--op", "warm_start", "--workload", "warm_tiny"), "GB/s")])
def test_reference_arm_line(args, unit):
    d = run_bench("--impl", "reference", "--steps", "1", "--warmup", "0", *args)
    assert d["impl"] == "reference" and d["unit"] == unit and d["value"] > 0
    for key in ("metric", "n_gpus", "steps", "warmup", "ms_per_step", "higher_is_better",
                "scaling", "dtype", "data", "config"):
        assert key in d, key
    assert d["higher_is_better"] is True and d["steps"] == 1 and d["n_gpus"] == 1
    cb = d["cpu_baseline"]
    assert cb["kind"] == "oracle" and cb["cores"] >= 1 and cb["sample"] and cb["value"] == d["value"]
    e = d["e2e"]
    assert e["value"] == d["value"] and e["unit"] == unit
    assert e["h2d_bytes_per_step"] == 0 and e["d2h_bytes_per_step"] == 0
