"""The benchmark's JSON line carries every key of its contract, with
consistent values: one small run (the tiny workload) end to end, the CPU
oracle baseline and the e2e leg included."""
import json
import os
import subprocess
import sys

import pytest

pytestmark = pytest.mark.gpu

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def test_bench_line_has_the_contract_keys():
    cmd = ["timeout", "-k", "30", "900", sys.executable, os.path.join(ROOT, "bench.py"), "--workload", "tiny",
           "--steps", "5", "--warmup", "3"]
    r = subprocess.run(cmd, capture_output=True, text=True, cwd=ROOT)
    assert r.returncode == 0, (r.stdout[-3000:], r.stderr[-3000:])
    lines = [ln for ln in r.stdout.splitlines() if ln.startswith("{")]
    assert len(lines) == 1
    out = json.loads(lines[0])
    for k in ("metric", "value", "unit", "n_gpus", "steps", "warmup", "ms_per_step", "higher_is_better",
              "scaling", "vs_baseline", "dtype", "data", "config", "roofline", "cpu_baseline", "e2e",
              "gpu_launches", "clocks"):
        assert k in out, k
    assert out["n_gpus"] == 1 and out["steps"] == 5 and out["warmup"] == 3 and out["higher_is_better"] is True
    assert out["unit"] == "params/s" and out["value"] > 0 and out["vs_baseline"] is None
    assert abs(out["value"] - out["config"]["P"] * 5 / (out["ms_per_step"] * 5e-3)) <= 1e-6 * out["value"]
    assert out["config"]["workload"].startswith("tiny")
    roof = out["roofline"]
    for k in ("bound", "achieved", "peak", "unit", "frac", "traffic"):
        assert k in roof, k
    assert roof["bound"] == "hbm" and roof["unit"] == "GB/s" and roof["achieved"] > 0
    assert abs(roof["frac"] - roof["achieved"] / roof["peak"]) <= 1e-12
    assert abs(roof["frac_of_nominal"] - roof["achieved"] / 8000.0) <= 1e-12  # the 8 TB/s spec figure
    assert roof["traffic"] is None  # no stored counters for this workload
    cb = out["cpu_baseline"]
    assert cb["kind"] == "oracle" and cb["cores"] >= 1 and cb["value"] > 0 and cb["sample"]
    e2e = out["e2e"]
    T = out["config"]["T"]
    assert e2e["value"] > 0 and e2e["unit"] == "params/s"
    assert e2e["h2d_bytes_per_step"] == out["config"]["R"] * T * 2  # every replica, 2 bytes an element
    assert e2e["d2h_bytes_per_step"] >= 2 * T  # the updated half parameters come back
    assert out["gpu_launches"] == 5 * 2  # one fused step and one gather per step
