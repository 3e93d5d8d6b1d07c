"""bench.py's two-pass clipping modes run end to end and say which norm
they used (the reduce-scatters' shares or a separate pass)."""
import json
import os
import subprocess
import sys

import pytest

pytestmark = pytest.mark.gpu

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


@pytest.mark.parametrize("clip_norm,accum", [("rs", 1), ("rs", 3), ("pass", 3)])
def test_two_pass_clip_bench(clip_norm, accum):
    cmd = ["timeout", "-k", "30", "600", sys.executable, os.path.join(ROOT, "bench.py"),
           "--path", "twopass", "--clip", "1.0", "--accum", str(accum), "--clip-norm", clip_norm,
           "--first-tensors", "6", "--steps", "3", "--warmup", "3", "--no-e2e", "--no-cpu-baseline"]
    r = subprocess.run(cmd, capture_output=True, text=True, cwd=ROOT)
    assert r.returncode == 0, (r.stdout[-3000:], r.stderr[-3000:])
    out = json.loads([ln for ln in r.stdout.splitlines() if ln.startswith("{")][-1])
    path = out["step"]["path"]
    if clip_norm == "rs":
        assert "norm shares" in path
    else:
        assert "clip pass" in path
    assert out["value"] > 0 and out["roofline"]["achieved"] > 0


@pytest.mark.parametrize("clip", [None, "0.5"])
def test_offload_bench_reports_both_clipped_cpu_steps(clip):
    # bench.py --offload on the small workload: the serialized and delayed
    # offloaded steps (clipped, with the norm from the device, under --clip),
    # and the clipped CPU step with the host scan against the one with the
    # norm from the device
    cmd = ["timeout", "-k", "30", "600", sys.executable, os.path.join(ROOT, "bench.py"), "--offload",
           "--workload", "tiny", "--steps", "3", "--warmup", "1", "--tokens", "256"]
    if clip:
        cmd += ["--clip", clip]
    r = subprocess.run(cmd, capture_output=True, text=True, cwd=ROOT)
    assert r.returncode == 0, (r.stdout[-3000:], r.stderr[-3000:])
    out = json.loads([ln for ln in r.stdout.splitlines() if ln.startswith("{")][-1])
    assert out["mode"] == "offload" and out["ms_serialized"] > 0 and out["ms_delayed_update"] > 0
    c = out["clipped_cpu_step"]
    assert c["ms_host_scan_first"] > 0 and c["ms_norm_from_device"] > 0
    assert c["host_bytes_per_param"]["norm_from_device"] < c["host_bytes_per_param"]["host_scan_first"]
    assert out["clip"] == (float(clip) if clip else None) and c["max_grad_norm"] == (float(clip) if clip else 1.0)
