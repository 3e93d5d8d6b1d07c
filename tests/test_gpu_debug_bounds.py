"""The bounds-checking debug build (ZERO_DEBUG_BOUNDS; compute-sanitizer is
not available here): every kernel checks each index and pointer it derives
before the access that uses it, skips a failing access and records it. A
cross-section of the hot path runs through that build in a child process,
with parity against the oracle, and must record no failing access."""
import json
import os
import subprocess
import sys

import pytest

pytestmark = pytest.mark.gpu

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def test_debug_build_records_no_out_of_range_access():
    sys.path.insert(0, ROOT)
    from zero_partitioned_mixed_reduce_b200 import build
    lib = build.build(debug=True)
    env = dict(os.environ, ZERO_B200_LIB=lib)
    r = subprocess.run([sys.executable, os.path.join(ROOT, "tests", "debug_bounds_run.py")],
                       capture_output=True, text=True, env=env, cwd=ROOT, timeout=900)
    assert r.returncode == 0, (r.stdout[-3000:], r.stderr[-3000:])
    rec = json.loads(r.stdout.strip().splitlines()[-1])
    assert rec["cases"] == 34
    assert rec["count"] == 0, rec
