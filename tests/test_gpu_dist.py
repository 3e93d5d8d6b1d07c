"""DistributedZero (the multi-GPU ZeRO step over CUDA-IPC peer mappings) launched
under torch.distributed.run on the GPUs this machine offers, compared with
the oracle in the worker (tests/dist_worker.py)."""
import os
import socket
import subprocess
import sys

import pytest
import torch

pytestmark = pytest.mark.gpu

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def test_distributed_zero_matches_oracle():
    nproc = 1  # every rank needs its own GPU; this suite runs on one
    env = dict(os.environ, NCCL_NVLS_ENABLE="0")
    cmd = ["timeout", "-k", "30", "300", sys.executable, "-m", "torch.distributed.run", "--nnodes=1",
           f"--nproc-per-node={nproc}", "--master-addr", "127.0.0.1", "--master-port", str(free_port()),
           os.path.join(ROOT, "tests", "dist_worker.py")]
    r = subprocess.run(cmd, capture_output=True, text=True, env=env, cwd=ROOT)
    assert r.returncode == 0, (r.stdout[-3000:], r.stderr[-3000:])
    assert "ok" in r.stdout


def test_bench_distributed_mode():
    # bench.py --dist: the real multi-GPU step (at one rank here) prints one JSON line
    import json
    env = dict(os.environ, NCCL_NVLS_ENABLE="0")
    cmd = ["timeout", "-k", "30", "600", sys.executable, "-m", "torch.distributed.run", "--nnodes=1",
           "--nproc-per-node=1", "--master-addr", "127.0.0.1", "--master-port", str(free_port()),
           os.path.join(ROOT, "bench.py"), "--dist", "--workload", "gpt2s", "--steps", "3", "--warmup", "3"]
    r = subprocess.run(cmd, capture_output=True, text=True, env=env, cwd=ROOT)
    assert r.returncode == 0, (r.stdout[-3000:], r.stderr[-3000:])
    line = [ln for ln in r.stdout.splitlines() if ln.startswith("{")][-1]
    out = json.loads(line)
    assert out["n_gpus"] == 1 and out["scaling"] == "strong" and out["config"]["parallelism"].startswith("dp1")
    assert out["value"] > 0 and out["config"]["R"] == 1 and out["state_check"] == "ok"
    assert out["roofline"]["bound"] in ("hbm", "nvlink") and out["roofline"]["achieved"] > 0
    assert out["gpu_launches"] > 0 and out["e2e"]["value"] > 0 and out["nccl"]["world_size"] == 1


def test_bench_distributed_zero2_mode():
    # bench.py --dist --zero2: the step pushes the parameters, no layer gathers
    import json
    env = dict(os.environ, NCCL_NVLS_ENABLE="0")
    cmd = ["timeout", "-k", "30", "600", sys.executable, "-m", "torch.distributed.run", "--nnodes=1",
           "--nproc-per-node=1", "--master-addr", "127.0.0.1", "--master-port", str(free_port()),
           os.path.join(ROOT, "bench.py"), "--dist", "--zero2", "--workload", "gpt2s", "--steps", "3",
           "--warmup", "3"]
    r = subprocess.run(cmd, capture_output=True, text=True, env=env, cwd=ROOT)
    assert r.returncode == 0, (r.stdout[-3000:], r.stderr[-3000:])
    out = json.loads([ln for ln in r.stdout.splitlines() if ln.startswith("{")][-1])
    assert out["gather"] is None and out["state_check"] == "ok" and "pushed" in out["step"]["path"]
    assert out["per_rank_bytes"]["gather_hbm"] == 0 and out["value"] > 0
