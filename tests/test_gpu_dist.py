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


@pytest.mark.parametrize("nproc", [2, 4, 8])
def test_ranks_sharing_one_gpu_over_gloo(nproc):
    # the multi-rank path on the GPU this suite has: nproc processes, each
    # mapping the others' gradient buffers, parameter shards and full-model
    # buffers through CUDA IPC; the step reads every replica (at two ranks the
    # staged kernel's bulk copies from the mapped buffer, at four the register
    # kernel's loads), pushes its parameters into every full-model buffer and
    # gathers from every shard, against the oracle.
    # The ordering all-reduces go through gloo, which blocks on the host; no
    # kernel waits for the other rank
    env = dict(os.environ, ZB_DIST_BACKEND="gloo")
    cmd = ["timeout", "-k", "30", "400", sys.executable, "-m", "torch.distributed.run", "--nnodes=1",
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


@pytest.mark.parametrize("nproc,zero2", [(2, False), (2, True), (8, False)])
def test_bench_distributed_mode_ranks_sharing_one_gpu(nproc, zero2):
    # bench.py --gpus 2 through its whole multi-rank path (the sharded step,
    # the per-rank byte counts, max-over-ranks timing, e2e, the ZeRO-1/2 push)
    # with both ranks on this GPU and gloo for the collectives: a functional
    # run, not a measurement
    import json
    env = dict(os.environ, ZB_BENCH_BACKEND="gloo")
    cmd = ["timeout", "-k", "30", "600", sys.executable, "-m", "torch.distributed.run", "--nnodes=1",
           f"--nproc-per-node={nproc}", "--master-addr", "127.0.0.1", "--master-port", str(free_port()),
           os.path.join(ROOT, "bench.py"), "--gpus", str(nproc), "--workload", "gpt2s", "--steps", "3",
           "--warmup", "3"]
    if zero2:
        cmd.append("--zero2")
    r = subprocess.run(cmd, capture_output=True, text=True, env=env, cwd=ROOT)
    assert r.returncode == 0, (r.stdout[-3000:], r.stderr[-3000:])
    lines = [ln for ln in r.stdout.splitlines() if ln.startswith("{")]
    assert len(lines) == 1  # rank 0 alone prints
    out = json.loads(lines[0])
    assert out["n_gpus"] == nproc and out["scaling"] == "strong" and out["state_check"] == "ok"
    assert out["config"]["R"] == nproc and out["config"]["parallelism"].startswith(f"dp{nproc}")
    assert out["nccl"]["backend"] == "gloo" and out["nccl"]["world_size"] == nproc
    assert out["value"] > 0 and out["e2e"]["value"] > 0
    assert (out["gather"] is None) == zero2 and ("pushed" in out["step"]["path"]) == zero2
