"""The benchmark's multi-rank path on CPU with gloo, world size 2: the
routing (N > 1 runs the sharded step), the whole-job aggregation (max of the
per-rank times, sum of the units) as the sharded step reports it, and the
reference arm under torch.distributed.run (rank 0 alone works and prints)."""
import datetime
import json
import multiprocessing as mp
import os
import socket
import subprocess
import sys


ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _worker(rank, world, port, q):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), RANK=str(rank),
                      WORLD_SIZE=str(world), LOCAL_RANK=str(rank))
    sys.path.insert(0, ROOT)
    import torch.distributed as dist
    import bench
    dist.init_process_group("gloo", rank=rank, world_size=world,
                            timeout=datetime.timedelta(seconds=60))
    try:
        ms, units = bench.aggregate(10.0 + rank, 100.0 * (rank + 1), world)
        bench.barrier(world)
        # the sharded step: every rank counts its P / N share of each of K
        # steps; the job's rate is P * K over the slowest rank's time
        args = bench.parse_args(["--gpus", str(world), "--steps", "7"])
        mode = bench.choose_mode(args, world)
        P, K = 1000, args.steps
        dms, dunits = bench.aggregate(5.0 * (rank + 1), float(P) * K / world, world)
        q.put((rank, ms, units, mode, dms, dunits))
    finally:
        dist.destroy_process_group()


def test_aggregate_max_time_sum_units_gloo():
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = free_port()
    procs = [ctx.Process(target=_worker, args=(r, 2, port, q)) for r in range(2)]
    for p in procs:
        p.start()
    for p in procs:
        p.join(120)
        assert p.exitcode == 0
    got = sorted(q.get(timeout=10) for _ in range(2))
    for rank, ms, units, mode, dms, dunits in got:
        assert ms == 11.0 and units == 300.0
        assert mode == "dist" and dms == 10.0 and dunits == 7000.0


def test_reference_arm_under_torchrun_two_ranks():
    env = dict(os.environ, CUDA_VISIBLE_DEVICES="")
    cmd = [sys.executable, "-m", "torch.distributed.run", "--nnodes=1", "--nproc-per-node=2",
           "--master-addr", "127.0.0.1", "--master-port", str(free_port()),
           os.path.join(ROOT, "bench.py"), "--impl", "reference", "--gpus", "2",
           "--steps", "1", "--warmup", "0"]
    r = subprocess.run(cmd, capture_output=True, text=True, timeout=600, env=env, cwd=ROOT)
    assert r.returncode == 0, r.stderr[-2000:]
    lines = [l for l in r.stdout.splitlines() if l.startswith("{")]
    assert len(lines) == 1  # rank 0 alone prints
    out = json.loads(lines[0])
    assert out["impl"] == "reference" and out["n_gpus"] == 2 and out["value"] > 0
    assert out["e2e"]["h2d_bytes_per_step"] == 0 and out["cpu_baseline"]["kind"] == "oracle"
    # the same `config` as the GPU arm of the same command line: the sharded
    # job over two ranks, its layout from the library's plan
    import bench
    import synth
    import zero_partitioned_mixed_reduce_b200 as Z
    args = bench.parse_args(["--gpus", "2"])
    wl = synth.workload(args.workload)
    plan = Z.Plan(wl["numels"], wl["layer_ids"], 2, wl["dtype"], 8, 0)
    assert out["config"] == bench.job_config(args, 2, wl, 2, plan.T, plan.S, len(plan.layers), True)
    assert out["config"]["parallelism"].startswith("dp2") and out["scaling"] == "strong"
