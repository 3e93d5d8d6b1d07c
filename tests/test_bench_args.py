"""bench.py's command line: the defaults the benchmark contract relies on."""
import bench


def test_defaults():
    a = bench.parse_args([])
    # the largest configuration that fits one GPU: the Llama-style 3B list, R = 4
    assert a.gpus == 1 and a.impl == "ours" and a.workload == "llama3b"
    assert a.warmup >= 3 and a.steps >= 1
    assert a.graph is True  # CUDA-graph replay of the captured step by default
    assert a.clip_norm == "rs"


def test_eager_and_graph_flags():
    assert bench.parse_args(["--eager"]).graph is False
    assert bench.parse_args(["--graph"]).graph is True


def test_workload_label_names_the_sizes():
    import synth
    wl = synth.workload("gpt2s")
    label = bench.workload_label("gpt2s", wl)
    assert "P=124439808" in label and "R=8" in label and "fp16" in label


def test_oracle_crew_runs_the_oracle_on_several_processes():
    # the all-core CPU baseline: spawned single-threaded oracle processes,
    # timed between a common barrier and the last end
    crew = bench.OracleCrew("tiny", 4096, procs=2)
    try:
        rate, sec = crew.run(1)
    finally:
        crew.close()
    assert rate > 0 and sec > 0 and crew.procs == 2


def test_mode_routing():
    # one GPU: the single-GPU step; N > 1: the sharded step over the job's
    # GPUs unless --replicas asks for independent copies
    p = bench.parse_args
    assert bench.choose_mode(p([]), 1) == "single"
    assert bench.choose_mode(p(["--gpus", "8"]), 8) == "dist"
    assert bench.choose_mode(p(["--gpus", "8", "--replicas"]), 8) == "single"
    assert bench.choose_mode(p(["--dist"]), 1) == "dist"
    assert bench.choose_mode(p(["--impl", "reference", "--gpus", "4"]), 4) == "reference"
    assert bench.choose_mode(p(["--rs-sweep"]), 1) == "rs_sweep"


def test_bucket_runs_cover_every_bucket_once_in_order():
    buckets = [(90, 100), (60, 90), (59, 60), (10, 59), (0, 10)]  # reverse flat order
    for group in (0, 1, 10, 31, 40, 1000):
        runs = bench.bucket_runs(buckets, group)
        covered = [b for first, count in runs for b in range(first, first + count)]
        assert covered == list(range(len(buckets)))
        for first, count in runs:
            n = sum(hi - lo for lo, hi in buckets[first:first + count])
            assert count == 1 or n <= group
    assert bench.bucket_runs(buckets, 0) == [(b, 1) for b in range(5)]
    assert bench.bucket_runs(buckets, 1000) == [(0, 5)]
    assert bench.bucket_runs(buckets, 40) == [(0, 2), (2, 1), (3, 1), (4, 1)]
    assert bench.bucket_runs(buckets, 60) == [(0, 3), (3, 2)]


def test_dist_bytes_and_roofline():
    T, N = 8 * 1000, 4
    S = T // N
    nb = bench.dist_step_bytes(T, S, N)
    assert nb["step_hbm"] == (2 * N + 26) * S and nb["nvlink_step"] == 2 * (N - 1) * S
    assert nb["gather_hbm"] == 2 * N * S + 2 * T and nb["nvlink_gather"] == 2 * (N - 1) * S
    # NVLink-bound when its bytes take longer at 770 GB/s than the HBM bytes at peak
    r = bench.dist_roofline({"hbm": 1e9, "nvlink": 1e9}, 2.0, 6000.0)
    assert r["bound"] == "nvlink" and abs(r["achieved"] - 500.0) < 1e-9
    assert abs(r["frac"] - 500.0 / bench.NVLINK_PEER_GBS) < 1e-12
    r = bench.dist_roofline({"hbm": 6e9, "nvlink": 0}, 1.0, 6000.0)
    assert r["bound"] == "hbm" and abs(r["frac"] - 1.0) < 1e-12


def test_tensor_range_selection():
    import synth
    a = bench.parse_args(["--tensors", "1:10"])
    assert a.tensor_range == (1, 10)
    assert bench.parse_args(["--first-tensors", "6"]).tensor_range == (0, 6)
    assert bench.parse_args([]).tensor_range is None
    wl = bench.restrict(synth.workload("llama3b"), (1, 10))
    # one decoder layer of the Llama-style list: norms, q/k/v/o, gate/up/down
    assert len(wl["numels"]) == 9 and sum(wl["numels"]) == 100_669_440
    assert wl["layer_ids"] == [0] * 9


def test_dist_bytes_with_the_parameter_push():
    T, N = 8 * 1000, 4
    S = T // N
    nb = bench.dist_step_bytes(T, S, N, push=True)
    assert nb["gather_hbm"] == 0 and nb["nvlink_gather"] == 0
    assert nb["step_hbm"] == (2 * N + 26) * S + 2 * T
    assert nb["nvlink_step"] == 4 * (N - 1) * S
    assert bench.parse_args(["--zero2"]).zero2 and not bench.parse_args([]).zero2


def test_reference_arm_reports_the_gpu_arms_config():
    # one GPU: the reference arm's `config` (from the oracle's layout) equals
    # the one the GPU arm builds from the library's plan
    import json
    import os
    import subprocess
    import sys
    import synth
    import zero_partitioned_mixed_reduce_b200 as Z
    root = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
    env = dict(os.environ, CUDA_VISIBLE_DEVICES="")
    r = subprocess.run([sys.executable, os.path.join(root, "bench.py"), "--impl", "reference", "--workload", "tiny",
                        "--steps", "1", "--warmup", "0"], capture_output=True, text=True, timeout=600, env=env,
                       cwd=root)
    assert r.returncode == 0, r.stderr[-2000:]
    out = json.loads([ln for ln in r.stdout.splitlines() if ln.startswith("{")][-1])
    args = bench.parse_args(["--workload", "tiny"])
    wl = synth.workload("tiny")
    plan = Z.Plan(wl["numels"], wl["layer_ids"], wl["R"], wl["dtype"], 8, wl["bucket_elems"])
    assert out["config"] == bench.job_config(args, 1, wl, wl["R"], plan.T, plan.S, len(plan.layers), False)
    assert out["config"]["parallelism"] == "1 GPU" and out["scaling"] == "weak"
