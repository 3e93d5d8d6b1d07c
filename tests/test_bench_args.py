"""bench.py's command line: the defaults the benchmark contract relies on."""
import bench


def test_defaults():
    a = bench.parse_args([])
    assert a.gpus == 1 and a.impl == "ours" and a.workload == "gpt2s"
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
