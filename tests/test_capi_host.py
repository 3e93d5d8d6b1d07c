"""Host-side checks of libzero_b200.so that need no GPU: the library loads
and exports every function include/zero_b200.h declares, the partition plan
matches the oracle's own layout bit for bit, plan errors return the right
status codes, and no GPU call pretends to succeed without a GPU."""
import ctypes
import os
import re
import subprocess

import numpy as np
import pytest
import torch

import oracle as O
import zero_partitioned_mixed_reduce_b200 as Z
from zero_partitioned_mixed_reduce_b200 import _capi
import synth

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def declared_functions():
    text = open(os.path.join(ROOT, "include", "zero_b200.h")).read()
    text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
    return sorted(set(re.findall(r"\b(zero_[a-z_]+)\s*\(", text)))


def test_exports_every_declared_function():
    names = declared_functions()
    assert len(names) >= 15
    lib = ctypes.CDLL(Z.LIB_PATH)
    missing = [n for n in names if not hasattr(lib, n)]
    assert not missing, missing
    nm = subprocess.run(["nm", "-D", "--defined-only", Z.LIB_PATH], capture_output=True,
                        text=True).stdout
    exported = set(re.findall(r" T (zero_\w+)", nm))
    assert set(names) <= exported


def test_version_and_error_buffer():
    assert "sm_100a" in Z.zero_version()
    with pytest.raises(Z.ZeroError):
        Z.zero_plan([], None, 2)
    assert "at least one tensor" in Z.zero_last_error()


def compare_plan(numels, R, align, bucket, layer_ids):
    lay = O.Layout(numels, R, align, bucket, layer_ids)
    p = Z.Plan(numels, layer_ids, R, Z.ZERO_FP16, align, bucket)
    assert (p.P, p.L, p.S, p.T) == (lay.P, lay.L, lay.S, lay.T)
    assert p.offsets == lay.offsets.tolist()
    assert p.buckets == lay.buckets
    assert p.layers == lay.layers
    for k in range(len(numels)):
        off, n, b, l = Z.zero_plan_tensor(p.handle, k)
        assert (off, n, b) == (lay.offsets[k], numels[k], lay.tensor_bucket[k])
    for stage in range(4):
        assert Z.zero_plan_memory(p.handle, stage) == O.model_state_bytes(stage, p.T, R)


@pytest.mark.parametrize("seed", range(200))
def test_plan_matches_oracle_layout_random(seed):
    rng = np.random.default_rng(1000 + seed)
    n = int(rng.integers(1, 30))
    numels = rng.integers(1, 500, n).tolist()
    R = int(rng.integers(1, 65))
    align = int(rng.choice([1, 2, 8, 16, 100]))
    bucket = int(rng.choice([-1, 0, 1, 64, 700, 5000]))
    steps = rng.integers(0, 2, n)
    steps[0] = 0
    layer_ids = np.cumsum(steps).tolist() if rng.random() < 0.7 else None
    compare_plan(numels, R, align, bucket, layer_ids)


@pytest.mark.parametrize("name", synth.WORKLOADS)
def test_plan_matches_oracle_layout_workloads(name):
    wl = synth.workload(name)
    compare_plan(wl["numels"], wl["R"], 8, wl["bucket_elems"], wl["layer_ids"])


def test_workload_shapes():
    # parameter counts of the model families the workloads are named after
    w = synth.workload("gpt2s")
    assert sum(w["numels"]) == 124_439_808 and len(w["numels"]) == 148  # GPT-2 small, tied head
    w = synth.workload("d1p3b")
    assert sum(w["numels"]) == 1_315_723_264 and len(w["numels"]) == 292
    w = synth.workload("llama3b")
    assert sum(w["numels"]) == 3_606_752_256 and len(w["numels"]) == 255
    w = synth.workload("tiny")
    assert sum(w["numels"]) == 1_037_800
    for name, R in (("irr_r16", 16), ("irr_r2", 2)):
        w = synth.workload(name)
        assert len(w["numels"]) == 10_000 and sum(w["numels"]) % R != 0
        assert min(w["numels"]) >= 1 and max(w["numels"]) <= (1 << 22) or name == "irr_r16"
    assert abs(sum(synth.workload("irr_r16")["numels"]) - 256e6) < 1e6
    assert 2.3e9 < sum(synth.workload("irr_r2")["numels"]) < 3.2e9


def test_cfg1_worked_plan():
    p = Z.Plan([1024 * 512, 512, 512 * 1000, 1000], [0, 0, 1, 1], R=4)
    assert (p.S, p.T) == (259_456, 1_037_824)
    assert p.buckets == [(0, 1_037_824)]


@pytest.mark.parametrize("kw,status", [
    (dict(numels=[], R=2), _capi.ZERO_ERR_INVALID_ARG),
    (dict(numels=[4, 0], R=2), _capi.ZERO_ERR_INVALID_ARG),
    (dict(numels=[4], R=0), _capi.ZERO_ERR_INVALID_ARG),
    (dict(numels=[4], R=65), _capi.ZERO_ERR_INVALID_ARG),
    (dict(numels=[4], R=2, tensor_align=0), _capi.ZERO_ERR_INVALID_ARG),
    (dict(numels=[4], R=2, dtype=7), _capi.ZERO_ERR_INVALID_ARG),
    (dict(numels=[4, 4], R=2, layer_ids=[1, 1]), _capi.ZERO_ERR_INVALID_ARG),
    (dict(numels=[4, 4, 4], R=2, layer_ids=[0, 2, 2]), _capi.ZERO_ERR_INVALID_ARG),
    (dict(numels=[1 << 34, 1 << 34], R=1), _capi.ZERO_ERR_RANGE),
])
def test_plan_errors(kw, status):
    args = dict(layer_ids=None, R=1, dtype=Z.ZERO_BF16, tensor_align=8, bucket_elems=0)
    args.update(kw)
    numels = args.pop("numels")
    with pytest.raises(Z.ZeroError) as e:
        Z.zero_plan(numels, args["layer_ids"], args["R"], args["dtype"], args["tensor_align"],
                    args["bucket_elems"])
    assert e.value.status == status


def test_queries_out_of_range():
    p = Z.Plan([10, 20], None, R=2)
    for f, i in ((Z.zero_plan_tensor, 2), (Z.zero_plan_bucket, 1), (Z.zero_plan_layer, 2)):
        with pytest.raises(Z.ZeroError) as e:
            f(p.handle, i)
        assert e.value.status == _capi.ZERO_ERR_RANGE
    with pytest.raises(Z.ZeroError):
        Z.zero_plan_memory(p.handle, 4)


@pytest.mark.skipif(torch.cuda.is_available(), reason="checks the no-GPU failure mode")
def test_no_gpu_fails_loudly():
    p = Z.Plan([10, 20], None, R=2)
    with pytest.raises(Z.ZeroError) as e:
        Z.zero_ctx_create(p.handle)
    assert e.value.status == _capi.ZERO_ERR_CUDA


def test_release_build_carries_no_bounds_checks():
    # the bounds-checking build is a separate test library; the release
    # build reports -1 without touching a GPU
    import os
    import zero_partitioned_mixed_reduce_b200 as Z
    if os.environ.get("ZERO_B200_LIB"):
        pytest.skip("another build is loaded")
    assert Z.zero_debug_bounds() == (-1, 0, 0)


@pytest.mark.parametrize("seed", range(6))
def test_pack_places_tensors_at_the_oracle_offsets(seed):
    # the host marshalling (Plan.pack / unpack) against the oracle's own layout
    import torch
    rng = np.random.default_rng(300 + seed)
    n = int(rng.integers(1, 12))
    numels = rng.integers(1, 300, n).tolist()
    R = int(rng.integers(1, 9))
    align = int(rng.choice([1, 8]))
    plan = Z.Plan(numels, None, R, Z.ZERO_BF16, align, 0)
    lay = O.Layout(numels, R, align)
    x = torch.from_numpy(rng.normal(0, 1, sum(numels)).astype(np.float32))
    packed = plan.pack(x, fill=-7.0)
    assert packed.numel() == lay.T
    idx = lay.flat_index()
    assert np.array_equal(packed.numpy()[idx], x.numpy())
    pad = np.ones(lay.T, bool)
    pad[idx] = False
    assert np.all(packed.numpy()[pad] == -7.0)
    assert torch.equal(plan.unpack(packed), x)


def test_every_declared_function_has_a_binding_of_the_same_name():
    hdr = open(os.path.join(os.path.dirname(os.path.dirname(os.path.abspath(__file__))), "include",
                            "zero_b200.h")).read()
    names = sorted(set(re.findall(r"^\w[\w\s\*]*?\b(zero_\w+)\s*\(", hdr, re.M)))
    assert len(names) >= 40
    assert [n for n in names if not callable(getattr(Z, n, None))] == []


@pytest.mark.parametrize("R,P", [(1, (1 << 32) + 8), (2, (1 << 33) + 24), (1, 5), (2, 4097)])
def test_staged_step_tiles_cover_long_shards(R, P):
    # shards of 2^32 + 8 and more elements (R = 1 at 34 GB of half gradients,
    # R = 2 at 8.6 G params): the staged step's tiles, in 64-bit arithmetic,
    # cover every element of every shard; host only, nothing is allocated
    p = Z.Plan([P], None, R, 0, 8, 0)
    tile, tps, total = Z.zero_plan_step_tiles(p.handle)
    assert tile == 4096 and total == R * tps
    assert (tps - 1) * tile < p.S <= tps * tile
    last = p.S - (tps - 1) * tile
    assert 8 <= last <= tile and last % 8 == 0
    if P == (1 << 32) + 8:
        assert p.S == (1 << 32) + 8 and tps == (1 << 20) + 1 and last == 8


def test_ipc_argument_errors_without_a_device():
    # the checks that need no GPU: a NULL buffer, an offset outside the
    # exported allocation, closing a handle that was never opened
    with pytest.raises(Z.ZeroError) as e:
        Z.zero_ipc_export(0)
    assert e.value.status == Z.ZERO_ERR_INVALID_ARG
    blob = bytes(64) + (4096).to_bytes(8, "little") + (4096).to_bytes(8, "little")
    with pytest.raises(Z.ZeroError) as e:
        Z.zero_ipc_open(blob)
    assert e.value.status == Z.ZERO_ERR_RANGE
    with pytest.raises(Z.ZeroError) as e:
        Z.zero_ipc_close(bytes(80))
    assert e.value.status == Z.ZERO_ERR_STATE
