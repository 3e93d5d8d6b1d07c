"""The C ABI used from C. tests/c_abi_client.c is compiled as strict C99
against include/zero_b200.h, linked against libzero_b200.so and run as a
separate process: it calls the host-side entry points (plan, plan queries,
memory accounting, zero_cpu_step, error reporting) and needs no GPU.
tests/c_gpu_client.c (GPU tests) runs whole fused steps with buffers from
cudaMalloc and no PyTorch in the process. Outputs are checked against the
oracle."""
import os
import shutil
import subprocess

import numpy as np
import pytest

import oracle as O
import zero_partitioned_mixed_reduce_b200 as Z

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
PKG = os.path.join(ROOT, "zero_partitioned_mixed_reduce_b200")


@pytest.fixture(scope="module")
def client(tmp_path_factory):
    if shutil.which("gcc") is None:
        pytest.skip("no C compiler")
    exe = str(tmp_path_factory.mktemp("cabi") / "c_abi_client")
    subprocess.run(["gcc", "-std=c99", "-pedantic", "-Wall", "-Wextra", "-Werror",
                    "-I", os.path.join(ROOT, "include"), os.path.join(ROOT, "tests", "c_abi_client.c"),
                    "-o", exe, "-L", PKG, "-lzero_b200", f"-Wl,-rpath,{PKG}"], check=True)
    return exe


def run(exe, *args):
    r = subprocess.run([exe, *map(str, args)], capture_output=True, text=True, timeout=120)
    assert r.returncode == 0, r.stderr
    return [line.split() for line in r.stdout.splitlines()]


@pytest.mark.parametrize("seed", range(6))
def test_plan_from_c_matches_oracle_layout(client, seed):
    rng = np.random.default_rng(seed)
    n = int(rng.integers(1, 40))
    numels = rng.integers(1, 5000, n).tolist()
    R = int(rng.choice([1, 2, 3, 8, 16, 64]))
    align = int(rng.choice([1, 8, 64]))
    bucket = int(rng.choice([0, 1, 3000, 20000]))
    dtype = int(rng.integers(0, 2))
    out = run(client, "plan", R, dtype, align, bucket, n, *numels)
    lay = O.Layout(numels, R, align, bucket)
    info = [int(x) for x in out[0][1:]]
    assert info == [lay.P, lay.L, lay.S, lay.T, n, len(lay.buckets), n]
    tensors = [[int(x) for x in row[1:]] for row in out if row[0] == "tensor"]
    assert [t[0] for t in tensors] == lay.offsets.tolist()
    assert [t[1] for t in tensors] == numels
    assert [t[2] for t in tensors] == lay.tensor_bucket.tolist()
    assert [t[3] for t in tensors] == list(range(n))
    buckets = [(int(r[1]), int(r[2])) for r in out if r[0] == "bucket"]
    layers = [(int(r[1]), int(r[2])) for r in out if r[0] == "layer"]
    assert buckets == lay.buckets and layers == lay.layers
    memory = {int(r[1]): int(r[2]) for r in out if r[0] == "memory"}
    for stage in range(4):
        assert memory[stage] == O.model_state_bytes(stage, lay.T, R)


@pytest.mark.parametrize("mode", ["cpu_step", "cpu_step_shard"])
@pytest.mark.parametrize("R,dtype", [(1, O.BF16), (4, O.FP16), (3, O.BF16)])
def test_cpu_step_from_c_matches_oracle(client, tmp_path, R, dtype, mode):
    # the whole CPU step, or the per-owner calls of a multi-process offload
    rng = np.random.default_rng(R * 7 + dtype)
    numels = [3001, 17, 4096]
    lay = O.Layout(numels, R, 8)
    S, P, idx = lay.S, lay.P, lay.flat_index()
    g = O.float_to_half(rng.normal(0, 1e-2, (R, P)).astype(np.float32), dtype)
    acc_u, _ = O.allreduce_sum(g, dtype)
    x = rng.normal(0, 0.02, P).astype(np.float32)
    st = O.State(x, dtype)

    def flat(a):
        f = np.zeros(lay.T, np.float32)
        f[idx] = a
        return f

    blob = np.concatenate([flat(acc_u), flat(x), np.zeros(lay.T, np.float32),
                           np.zeros(lay.T, np.float32)])
    fin, fout = tmp_path / "in.bin", tmp_path / "out.bin"
    blob.tofile(fin)
    out = run(client, mode, R, dtype, len(numels), *numels, fin, fout)
    fsm = O.make_fsm(O.SCALE_NONE)
    O.step(st, g, O.AdamW(1e-3, 0.9, 0.999, 1e-8, 0.01), fsm)
    state = out[0]
    assert state[0] == "state" and int(state[1]) == 1 and state[2:4] == ["0", "0"]
    assert abs(float(state[4]) - fsm.grad_norm_sq) <= 1e-12 * fsm.grad_norm_sq
    raw = np.fromfile(fout, np.uint8)
    f = raw[:12 * lay.T].view(np.float32).reshape(3, lay.T)
    param = raw[12 * lay.T:].view(np.uint16)
    for k, want in enumerate((st.master, st.m, st.v)):
        assert np.array_equal(f[k][idx].view(np.uint32), want.view(np.uint32))
    assert np.array_equal(param[idx], st.param)


def test_errors_from_c(client):
    out = run(client, "errors")
    err = {r[1]: (int(r[2]), " ".join(r[4:])) for r in out if r[0] == "error"}
    assert err["empty_list"][0] == Z.ZERO_ERR_INVALID_ARG
    assert err["zero_numel"][0] == Z.ZERO_ERR_INVALID_ARG
    assert err["too_many_ranks"][0] == Z.ZERO_ERR_INVALID_ARG
    assert err["bad_dtype"][0] == Z.ZERO_ERR_INVALID_ARG
    assert err["layer_gap"][0] == Z.ZERO_ERR_INVALID_ARG
    assert err["bucket_range"][0] == Z.ZERO_ERR_RANGE
    assert err["layer_range"][0] == Z.ZERO_ERR_RANGE
    assert err["memory_stage"][0] == Z.ZERO_ERR_INVALID_ARG
    assert err["ctx_null"][0] == Z.ZERO_OK
    for k in ("empty_list", "bucket_range", "memory_stage"):
        assert err[k][1].startswith("zero_plan")
    version = [r for r in out if r[0] == "version"][0]
    assert "sm_100a" in " ".join(version[1:])


@pytest.fixture(scope="module")
def gpu_client(tmp_path_factory):
    cuda = os.environ.get("CUDA_HOME", "/usr/local/cuda")
    exe = str(tmp_path_factory.mktemp("cgpu") / "c_gpu_client")
    subprocess.run(["gcc", "-std=c99", "-Wall", "-Wextra", "-Werror", "-I", os.path.join(ROOT, "include"),
                    "-I", os.path.join(cuda, "include"), os.path.join(ROOT, "tests", "c_gpu_client.c"),
                    "-o", exe, "-L", PKG, "-lzero_b200", "-L", os.path.join(cuda, "lib64"), "-lcudart",
                    f"-Wl,-rpath,{PKG}", f"-Wl,-rpath,{os.path.join(cuda, 'lib64')}"], check=True)
    return exe


@pytest.mark.gpu
@pytest.mark.parametrize("R,dtype,mode", [(4, O.FP16, O.SCALE_DYNAMIC), (2, O.BF16, O.SCALE_NONE),
                                          (8, O.FP16, O.SCALE_STATIC)])
def test_gpu_step_from_c_matches_oracle(gpu_client, tmp_path, R, dtype, mode):
    # the whole GPU step driven from C: cudaMalloc'd buffers, no PyTorch
    rng = np.random.default_rng(R * 3 + mode)
    numels = [3001, 17, 4096, 70_001]
    lay = O.Layout(numels, R, 8)
    T, P, idx = lay.T, lay.P, lay.flat_index()
    steps, init, interval = 4, 256.0, 2
    x = rng.normal(0, 0.02, P).astype(np.float32)
    st = O.State(x, dtype)
    fsm = O.make_fsm(mode, scale=init if mode != O.SCALE_NONE else 1.0, interval=interval)
    hp = O.AdamW(1e-3, 0.9, 0.999, 1e-8, 0.01)
    master = np.zeros(T, np.float32)
    master[idx] = x
    param = np.zeros(T, np.uint16)
    param[idx] = st.param
    blobs = [np.array([len(numels), R, dtype, mode, steps, interval], np.int64).tobytes(),
             np.float32(init).tobytes(), np.array(numels, np.int64).tobytes(), master.tobytes(),
             param.tobytes()]
    for s in range(steps):
        scale = fsm.scale if mode != O.SCALE_NONE else 1.0
        g = O.float_to_half((rng.normal(0, 1e-2, (R, P)) * scale).astype(np.float32), dtype)
        if s == 2:
            g[R - 1, 11] = 0x7C00 if dtype == O.FP16 else 0x7F80
        gp = np.zeros((R, T), np.uint16)
        gp[:, idx] = g
        blobs.append(gp.tobytes())
        O.step(st, g, hp, fsm)
    fin, fout = tmp_path / "in.bin", tmp_path / "out.bin"
    fin.write_bytes(b"".join(blobs))
    r = subprocess.run([gpu_client, str(fin), str(fout)], capture_output=True, text=True, timeout=300)
    assert r.returncode == 0, r.stderr
    raw = fout.read_bytes()
    scale, cur = np.frombuffer(raw[:8], np.float32)[0], np.frombuffer(raw[4:8], np.int32)[0]
    good, t = np.frombuffer(raw[8:24], np.int64)
    last_overflow, last_skipped = np.frombuffer(raw[24:32], np.int32)
    norm = np.frombuffer(raw[32:40], np.float64)[0]
    assert (t, good, last_overflow, last_skipped) == (fsm.t, fsm.good, fsm.last_overflow, fsm.last_skipped)
    assert np.float32(scale) == np.float32(fsm.scale) and cur in (0, 1)
    assert abs(norm - fsm.grad_norm_sq) <= 1e-9 * abs(fsm.grad_norm_sq) or not np.isfinite(fsm.grad_norm_sq)
    body = np.frombuffer(raw[40:], np.uint8)
    f = body[:12 * T].view(np.float32).reshape(3, T)
    got_param = body[12 * T:].view(np.uint16)
    for k, want in enumerate((st.master, st.m, st.v)):
        a = f[k][idx]
        fin_ = np.isfinite(want)
        assert np.array_equal(np.isfinite(a), fin_)
        assert np.array_equal(a[fin_].view(np.uint32), want[fin_].view(np.uint32))
    nan = O.half_to_float(st.param, dtype) != O.half_to_float(st.param, dtype)
    assert np.array_equal(got_param[idx][~nan], st.param[~nan])
