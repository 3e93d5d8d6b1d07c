"""GPU parity: every kernel path against the CPU oracle on the same seeded
bytes, at sizes the oracle finishes in seconds that still span several
tiles and a ragged tail. Layout, overflow flags and skip decisions must be
bit-exact; fp32 master/m/v within 1e-5 relative and half params within one
ulp (the kernels are designed to match bit for bit, which is also checked).
"""
import numpy as np
import pytest
import torch

import oracle as O

pytestmark = pytest.mark.gpu

if torch.cuda.is_available():
    import zero_partitioned_mixed_reduce_b200 as Z
    from gpu_harness import Case, u16


def tensor_list(seed, big=False):
    rng = np.random.default_rng(seed)
    n = int(rng.integers(3, 9))
    sizes = rng.integers(1, 3000, n)
    sizes[0] = int(rng.choice([1, 7, 8, 9]))
    if big:
        sizes[-1] = 70_001  # many block passes and staged tiles, and a ragged tail
    return sizes.tolist()


PATHS = [("inplace", O.SCALE_NONE), ("inplace", O.SCALE_STATIC), ("pingpong", O.SCALE_NONE),
         ("pingpong", O.SCALE_DYNAMIC), ("twopass", O.SCALE_STATIC), ("twopass", O.SCALE_DYNAMIC),
         ("twopass_pp", O.SCALE_NONE), ("twopass_pp", O.SCALE_DYNAMIC)]


@pytest.mark.parametrize("R", [1, 2, 3, 4, 8, 16])
@pytest.mark.parametrize("dtype", [O.BF16, O.FP16])
@pytest.mark.parametrize("align", [1, 8])
@pytest.mark.parametrize("path,mode", PATHS)
def test_paths_match_oracle(R, dtype, align, path, mode):
    numels = tensor_list(R * 100 + dtype * 10 + align, big=(R in (3, 8)))
    init = 1024.0 if mode != O.SCALE_NONE else 1.0
    c = Case(numels, R, dtype, align, mode, init_scale=init, interval=2, path=path,
             bucket_elems=1500)
    try:
        for _ in range(3):
            c.step()
            c.compare()
    finally:
        c.close()


def inf_bits(dtype):
    return 0x7C00 if dtype == O.FP16 else 0x7F80


def nan_bits(dtype):
    return 0x7E00 if dtype == O.FP16 else 0x7FC0


@pytest.mark.parametrize("path", ["pingpong", "twopass", "twopass_pp"])
@pytest.mark.parametrize("dtype", [O.BF16, O.FP16])
@pytest.mark.parametrize("where", ["first", "last", "before_pad", "after_pad"])
@pytest.mark.parametrize("kind", ["inf", "nan"])
def test_overflow_skips_and_backs_off(path, dtype, where, kind):
    numels = [13, 8, 29, 4]  # align 8 leaves padding after tensors 0 and 2
    R = 4
    c = Case(numels, R, dtype, 8, O.SCALE_DYNAMIC, init_scale=256.0, interval=3, path=path)
    lay = c.lay
    ends = np.cumsum(numels)
    e = {"first": 0, "last": lay.P - 1, "before_pad": int(ends[0]) - 1,
         "after_pad": int(ends[0])}[where]
    bits = inf_bits(dtype) if kind == "inf" else nan_bits(dtype)
    try:
        c.step()
        c.compare()
        before = c.gpu_state()
        skipped = c.step(inject=[(R - 1, e, bits)])
        assert skipped
        f = c.gpu_fsm()
        assert f["last_overflow"] == 1 and f["last_skipped"] == 1
        assert f["scale"] == 128.0 and f["t"] == 1
        c.compare()
        after = c.gpu_state()
        for k in ("master", "m", "v", "param"):
            assert np.array_equal(before[k], after[k])
        for _ in range(3):  # recovers, then grows after 3 clean steps
            c.step()
            c.compare()
        assert c.gpu_fsm()["scale"] == 256.0
    finally:
        c.close()


@pytest.mark.parametrize("dtype", [O.BF16, O.FP16])
def test_static_overflow_reported_not_skipped(dtype):
    c = Case([100, 37], 2, dtype, 8, O.SCALE_STATIC, init_scale=4.0, path="inplace")
    try:
        c.step(inject=[(0, 5, inf_bits(dtype))])
        f = c.gpu_fsm()
        assert f["last_overflow"] == 1 and f["last_skipped"] == 0 and f["t"] == 1
        c.compare()
    finally:
        c.close()


def test_bf16_sum_overflow_is_overflow():
    # two finite bf16 values whose fp32 sum is +inf
    big = int(O.float_to_half(np.array([3.0e38], np.float32), O.BF16)[0])
    c = Case([40], 2, O.BF16, 8, O.SCALE_DYNAMIC, init_scale=1.0, path="twopass")
    try:
        c.step(inject=[(0, 9, big), (1, 9, big)])
        f = c.gpu_fsm()
        assert f["last_overflow"] == 1 and f["last_skipped"] == 1
        c.compare()
    finally:
        c.close()


@pytest.mark.parametrize("align", [1, 8])
@pytest.mark.parametrize("bucket", [1, 7, 64, 333, 0])
def test_buckets_crossing_shards(align, bucket):
    # small buckets over a list whose shards cut through tensors
    numels = [5, 300, 1, 77, 640, 9, 123, 2]
    c = Case(numels, 8, O.FP16, align, O.SCALE_DYNAMIC, init_scale=64.0, path="twopass",
             bucket_elems=bucket)
    S = c.plan.S
    crossing = [b for b in c.plan.buckets if b[0] // S != (b[1] - 1) // S]
    if bucket in (333, 0):
        assert crossing
    try:
        for _ in range(2):
            c.step()
            c.compare()
    finally:
        c.close()


@pytest.mark.parametrize("align", [1, 8])
@pytest.mark.parametrize("path", ["pingpong", "inplace"])
def test_gather_layers(align, path):
    numels = [3001, 17, 8, 2048, 5, 700, 1]
    layer_ids = [0, 0, 1, 1, 2, 2, 3]
    c = Case(numels, 4, O.BF16, align, O.SCALE_NONE, path=path, layer_ids=layer_ids)
    try:
        for _ in range(2):
            c.step()
        c.compare()
        st = c.ostate
        # oracle params placed at their padded positions, padding zero
        flat = np.zeros(c.plan.T, np.uint16)
        flat[c.idx] = st.param
        for l, (lo, hi) in enumerate(c.lay.layers):
            out = torch.full((hi - lo + 8,), -1, dtype=torch.int16, device="cuda")
            Z.zero_gather_layer(c.ctx, l, c.handle, out)
            got = u16(out)
            assert np.array_equal(got[:hi - lo], flat[lo:hi]), l
            assert np.all(got[hi - lo:] == 0xFFFF)  # nothing written past the layer
    finally:
        c.close()


@pytest.mark.parametrize("align", [1, 8])
@pytest.mark.parametrize("R", [1, 3, 8])
def test_bucketed_gather_matches_oracle_and_single_gathers(align, R):
    numels = [3001, 17, 8, 2048, 5, 700, 1, 9000, 64, 3]
    layer_ids = [0, 0, 1, 1, 2, 2, 3, 4, 5, 5]
    c = Case(numels, R, O.FP16, align, O.SCALE_DYNAMIC, 64.0, path="pingpong", layer_ids=layer_ids)
    try:
        for _ in range(2):
            c.step()
        c.compare()
        flat = np.zeros(c.plan.T, np.uint16)
        flat[c.idx] = c.ostate.param
        L = c.lay.layers
        for first, count in ((0, len(L)), (1, 3), (4, 2), (5, 1), (2, 1)):
            outs = [torch.full((L[l][1] - L[l][0] + 8,), -1, dtype=torch.int16, device="cuda")
                    for l in range(first, first + count)]
            Z.zero_gather_layers(c.ctx, first, outs, c.handle)
            for i, l in enumerate(range(first, first + count)):
                lo, hi = L[l]
                got = u16(outs[i])
                assert np.array_equal(got[:hi - lo], flat[lo:hi]), (first, count, l)
                assert np.all(got[hi - lo:] == 0xFFFF)
                single = torch.empty(hi - lo, dtype=torch.int16, device="cuda")
                Z.zero_gather_layer(c.ctx, l, c.handle, single)
                assert np.array_equal(u16(single), got[:hi - lo])
        with pytest.raises(Z.ZeroError) as e:
            Z.zero_gather_layers(c.ctx, 4, [outs[0]] * 3, c.handle)
        assert e.value.status == 5
    finally:
        c.close()


def test_deterministic_bit_for_bit():
    runs = []
    for _ in range(2):
        c = Case([70_001, 3, 999], 8, O.FP16, 8, O.SCALE_DYNAMIC, init_scale=512.0,
                 path="pingpong")
        try:
            for _ in range(3):
                c.step()
            s = c.gpu_state()
            runs.append((s, c.gpu_fsm()))
        finally:
            c.close()
    (a, fa), (b, fb) = runs
    assert fa == fb
    for k in ("master", "m", "v", "param"):
        assert np.array_equal(np.asarray(a[k]).view(np.uint8), np.asarray(b[k]).view(np.uint8))


@pytest.mark.parametrize("path", ["pingpong", "twopass", "twopass_pp"])
def test_checkpoint_resume(path):
    numels = [1000, 33, 4097]
    straight = Case(numels, 4, O.FP16, 8, O.SCALE_DYNAMIC, 32.0, interval=2, path=path)
    resumed = Case(numels, 4, O.FP16, 8, O.SCALE_DYNAMIC, 32.0, interval=2, path=path)
    try:
        for _ in range(5):
            straight.step()
        for _ in range(3):
            resumed.step()
        # save: the loss-scale state and the current set's buffers
        saved = Z.zero_loss_scale(resumed.ctx)
        k = saved["cur"] if resumed.sets == 2 else 0
        bufs = [[t.clone() for t in getattr(resumed, f)[k]] for f in ("master", "m", "v", "param")]
        # restore into a fresh context, with the model in set 0
        Z.zero_ctx_destroy(resumed.ctx)
        resumed.ctx = Z.zero_ctx_create(resumed.plan.handle, O.SCALE_DYNAMIC, 32.0, 2)
        for f, b in zip(("master", "m", "v", "param"), bufs):
            for dst, src in zip(getattr(resumed, f)[0], b):
                dst.copy_(src)
        saved["cur"] = 0
        Z.zero_loss_scale(resumed.ctx, Z.ZERO_LOSS_SCALE_SET, saved)
        for _ in range(2):
            resumed.step()
        a, b = straight.gpu_state(), resumed.gpu_state()
        for f in ("master", "m", "v", "param"):
            assert np.array_equal(np.asarray(a[f]).view(np.uint8), np.asarray(b[f]).view(np.uint8))
        fa, fb = Z.zero_loss_scale(straight.ctx), Z.zero_loss_scale(resumed.ctx)
        for key in ("scale", "good", "t", "grad_norm_sq"):
            assert fa[key] == fb[key]
        resumed.compare()
    finally:
        straight.close()
        resumed.close()


def test_argument_errors():
    c = Case([100, 50], 2, O.BF16, 8, O.SCALE_DYNAMIC, 4.0, path="pingpong")
    try:
        with pytest.raises(Z.ZeroError) as e:
            Z.zero_reduce_scatter_bucket(c.ctx, 99, c.grads, c.master[0])
        assert e.value.status == 5  # range
        bad = [g[1:] for g in c.grads]  # 2-byte offset: not 16-byte aligned
        with pytest.raises(Z.ZeroError) as e:
            Z.zero_step(c.ctx, c.hp, c.handle, bad)
        assert e.value.status == 2  # align
        one_set = Z.StateHandle([dict(master=c.master[0], m=c.m[0], v=c.v[0],
                                      param=c.param[0])])
        with pytest.raises(Z.ZeroError) as e:  # DYNAMIC fused needs two sets
            Z.zero_step(c.ctx, c.hp, one_set, c.grads)
        assert e.value.status == 1
        with pytest.raises(Z.ZeroError) as e:
            Z.zero_gather_layer(c.ctx, 7, c.handle, c.grads[0])
        assert e.value.status == 5
        c.step()
        c.compare()
        with pytest.raises(Z.ZeroError) as e:  # after a ping-pong step, one set is not enough
            Z.zero_gather_layer(c.ctx, 0, one_set, c.grads[0])
        assert e.value.status == 7
        with pytest.raises(Z.ZeroError):
            Z.zero_loss_scale(c.ctx, Z.ZERO_LOSS_SCALE_SET, dict(scale=-1.0, cur=0, t=0, good=0))
    finally:
        c.close()


@pytest.mark.parametrize("R", [5, 7, 32, 64])
@pytest.mark.parametrize("path,mode", [("inplace", O.SCALE_NONE), ("pingpong", O.SCALE_DYNAMIC),
                                       ("twopass", O.SCALE_STATIC)])
def test_many_ranks_match_oracle(R, path, mode):
    # the runtime-R kernels, up to the ABI's maximum of 64 ranks, where most
    # shards are short and several are pure padding
    numels = tensor_list(R * 7 + len(path), big=(R == 7))
    init = 1024.0 if mode != O.SCALE_NONE else 1.0
    c = Case(numels, R, O.FP16, 8, mode, init_scale=init, interval=2, path=path, bucket_elems=2000)
    try:
        for _ in range(3):
            c.step()
            c.compare()
    finally:
        c.close()


@pytest.mark.parametrize("R", [1, 2, 8, 64])
@pytest.mark.parametrize("path", ["inplace", "pingpong", "twopass"])
def test_single_parameter_model(R, path):
    # P = 1: one real element, the rest of every shard is padding
    mode = O.SCALE_DYNAMIC if path == "pingpong" else O.SCALE_NONE
    c = Case([1], R, O.BF16, 8, mode, init_scale=8.0, interval=2, path=path)
    try:
        for _ in range(3):
            c.step()
            c.compare()
        assert c.plan.T == 8 * R
    finally:
        c.close()
