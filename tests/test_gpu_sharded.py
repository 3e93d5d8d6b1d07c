"""The per-rank step of a multi-GPU ZeRO run, emulated in one process:
zero_step_shard / zero_step_shard_ex over each owner range (no kernel waits
on another; the launches simply follow each other), the per-range totals
summed as the cross-rank all-reduce would, then zero_step_commit. The
two-pass variant reduce-scatters each range's part of every bucket with
zero_reduce_scatter_shard (with accumulation over micro-batches), and
clipping sums the ranges' zero_grad_norm_shard partials first. The result
must equal the oracle bit for bit (the gradient norm within its
summation-order bound)."""
import numpy as np
import pytest
import torch

import oracle as O

pytestmark = pytest.mark.gpu

if torch.cuda.is_available():
    import zero_partitioned_mixed_reduce_b200 as Z
    from gpu_harness import Case


def one_per_rank(R):
    return [(o, o + 1) for o in range(R)]


@pytest.mark.parametrize("R", [1, 2, 3, 4, 8])
@pytest.mark.parametrize("dtype,mode,path", [(O.FP16, O.SCALE_DYNAMIC, "pingpong"),
                                              (O.BF16, O.SCALE_NONE, "inplace"),
                                              (O.BF16, O.SCALE_STATIC, "pingpong")])
def test_sharded_step_matches_oracle(R, dtype, mode, path):
    numels = [70_001, 13, 4096, 7, 999]
    c = Case(numels, R, dtype, 8, mode, init_scale=256.0, interval=2, path=path)
    try:
        for step in range(4):
            splits = one_per_rank(R) if step % 2 == 0 else [(0, (R + 1) // 2), ((R + 1) // 2, R)][: 1 if R == 1 else 2]
            c.step_sharded(splits)
            c.compare()
    finally:
        c.close()


def test_overflow_on_one_rank_skips_every_rank():
    R = 4
    c = Case([20_000, 300], R, O.FP16, 8, O.SCALE_DYNAMIC, init_scale=64.0, path="pingpong")
    try:
        c.step_sharded(one_per_rank(R))
        c.compare()
        before = c.gpu_state()
        # an inf in replica 2 at an element owned by the last shard
        e = c.lay.P - 5
        skipped, partials = c.step_sharded(one_per_rank(R), inject=[(2, e, 0x7C00)])
        assert skipped
        flags = [p[1] for p in partials]
        owner = int(c.idx[e]) // c.plan.S
        assert flags == [1.0 if o == owner else 0.0 for o in range(R)]
        c.compare()
        after = c.gpu_state()
        for k in ("master", "m", "v", "param"):
            assert np.array_equal(before[k], after[k])
    finally:
        c.close()


def test_shard_argument_errors():
    c = Case([1000], 2, O.FP16, 8, O.SCALE_DYNAMIC, 8.0, path="pingpong")
    part = torch.zeros(2, dtype=torch.float64, device="cuda")
    try:
        for lo, hi in ((1, 1), (-1, 1), (0, 3)):
            with pytest.raises(Z.ZeroError) as e:
                Z.zero_step_shard(c.ctx, c.hp, c.handle, c.grads, lo, hi, part)
            assert e.value.status == 5
        one = Z.StateHandle([dict(master=c.master[0], m=c.m[0], v=c.v[0], param=c.param[0])])
        with pytest.raises(Z.ZeroError) as e:  # dynamic needs ping-pong
            Z.zero_step_shard(c.ctx, c.hp, one, c.grads, 0, 1, part)
        assert e.value.status == 1
    finally:
        c.close()


SPLITS = {1: [[(0, 1)]], 2: [[(0, 1), (1, 2)], [(0, 2)]], 3: [[(0, 1), (1, 2), (2, 3)], [(0, 2), (2, 3)]],
          4: [[(0, 1), (1, 2), (2, 3), (3, 4)], [(0, 2), (2, 4)]],
          8: [[(o, o + 1) for o in range(8)], [(0, 3), (3, 8)]]}


@pytest.mark.parametrize("R", [1, 2, 3, 4, 8])
@pytest.mark.parametrize("path,mode,dtype", [("twopass_pp", O.SCALE_DYNAMIC, O.FP16),
                                             ("twopass", O.SCALE_NONE, O.BF16),
                                             ("twopass", O.SCALE_STATIC, O.FP16)])
@pytest.mark.parametrize("n_micro,divisor,clip", [(1, 1.0, 0.0), (2, 2.0, 0.0), (3, 3.0, 1e-3), (1, 1.0, 1e9)])
def test_sharded_two_pass_matches_oracle(R, path, mode, dtype, n_micro, divisor, clip):
    # multi-rank accumulation and clipping: per-range reduce-scatters into the
    # owners' accumulators, the norm summed across ranges, per-range steps
    c = Case([70_001, 13, 4096, 7, 999], R, dtype, 8, mode, init_scale=256.0, interval=2, path=path,
             bucket_elems=9000, seed=R * 5 + n_micro)
    try:
        for step in range(3):
            c.step_sharded_ex(SPLITS[R][step % len(SPLITS[R])], n_micro, divisor, clip)
            c.compare()
        if clip == 1e-3:
            assert c.ofsm.grad_norm_sq > 1e-4
    finally:
        c.close()


@pytest.mark.parametrize("R", [1, 2, 3, 4, 8])
@pytest.mark.parametrize("path,mode,dtype", [("twopass_pp", O.SCALE_DYNAMIC, O.FP16),
                                             ("twopass", O.SCALE_NONE, O.BF16)])
@pytest.mark.parametrize("n_micro,divisor,clip", [(1, 1.0, 1e-3), (3, 3.0, 1e-3), (2, 2.0, 1e9)])
def test_sharded_norm_from_the_reduce_scatters_matches_oracle(R, path, mode, dtype, n_micro, divisor, clip):
    # each range's last reduce-scatters take its norm share (ZERO_RS_NORM);
    # zero_grad_norm_shard sums the shares instead of reading the accumulator
    c = Case([70_001, 13, 4096, 7, 999], R, dtype, 8, mode, init_scale=256.0, interval=2, path=path,
             bucket_elems=9000, seed=R * 7 + n_micro)
    try:
        for step in range(3):
            c.step_sharded_ex(SPLITS[R][step % len(SPLITS[R])], n_micro, divisor, clip, rs_norm=True)
            c.compare()
    finally:
        c.close()


def test_sharded_norm_shares_refusals():
    c = Case([3000, 17, 2048], 2, O.BF16, 8, O.SCALE_NONE, path="twopass", bucket_elems=1000)
    nb = len(c.plan.buckets)
    part = torch.zeros(2, dtype=torch.float64, device="cuda")
    acc0 = [c.acc[0], None]
    try:
        # no shares yet
        with pytest.raises(Z.ZeroError) as e:
            Z.zero_grad_norm_shard(c.ctx, None, None, 0, 1, part)
        assert e.value.status == Z.ZERO_ERR_STATE
        for b in range(nb):
            Z.zero_reduce_scatter_shard(c.ctx, b, c.grads, acc0, 0, 1, Z.ZERO_RS_NORM)
        Z.zero_grad_norm_shard(c.ctx, None, None, 0, 1, part)  # current: accepted
        # another owner range, or another divisor: refused
        with pytest.raises(Z.ZeroError) as e:
            Z.zero_grad_norm_shard(c.ctx, None, None, 1, 2, part)
        assert e.value.status == Z.ZERO_ERR_STATE
        with pytest.raises(Z.ZeroError) as e:
            Z.zero_grad_norm_shard(c.ctx, None, None, 0, 1, part, 2.0)
        assert e.value.status == Z.ZERO_ERR_STATE
        # a range's shares never feed the whole-model step
        with pytest.raises(Z.ZeroError) as e:
            Z.zero_step_ex(c.ctx, c.hp, c.handle, None, 1.0, 1.0, flags=Z.ZERO_STEP_NORM_FROM_RS)
        assert e.value.status == Z.ZERO_ERR_STATE
        # a later reduce-scatter of a bucket without the flag makes it stale
        Z.zero_reduce_scatter_shard(c.ctx, 0, c.grads, acc0, 0, 1, 0)
        with pytest.raises(Z.ZeroError) as e:
            Z.zero_grad_norm_shard(c.ctx, None, None, 0, 1, part)
        assert e.value.status == Z.ZERO_ERR_STATE
    finally:
        c.close()


@pytest.mark.parametrize("R", [1, 2, 4, 8])
@pytest.mark.parametrize("path,mode", [("pingpong", O.SCALE_DYNAMIC), ("inplace", O.SCALE_NONE)])
@pytest.mark.parametrize("clip", [1e-3, 1e9])
def test_sharded_fused_clip_matches_oracle(R, path, mode, clip):
    c = Case([70_001, 13, 4096, 7, 999], R, O.FP16, 8, mode, init_scale=256.0, interval=2, path=path,
             seed=R + 40)
    try:
        for step in range(3):
            c.step_sharded_ex(SPLITS[R][step % len(SPLITS[R])], 1, 1.0, clip)
            c.compare()
    finally:
        c.close()


def test_sharded_two_pass_overflow_on_one_rank_skips_every_rank():
    R = 4
    c = Case([20_000, 300], R, O.FP16, 8, O.SCALE_DYNAMIC, init_scale=64.0, path="twopass_pp")
    try:
        c.step_sharded_ex(SPLITS[R][0], 2, 2.0, 0.5)
        c.compare()
        before = c.gpu_state()
        assert c.step_sharded_ex(SPLITS[R][0], 2, 2.0, 0.5, inject=[(1, 2, c.lay.P - 3, 0x7C00)])
        c.compare()
        after = c.gpu_state()
        for k in ("master", "m", "v", "param"):
            assert np.array_equal(before[k], after[k])
        c.step_sharded_ex(SPLITS[R][1], 1, 1.0, 0.0)
        c.compare()
    finally:
        c.close()


def test_sharded_ex_argument_errors():
    c = Case([1000], 2, O.BF16, 8, O.SCALE_NONE, path="twopass")
    try:
        part = torch.zeros(2, dtype=torch.float64, device="cuda")
        with pytest.raises(Z.ZeroError) as e:  # clipping without the global norm
            Z.zero_step_shard_ex(c.ctx, c.hp, c.handle, None, 0, 1, part, 1.0, 1.0, None)
        assert e.value.status == Z.ZERO_ERR_INVALID_ARG
        with pytest.raises(Z.ZeroError) as e:  # both sources for the norm
            Z.zero_grad_norm_shard(c.ctx, c.grads, c.acc, 0, 1, part)
        assert e.value.status == Z.ZERO_ERR_INVALID_ARG
        with pytest.raises(Z.ZeroError) as e:
            Z.zero_reduce_scatter_shard(c.ctx, 0, c.grads, c.acc, 1, 1)
        assert e.value.status == Z.ZERO_ERR_RANGE
        with pytest.raises(Z.ZeroError) as e:  # an owned accumulator missing
            Z.zero_reduce_scatter_shard(c.ctx, -1, c.grads, [c.acc[0], None], 0, 2)
        assert e.value.status == Z.ZERO_ERR_INVALID_ARG
    finally:
        c.close()


@pytest.mark.parametrize("R", [1, 2, 4, 8])
@pytest.mark.parametrize("n_micro", [2, 3])
def test_sharded_fused_last_micro_batch_matches_oracle(R, n_micro):
    c = Case([70_001, 13, 4096, 7, 999], R, O.FP16, 8, O.SCALE_DYNAMIC, init_scale=256.0, interval=2,
             path="fused_acc", bucket_elems=9000, seed=R + 60)
    try:
        for step in range(3):
            c.step_sharded_ex(SPLITS[R][step % len(SPLITS[R])], n_micro, float(n_micro))
            c.compare()
    finally:
        c.close()
