"""GPU parity of gradient accumulation (reduce-scatter with ZERO_RS_ACCUMULATE
over micro-batches) and global-norm clipping (zero_step_ex, two-pass path)
against the oracle's oracle_step_ex on the same bytes."""
import numpy as np
import pytest
import torch

import oracle as O

pytestmark = pytest.mark.gpu

if torch.cuda.is_available():
    import zero_partitioned_mixed_reduce_b200 as Z
    from gpu_harness import Case


@pytest.mark.parametrize("R", [2, 3, 8])
@pytest.mark.parametrize("dtype", [O.BF16, O.FP16])
@pytest.mark.parametrize("n_micro,divisor", [(1, 1.0), (2, 2.0), (3, 3.0), (4, 1.0)])
@pytest.mark.parametrize("clip", [0.0, 1e-3, 1e9])
@pytest.mark.parametrize("path", ["twopass", "twopass_pp"])
def test_accumulate_and_clip_match_oracle(R, dtype, n_micro, divisor, clip, path):
    numels = [70_001, 13, 4096, 7, 999]
    mode = O.SCALE_DYNAMIC if dtype == O.FP16 else O.SCALE_NONE
    c = Case(numels, R, dtype, 8 if R != 3 else 1, mode, init_scale=256.0, interval=2,
             path=path, bucket_elems=5000)
    try:
        for _ in range(3):
            c.step_ex(n_micro, divisor, clip)
            c.compare()
        if clip == 1e-3:  # the clip was active: the norm is far above 1e-3
            assert c.ofsm.grad_norm_sq > 1e-4
    finally:
        c.close()


@pytest.mark.parametrize("micro", [0, 1, 2])
@pytest.mark.parametrize("path", ["twopass", "twopass_pp"])
def test_overflow_in_one_micro_batch_skips(micro, path):
    c = Case([5000, 33], 4, O.FP16, 8, O.SCALE_DYNAMIC, init_scale=64.0, path=path)
    try:
        c.step_ex(3, 3.0, 0.5)
        c.compare()
        before = c.gpu_state()
        assert c.step_ex(3, 3.0, 0.5, inject=[(micro, 1, 17, 0x7C00)])
        f = c.gpu_fsm()
        assert f["last_skipped"] == 1 and f["scale"] == 32.0
        c.compare()
        after = c.gpu_state()
        for k in ("master", "m", "v", "param"):
            assert np.array_equal(before[k], after[k])
    finally:
        c.close()


def test_bad_options():
    c = Case([100], 2, O.BF16, 8, O.SCALE_NONE, path="inplace")
    try:
        with pytest.raises(Z.ZeroError) as e:
            Z.zero_step_ex(c.ctx, c.hp, c.handle, c.grads, 1.0, -1.0)
        assert e.value.status == 1
        with pytest.raises(Z.ZeroError):
            Z.zero_step_ex(c.ctx, c.hp, c.handle, c.grads, 0.5, 0.0)
        with pytest.raises(Z.ZeroError):
            Z.zero_reduce_scatter_bucket_ex(c.ctx, 0, c.grads, c.master[0], 4)
        # divisor on the fused path is allowed and matches the oracle
        c.step()
        c.compare()
    finally:
        c.close()


@pytest.mark.parametrize("R", [1, 2, 3, 4, 8])
@pytest.mark.parametrize("dtype", [O.BF16, O.FP16])
@pytest.mark.parametrize("path", ["inplace", "pingpong"])
@pytest.mark.parametrize("clip,divisor", [(1e-3, 1.0), (1e9, 1.0), (2e-3, 2.0)])
def test_fused_clip_matches_oracle(R, dtype, path, clip, divisor):
    # global-norm clipping on the fused path: a norm pass over the replicas,
    # then the fused step with the coefficient
    mode = O.SCALE_DYNAMIC if (dtype == O.FP16 and path == "pingpong") else O.SCALE_NONE
    c = Case([70_001, 13, 4096, 7, 999], R, dtype, 8, mode, init_scale=256.0, interval=2, path=path,
             seed=R + 11)
    try:
        for _ in range(3):
            c.step_fused_ex(divisor, clip)
            c.compare()
        if clip == 1e-3:
            assert c.ofsm.grad_norm_sq > 1e-4  # the clip was active
    finally:
        c.close()


def test_fused_clip_overflow_skips():
    c = Case([20_000, 33], 2, O.FP16, 8, O.SCALE_DYNAMIC, init_scale=64.0, path="pingpong")
    try:
        c.step_fused_ex(1.0, 1e-2)
        c.compare()
        before = c.gpu_state()
        assert c.step_fused_ex(1.0, 1e-2, inject=[(1, 17, 0x7C00)])
        c.compare()
        after = c.gpu_state()
        for k in ("master", "m", "v", "param"):
            assert np.array_equal(before[k], after[k])
        c.step_fused_ex(1.0, 1e-2)
        c.compare()
    finally:
        c.close()


@pytest.mark.parametrize("R", [1, 2, 3, 4, 8, 16])
@pytest.mark.parametrize("dtype", [O.BF16, O.FP16])
@pytest.mark.parametrize("n_micro,divisor", [(2, 2.0), (3, 3.0), (4, 1.0)])
def test_fused_last_micro_batch_matches_oracle(R, dtype, n_micro, divisor):
    # ZERO_STEP_ADD_ACC: the last micro-batch is summed into the step itself
    mode = O.SCALE_DYNAMIC if dtype == O.FP16 else O.SCALE_NONE
    c = Case([70_001, 13, 4096, 7, 999], R, dtype, 8, mode, init_scale=256.0, interval=2,
             path="fused_acc", bucket_elems=5000, seed=R + 3 * n_micro)
    try:
        for _ in range(3):
            c.step_fused_accum(n_micro, divisor)
            c.compare()
    finally:
        c.close()


@pytest.mark.parametrize("micro", [0, 2])
def test_fused_last_micro_batch_overflow_skips(micro):
    c = Case([20_000, 33], 4, O.FP16, 8, O.SCALE_DYNAMIC, init_scale=64.0, path="fused_acc")
    try:
        c.step_fused_accum(3, 3.0)
        c.compare()
        before = c.gpu_state()
        assert c.step_fused_accum(3, 3.0, inject=[(micro, 1, 17, 0x7C00)])
        c.compare()
        after = c.gpu_state()
        for k in ("master", "m", "v", "param"):
            assert np.array_equal(before[k], after[k])
    finally:
        c.close()


def test_add_acc_argument_errors():
    c = Case([1000], 2, O.BF16, 8, O.SCALE_NONE, path="fused_acc")
    try:
        with pytest.raises(Z.ZeroError):  # with clipping
            Z.zero_step_ex(c.ctx, c.hp, c.handle, c.grads, 1.0, 1.0, flags=Z.ZERO_STEP_ADD_ACC)
        with pytest.raises(Z.ZeroError):  # on the two-pass path
            Z.zero_step_ex(c.ctx, c.hp, c.handle, None, 1.0, 0.0, flags=Z.ZERO_STEP_ADD_ACC)
        with pytest.raises(Z.ZeroError):  # unknown flag
            Z.zero_step_ex(c.ctx, c.hp, c.handle, c.grads, 1.0, 0.0, flags=2)
        no_acc = Z.StateHandle([dict(master=c.master[k], m=c.m[k], v=c.v[k], param=c.param[k])
                                for k in range(2)])
        with pytest.raises(Z.ZeroError):  # no accumulators
            Z.zero_step_ex(c.ctx, c.hp, no_acc, c.grads, 1.0, 0.0, flags=Z.ZERO_STEP_ADD_ACC)
    finally:
        c.close()


@pytest.mark.parametrize("R", [2, 3, 8, 16])
@pytest.mark.parametrize("dtype", [O.BF16, O.FP16])
@pytest.mark.parametrize("n_micro,divisor", [(1, 1.0), (2, 2.0), (3, 3.0)])
@pytest.mark.parametrize("clip", [1e-3, 1e9])
@pytest.mark.parametrize("whole", [False, True])
def test_norm_from_reduce_scatter_matches_oracle(R, dtype, n_micro, divisor, clip, whole):
    # the clipping norm taken by the last micro-batch's reduce-scatters
    # (ZERO_RS_NORM) instead of a pass over the accumulators: the same bytes
    mode = O.SCALE_DYNAMIC if dtype == O.FP16 else O.SCALE_NONE
    c = Case([70_001, 13, 4096, 7, 999], R, dtype, 8 if R != 3 else 1, mode, init_scale=256.0,
             interval=2, path="twopass_pp" if R != 16 else "twopass", bucket_elems=5000)
    try:
        for _ in range(3):
            c.step_ex(n_micro, divisor, clip, rs_norm=True, whole=whole)
            c.compare()
        if clip == 1e-3:
            assert c.ofsm.grad_norm_sq > 1e-4
    finally:
        c.close()


def test_norm_from_reduce_scatter_skips_on_overflow():
    c = Case([5000, 33], 4, O.FP16, 8, O.SCALE_DYNAMIC, init_scale=64.0, path="twopass_pp",
             bucket_elems=1000)
    try:
        c.step_ex(2, 2.0, 0.5, rs_norm=True)
        c.compare()
        before = c.gpu_state()
        assert c.step_ex(2, 2.0, 0.5, inject=[(1, 2, 40, 0x7C00)], rs_norm=True)
        assert c.gpu_fsm()["last_skipped"] == 1
        c.compare()
        after = c.gpu_state()
        for k in ("master", "m", "v", "param"):
            assert np.array_equal(before[k], after[k])
        c.step_ex(2, 2.0, 0.5, rs_norm=True)
        c.compare()
    finally:
        c.close()


def test_norm_from_reduce_scatter_refusals():
    c = Case([3000, 17, 2048], 4, O.BF16, 8, O.SCALE_NONE, path="twopass", bucket_elems=1000)
    nb = len(c.plan.buckets)
    assert nb >= 3
    norm_step = dict(flags=Z.ZERO_STEP_NORM_FROM_RS)
    try:
        with pytest.raises(Z.ZeroError) as e:
            Z.zero_ctx_set_grad_divisor(c.ctx, 0.5)
        assert e.value.status == Z.ZERO_ERR_INVALID_ARG
        # no reduce-scatter recorded a norm share
        with pytest.raises(Z.ZeroError) as e:
            Z.zero_step_ex(c.ctx, c.hp, c.handle, None, 1.0, 1.0, **norm_step)
        assert e.value.status == Z.ZERO_ERR_STATE
        # every bucket with its share, then bucket 1 again without: stale
        for b in range(nb):
            Z.zero_reduce_scatter_bucket_ex(c.ctx, b, c.grads, c.acc, Z.ZERO_RS_NORM)
        Z.zero_reduce_scatter_bucket_ex(c.ctx, 1, c.grads, c.acc, 0)
        with pytest.raises(Z.ZeroError) as e:
            Z.zero_step_ex(c.ctx, c.hp, c.handle, None, 1.0, 1.0, **norm_step)
        assert e.value.status == Z.ZERO_ERR_STATE
        # shares taken with another divisor
        Z.zero_ctx_set_grad_divisor(c.ctx, 2.0)
        for b in range(nb):
            Z.zero_reduce_scatter_bucket_ex(c.ctx, b, c.grads, c.acc, Z.ZERO_RS_NORM)
        with pytest.raises(Z.ZeroError) as e:
            Z.zero_step_ex(c.ctx, c.hp, c.handle, None, 1.0, 1.0, **norm_step)
        assert e.value.status == Z.ZERO_ERR_STATE
        # a whole-range call without the flag makes every share stale
        Z.zero_reduce_scatter_bucket_ex(c.ctx, -1, c.grads, c.acc, 0)
        with pytest.raises(Z.ZeroError) as e:
            Z.zero_step_ex(c.ctx, c.hp, c.handle, None, 2.0, 1.0, **norm_step)
        assert e.value.status == Z.ZERO_ERR_STATE
        # the flag needs the two-pass path and clipping
        with pytest.raises(Z.ZeroError) as e:
            Z.zero_step_ex(c.ctx, c.hp, c.handle, None, 1.0, 0.0, **norm_step)
        assert e.value.status == Z.ZERO_ERR_INVALID_ARG
        with pytest.raises(Z.ZeroError) as e:
            Z.zero_step_ex(c.ctx, c.hp, c.handle, c.grads, 1.0, 1.0, **norm_step)
        assert e.value.status == Z.ZERO_ERR_INVALID_ARG
        # nothing above stepped: a proper step still matches the oracle
        Z.zero_ctx_set_grad_divisor(c.ctx, 1.0)
        c.step_ex(1, 1.0, 1e-3, rs_norm=True)
        c.compare()
        # a step consumes the shares
        with pytest.raises(Z.ZeroError) as e:
            Z.zero_step_ex(c.ctx, c.hp, c.handle, None, 1.0, 1.0, **norm_step)
        assert e.value.status == Z.ZERO_ERR_STATE
    finally:
        c.close()


@pytest.mark.parametrize("R,dtype", [(3, O.FP16), (8, O.BF16)])
@pytest.mark.parametrize("rs_norm", [False, True])
def test_grouped_reduce_scatters_match_oracle(R, dtype, rs_norm):
    # consecutive buckets in one launch each (zero_reduce_scatter_buckets):
    # the oracle's bytes, with accumulation, clipping and the norm shares
    mode = O.SCALE_DYNAMIC if dtype == O.FP16 else O.SCALE_NONE
    c = Case([70_001, 13, 4096, 7, 999, 20_000, 3, 5000], R, dtype, 8 if R != 3 else 1, mode,
             init_scale=256.0, interval=2, path="twopass_pp", bucket_elems=3000)
    nb = len(c.plan.buckets)
    assert nb >= 5
    try:
        for groups in ([(0, nb)], [(0, 2), (2, 1), (3, nb - 3)], [(b, 1) for b in range(nb)]):
            c.step_ex(2, 2.0, 1e-3, rs_norm=rs_norm, groups=groups)
            c.compare()
    finally:
        c.close()


def test_grouped_reduce_scatter_range_errors():
    c = Case([3000, 17, 2048], 2, O.BF16, 8, O.SCALE_NONE, path="twopass", bucket_elems=1000)
    nb = len(c.plan.buckets)
    try:
        for first, count in ((0, 0), (-2, 1), (-1, 2), (1, nb), (nb, 1)):
            with pytest.raises(Z.ZeroError) as e:
                Z.zero_reduce_scatter_buckets(c.ctx, first, count, c.grads, c.acc)
            assert e.value.status == Z.ZERO_ERR_RANGE, (first, count)
        with pytest.raises(Z.ZeroError) as e:
            Z.zero_reduce_scatter_buckets(c.ctx, 0, 1, c.grads, c.acc, 8)
        assert e.value.status == Z.ZERO_ERR_INVALID_ARG
    finally:
        c.close()
