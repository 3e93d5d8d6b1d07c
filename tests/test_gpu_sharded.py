"""The per-rank step of a multi-GPU ZeRO run, emulated in one process:
zero_step_shard over each owner range (no kernel waits on another; the
launches simply follow each other), the per-range totals summed as the
cross-rank all-reduce would, then zero_step_commit. The result must equal
the oracle bit for bit (the gradient norm within its summation-order bound)."""
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
