"""The error path of the staged fused step (R <= 2), exercised without a
fault: zero_test_drop_tile makes the kernel issue no copy for one tile, so
the block that waits for it gives up after its 2 s limit. The step must then
be abandoned (t, scale, good and cur unchanged, the current ping-pong set
untouched), reported as ZERO_ERR_TIMEOUT, cleared by a SET, and the context
must keep stepping in lockstep with the oracle afterwards."""
import numpy as np
import pytest
import torch

import oracle as O

pytestmark = pytest.mark.gpu

if torch.cuda.is_available():
    import zero_partitioned_mixed_reduce_b200 as Z
    from gpu_harness import Case


def _write_grads(c):
    c.step_no += 1
    g = c.make_grads()
    for r in range(c.R):
        gp = np.zeros(c.plan.T, np.uint16)
        gp[c.idx] = g[r]
        c.grads[r].view(torch.int16).copy_(torch.from_numpy(gp.view(np.int16)))


def _same_state(a, b):
    for k in ("master", "m", "v", "param"):
        assert np.array_equal(np.asarray(a[k]).view(np.uint8), np.asarray(b[k]).view(np.uint8)), k


@pytest.mark.parametrize("R,dtype,mode", [(2, O.FP16, O.SCALE_DYNAMIC), (1, O.BF16, O.SCALE_NONE)])
def test_timed_out_step_is_abandoned_and_reported(R, dtype, mode):
    c = Case([40_000, 3_000], R, dtype, mode=mode, init_scale=256.0, interval=2, path="pingpong",
             seed=71)
    try:
        c.step()
        c.compare()
        before, f0 = c.gpu_state(), c.gpu_fsm()
        Z.zero_test_drop_tile(c.ctx, 3)
        _write_grads(c)  # this step's gradients never reach the oracle
        Z.zero_step(c.ctx, c.hp, c.handle, c.grads)
        torch.cuda.synchronize()
        with pytest.raises(Z.ZeroError) as e:
            Z.zero_loss_scale(c.ctx)
        assert e.value.status == Z.ZERO_ERR_TIMEOUT
        c.g.check()
        # SET clears the error; the abandoned step left the state as it was
        Z.zero_loss_scale(c.ctx, Z.ZERO_LOSS_SCALE_SET, f0)
        f1 = c.gpu_fsm()
        assert (f1["t"], f1["cur"], f1["good"], f1["scale"]) == (f0["t"], f0["cur"], f0["good"], f0["scale"])
        _same_state(before, c.gpu_state())
        # the hook was one-shot: the next steps run and match the oracle
        for _ in range(2):
            c.step()
            c.compare()
    finally:
        c.close()


def test_timed_out_shard_is_abandoned_locally():
    c = Case([30_000, 500], 2, O.FP16, mode=O.SCALE_DYNAMIC, init_scale=64.0, path="pingpong", seed=72)
    try:
        c.step_sharded([(0, 1), (1, 2)])
        c.compare()
        before, f0 = c.gpu_state(), c.gpu_fsm()
        Z.zero_test_drop_tile(c.ctx, 1)
        _write_grads(c)
        part = torch.zeros(2, dtype=torch.float64, device="cuda")
        Z.zero_step_shard(c.ctx, c.hp, c.handle, c.grads, 0, 2, part)
        Z.zero_step_commit(c.ctx, part)
        torch.cuda.synchronize()
        with pytest.raises(Z.ZeroError) as e:
            Z.zero_loss_scale(c.ctx)
        assert e.value.status == Z.ZERO_ERR_TIMEOUT
        Z.zero_loss_scale(c.ctx, Z.ZERO_LOSS_SCALE_SET, f0)
        _same_state(before, c.gpu_state())
        c.step_sharded([(0, 2)])
        c.compare()
    finally:
        c.close()


def test_drop_tile_argument_errors():
    c = Case([1_000], 2, O.BF16, path="pingpong", seed=73)
    try:
        with pytest.raises(Z.ZeroError):
            Z.zero_test_drop_tile(c.ctx, -1)
        with pytest.raises(Z.ZeroError):
            Z.zero_test_drop_tile(c.ctx, 1 << 40)
    finally:
        c.close()
