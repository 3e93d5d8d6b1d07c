"""The ZeRO-1/2 parameter all-gather done by the step itself
(ZERO_STEP_PUSH_PARAMS): every updated half parameter vector is also stored
into every rank's registered full-model buffer of the set the step writes.
After each step (and each sharded step's commit), every rank's buffer of the
current set must equal the oracle's parameters in the flat layout, padding
zero; a skipped step leaves the current set's buffers as they were. R
simulated ranks on one GPU; with one process per GPU the same kernels store
into peer-mapped buffers."""
import numpy as np
import pytest
import torch

import oracle as O

pytestmark = pytest.mark.gpu

if torch.cuda.is_available():
    import zero_partitioned_mixed_reduce_b200 as Z
    from gpu_harness import Case, u16

INF = {O.FP16: 0x7C00, O.BF16: 0x7F80}


def _register(c):
    full = [[c.g.half(c.plan.T, c.dtype) for _ in range(c.R)] for _ in range(c.sets)]
    Z.zero_ctx_set_param_push(c.ctx, full[0], full[1] if c.sets == 2 else None)
    return full


def _hp(c):
    return O.AdamW(**{k: c.hp[k] for k in ("lr", "beta1", "beta2", "eps", "weight_decay")})


def _load(c, g):
    for r in range(c.R):
        gp = np.zeros(c.plan.T, np.uint16)
        gp[c.idx] = g[r]
        c.grads[r].view(torch.int16).copy_(torch.from_numpy(gp.view(np.int16)))


def _step(c, how, inject=None, splits=None, clip=0.0):
    c.step_no += 1
    g = c.make_grads(inject)
    _load(c, g)
    F = Z.ZERO_STEP_PUSH_PARAMS
    if how == "fused":
        Z.zero_step_ex(c.ctx, c.hp, c.handle, c.grads, 1.0, clip, flags=F)
    elif how == "twopass":
        Z.zero_reduce_scatter_bucket(c.ctx, -1, c.grads, c.acc)
        Z.zero_step_ex(c.ctx, c.hp, c.handle, None, 1.0, clip, flags=F)
    else:  # sharded: one launch per owner range, the partials summed as an all-reduce would
        parts = []
        for lo, hi in splits:
            part = torch.zeros(2, dtype=torch.float64, device="cuda")
            Z.zero_step_shard_ex(c.ctx, c.hp, c.handle, c.grads, lo, hi, part, flags=F)
            parts.append(part)
        Z.zero_step_commit(c.ctx, torch.stack(parts).sum(0))
    if clip > 0:
        O.step_ex(c.ostate, g[None], _hp(c), c.ofsm, 1.0, clip)
    else:
        O.step(c.ostate, g, _hp(c), c.ofsm)
    c.g.check()


def _check_full(c, full):
    f = c.gpu_fsm()
    cur = f["cur"] if c.sets == 2 else 0
    want = np.zeros(c.plan.T, np.uint16)
    want[c.idx] = c.ostate.param
    for r in range(c.R):
        assert np.array_equal(u16(full[cur][r]), want), r


@pytest.mark.parametrize("R", [1, 2, 3, 4, 8])
def test_fused_pingpong_push_with_a_skipped_step(R):
    c = Case([70_001, 13, 4096, 999], R, O.FP16, 8 if R != 3 else 1, O.SCALE_DYNAMIC, init_scale=256.0,
             interval=2, path="pingpong", seed=R + 200)
    try:
        full = _register(c)
        for s in range(4):
            _step(c, "fused", inject=[(R - 1, 5, INF[O.FP16])] if s == 1 else None)
            c.compare()
            _check_full(c, full)
        assert c.ofsm.t == 3 and c.ofsm.last_skipped == 0
    finally:
        c.close()


def test_fused_in_place_push_bf16_and_clipped():
    c = Case([50_000, 777, 3], 4, O.BF16, 8, O.SCALE_NONE, path="inplace", seed=211)
    try:
        full = _register(c)
        for clip in (0.0, 1e-3, 0.0):
            _step(c, "fused", clip=clip)
            c.compare()
            _check_full(c, full)
    finally:
        c.close()


@pytest.mark.parametrize("path,mode", [("twopass", O.SCALE_STATIC), ("twopass_pp", O.SCALE_DYNAMIC)])
def test_two_pass_push(path, mode):
    c = Case([40_000, 17, 9000], 3, O.FP16, 1, mode, init_scale=64.0, interval=2, path=path, seed=212)
    try:
        full = _register(c)
        for s in range(3):
            _step(c, "twopass", inject=[(0, 11, INF[O.FP16])] if (s == 1 and mode == O.SCALE_DYNAMIC) else None)
            c.compare()
            _check_full(c, full)
    finally:
        c.close()


def test_sharded_push_every_range_writes_every_rank():
    c = Case([60_000, 5, 12_345], 4, O.FP16, 8, O.SCALE_DYNAMIC, init_scale=128.0, interval=2,
             path="pingpong", seed=213)
    try:
        full = _register(c)
        for s in range(3):
            _step(c, "sharded", splits=[(0, 1), (1, 2), (2, 4)],
                  inject=[(2, 70, INF[O.FP16])] if s == 1 else None)
            c.compare()
            _check_full(c, full)
        assert c.ofsm.t == 2
    finally:
        c.close()


def test_push_needs_registered_buffers():
    c = Case([1_000], 2, O.BF16, 8, O.SCALE_NONE, path="pingpong", seed=214)
    try:
        c.step_no += 1
        _load(c, c.make_grads())
        with pytest.raises(Z.ZeroError) as e:
            Z.zero_step_ex(c.ctx, c.hp, c.handle, c.grads, flags=Z.ZERO_STEP_PUSH_PARAMS)
        assert e.value.status == Z.ZERO_ERR_STATE
        # set 0 alone is not enough for ping-pong state
        one = [c.g.half(c.plan.T, c.dtype) for _ in range(c.R)]
        Z.zero_ctx_set_param_push(c.ctx, one)
        with pytest.raises(Z.ZeroError) as e:
            Z.zero_step_ex(c.ctx, c.hp, c.handle, c.grads, flags=Z.ZERO_STEP_PUSH_PARAMS)
        assert e.value.status == Z.ZERO_ERR_STATE
        Z.zero_ctx_set_param_push(c.ctx, None)
    finally:
        c.close()


def test_push_registration_errors():
    c = Case([1_000], 2, O.BF16, 8, O.SCALE_NONE, path="inplace", seed=215)
    try:
        full = [c.g.half(c.plan.T, c.dtype) for _ in range(c.R)]
        with pytest.raises(Z.ZeroError) as e:
            Z.zero_ctx_set_param_push(c.ctx, [full[0], None])
        assert e.value.status == Z.ZERO_ERR_INVALID_ARG
        with pytest.raises(Z.ZeroError) as e:
            Z.zero_ctx_set_param_push(c.ctx, [full[0].data_ptr() + 2, full[1]])
        assert e.value.status == Z.ZERO_ERR_ALIGN
        with pytest.raises(Z.ZeroError) as e:  # the push is not a CPU-step flag, nor CLEAN a GPU one
            Z.zero_step_ex(c.ctx, c.hp, c.handle, c.grads, flags=Z.ZERO_STEP_CLEAN)
        assert e.value.status == Z.ZERO_ERR_INVALID_ARG
    finally:
        c.close()
