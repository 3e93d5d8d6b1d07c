"""Pin the oracle's reduction and the ZeRO invariant: the partitioned step
over the padded layout equals plain data-parallel training (mbrenndoerfer
introduction: every replica applies the same update; inferensys
instruction-tuning glossary: the reduce-scatter averages like the DP
all-reduce it replaces)."""
import numpy as np
import pytest
import torch

import oracle as O

HP = O.AdamW(1e-3, 0.9, 0.999, 1e-8, 0.01)
TORCH = {O.BF16: torch.bfloat16, O.FP16: torch.float16}


def torch_decode(h, dtype):
    return torch.from_numpy(np.ascontiguousarray(h).view(np.int16)).view(TORCH[dtype]).float().numpy()


@pytest.mark.parametrize("dtype", [O.BF16, O.FP16])
@pytest.mark.parametrize("R", [1, 2, 3, 5, 16])
def test_allreduce_matches_numpy_rank_order_sum(dtype, R):
    rng = np.random.default_rng(R)
    P = 1001
    g = O.float_to_half(rng.standard_t(3, (R, P)).astype(np.float32), dtype)
    acc, ovf = O.allreduce_sum(g, dtype)
    f = torch_decode(g, dtype)
    want = f[0].copy()
    for r in range(1, R):
        want = want + f[r]  # numpy float32 add: one rounding per rank
    assert not ovf
    assert np.array_equal(acc.view(np.uint32), want.view(np.uint32))


def test_grad_norm_matches_numpy():
    rng = np.random.default_rng(2)
    R, P = 4, 5000
    g = O.float_to_half(rng.normal(0, 1e-2, (R, P)).astype(np.float32) * 256, O.FP16)
    st = O.State(np.zeros(P, np.float32), O.FP16)
    fsm = O.make_fsm(O.SCALE_STATIC, scale=256.0)
    O.step(st, g, HP, fsm)
    acc, _ = O.allreduce_sum(g, O.FP16)
    gg = (acc * np.float32(1.0 / (R * 256.0))).astype(np.float64)
    want = np.sum(gg * gg)
    assert abs(fsm.grad_norm_sq - want) <= 1e-12 * want


def pack(lay, values_unpadded, fill=0):
    out = np.full(lay.T, fill, dtype=values_unpadded.dtype)
    out[lay.flat_index()] = values_unpadded
    return out


@pytest.mark.parametrize("seed", range(12))
def test_sharded_step_equals_unsharded(seed):
    rng = np.random.default_rng(100 + seed)
    n = int(rng.integers(1, 9))
    numels = rng.integers(1, 40, n)
    R = int(rng.choice([1, 2, 3, 4, 7, 8]))
    A = int(rng.choice([1, 8]))
    dtype = int(rng.choice([O.BF16, O.FP16]))
    mode = int(rng.choice([O.SCALE_NONE, O.SCALE_STATIC, O.SCALE_DYNAMIC]))
    lay = O.Layout(numels, R, A)
    P = lay.P
    x = rng.normal(0, 0.02, P).astype(np.float32)

    flat = O.State(x, dtype)
    f_flat = O.make_fsm(mode, scale=64.0, interval=3)
    f_shard = O.make_fsm(mode, scale=64.0, interval=3)
    master, m, v = pack(lay, x), np.zeros(lay.T, np.float32), np.zeros(lay.T, np.float32)
    param = pack(lay, flat.param)
    for s in range(6):
        g = O.float_to_half(rng.normal(0, 1e-2, (R, P)).astype(np.float32) * 64, dtype)
        if s == 3:
            g[int(rng.integers(0, R)), int(rng.integers(0, P))] = 0x7C00 if dtype == O.FP16 else 0x7F80
        gp = np.zeros((R, lay.T), np.uint16)
        gp[:, lay.flat_index()] = g
        k1 = O.step(flat, g, HP, f_flat)
        k2, gathered = O.step_sharded(lay.S, R, dtype, gp, master, m, v, param, HP, f_shard)
        assert k1 == k2
        idx = lay.flat_index()
        for a, b in ((flat.master, master), (flat.m, m), (flat.v, v)):
            assert np.array_equal(a.view(np.uint32), b[idx].view(np.uint32))
        assert np.array_equal(flat.param, param[idx])
        assert np.array_equal(gathered, param)
        # padding never moves
        pad = np.ones(lay.T, bool)
        pad[idx] = False
        if mode != O.SCALE_NONE or s < 3:
            assert np.all(master[pad] == 0) and np.all(param[pad] == 0)
        assert (f_flat.scale, f_flat.t, f_flat.good, f_flat.last_overflow) == \
               (f_shard.scale, f_shard.t, f_shard.good, f_shard.last_overflow)
        same_norm = (f_flat.grad_norm_sq == f_shard.grad_norm_sq) or (
            np.isnan(f_flat.grad_norm_sq) and np.isnan(f_shard.grad_norm_sq))
        assert same_norm


@pytest.mark.parametrize("R", [2, 4, 8, 16])
@pytest.mark.parametrize("dtype", [O.BF16, O.FP16])
def test_identical_replicas_equal_single_rank(R, dtype):
    # Summing R equal half values in fp32 is exact and dividing by a power of
    # two is exact, so R identical replicas must reproduce R = 1 bit for bit.
    rng = np.random.default_rng(R)
    P = 777
    x = rng.normal(0, 0.02, P).astype(np.float32)
    one, many = O.State(x, dtype), O.State(x, dtype)
    f1, fr = O.make_fsm(O.SCALE_NONE), O.make_fsm(O.SCALE_NONE)
    for _ in range(4):
        g = O.float_to_half(rng.normal(0, 1e-2, P).astype(np.float32), dtype)
        O.step(one, g[None, :], HP, f1)
        O.step(many, np.tile(g, (R, 1)), HP, fr)
    for a in ("master", "m", "v", "param"):
        assert np.array_equal(getattr(one, a), getattr(many, a))


def test_dp_replicas_stay_identical():
    # plain DP: each replica all-reduces the same gradients and updates its own
    # full copy; all copies stay equal
    rng = np.random.default_rng(4)
    R, P = 4, 500
    x = rng.normal(0, 0.02, P).astype(np.float32)
    reps = [O.State(x, O.FP16) for _ in range(R)]
    fs = [O.make_fsm(O.SCALE_STATIC, scale=8.0) for _ in range(R)]
    for _ in range(3):
        g = O.float_to_half(rng.normal(0, 1e-2, (R, P)).astype(np.float32) * 8, O.FP16)
        for st, f in zip(reps, fs):
            O.step(st, g, HP, f)
    for st in reps[1:]:
        assert np.array_equal(st.master, reps[0].master) and np.array_equal(st.param, reps[0].param)
