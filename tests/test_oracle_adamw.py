"""Pins for the oracle's AdamW arithmetic, none of which restates its formula:
a hand-computed two-step case, closed forms for constant and zero
gradients, and torch.optim.AdamW (single-tensor path) as a library special
case."""
import os

import numpy as np
import pytest
import torch

import oracle as O

HP = dict(lr=1e-3, beta1=0.9, beta2=0.999, eps=1e-8, weight_decay=0.01)


def hp(**kw):
    d = dict(HP)
    d.update(kw)
    return O.AdamW(d["lr"], d["beta1"], d["beta2"], d["eps"], d["weight_decay"])


def rel(a, b):
    return np.abs(np.float64(a) - np.float64(b)) / np.maximum(np.abs(np.float64(b)), 1e-30)


def read_golden(path):
    rows = []
    for line in open(path):
        line = line.strip()
        if line and not line.startswith("#"):
            rows.append([float(x) for x in line.split()])
    return rows


def test_hand_computed_two_steps(golden_dir):
    rows = read_golden(os.path.join(golden_dir, "adamw_one_param.txt"))
    # R = 1, loss scale 1: the half gradient 0.5 is exact in both formats
    for dtype in (O.BF16, O.FP16):
        st = O.State(np.array([1.0], np.float32), dtype)
        fsm = O.make_fsm(O.SCALE_NONE)
        g = O.float_to_half(np.array([[0.5]], np.float32), dtype)
        for step, p, m, v in rows:
            O.step(st, g, hp(), fsm)
            assert fsm.t == int(step)
            assert rel(st.master[0], p) < 1e-6
            assert rel(st.m[0], m) < 1e-6
            assert rel(st.v[0], v) < 1e-6


@pytest.mark.parametrize("gval", [0.5, -3.0, 1e-3, 2.0 ** -20])
def test_constant_gradient_closed_form(gval):
    # With g fixed, m_t = g (1 - b1^t) and v_t = g^2 (1 - b2^t) exactly, so the
    # bias-corrected update is lr * g / (|g| + eps) every step:
    #   p_t = p_{t-1} (1 - lr wd) - lr g / (|g| + eps).
    # A tiny |g| (2^-20 vs eps 1e-8 is still large; 1e-3 and 2^-20 differ in how
    # much eps matters) separates eps placements.
    p0 = np.float32(0.25)
    st = O.State(np.array([p0], np.float32), O.FP16)
    fsm = O.make_fsm(O.SCALE_NONE)
    gh = O.float_to_half(np.array([[gval]], np.float32), O.FP16)
    g = float(O.half_to_float(gh[0], O.FP16)[0])
    p = float(p0)
    lr, wd, eps = HP["lr"], HP["weight_decay"], HP["eps"]
    for _ in range(12):
        O.step(st, gh, hp(), fsm)
        p = p * (1 - lr * wd) - lr * g / (abs(g) + eps)
        assert abs(st.master[0] - p) <= 2e-6 * abs(p) + 1e-9


def test_eps_placement_with_tiny_gradient():
    # |g| far below eps: the update is lr * g / (|g| + eps) ~ lr * g / eps; an
    # eps inside the square root would give lr * g / sqrt(eps) instead.
    g = 2.0 ** -30
    st = O.State(np.array([0.0], np.float32), O.BF16)
    fsm = O.make_fsm(O.SCALE_NONE)
    gh = O.float_to_half(np.array([[g]], np.float32), O.BF16)
    O.step(st, gh, hp(weight_decay=0.0), fsm)
    want = -HP["lr"] * g / (g + HP["eps"])
    assert rel(st.master[0], want) < 1e-5


def test_zero_gradient_is_pure_decay():
    # g = 0: m = v = 0, the Adam term is 0 / eps = 0, so only p (1 - lr wd) remains.
    x = np.array([1.0, -2.5, 0.125, 3e-5], np.float32)
    st = O.State(x, O.FP16)
    fsm = O.make_fsm(O.SCALE_NONE)
    z = np.zeros((1, x.size), np.uint16)
    for k in range(1, 4):
        O.step(st, z, hp(), fsm)
        want = x.astype(np.float64) * (1 - HP["lr"] * HP["weight_decay"]) ** k
        assert np.all(rel(st.master, want) < 1e-6)
    assert np.all(st.m == 0) and np.all(st.v == 0)


def test_averaging_and_unscale():
    # R identical replicas and a loss scale s give the same update as one
    # replica of the unscaled gradient: the step sees sum / (R s).
    rng = np.random.default_rng(3)
    P = 257
    x = rng.normal(0, 0.02, P).astype(np.float32)
    g = rng.normal(0, 1e-3, P).astype(np.float32)
    for dtype in (O.BF16, O.FP16):
        ref = O.State(x, dtype)
        f1 = O.make_fsm(O.SCALE_NONE)
        O.step(ref, O.float_to_half(g, dtype)[None, :], hp(), f1)
        for R, scale in ((4, 1.0), (8, 1024.0), (2, 65536.0)):
            gs = O.float_to_half(g * np.float32(scale), dtype)
            # only compare where the scaled half value is the same number as
            # the unscaled one times the scale (no rounding difference)
            same = O.half_to_float(gs, dtype) == O.half_to_float(
                O.float_to_half(g, dtype), dtype) * np.float32(scale)
            st = O.State(x, dtype)
            fr = O.make_fsm(O.SCALE_STATIC, scale=scale)
            O.step(st, np.tile(gs, (R, 1)), hp(), fr)
            assert np.array_equal(st.master[same], ref.master[same])
            assert np.array_equal(st.m[same], ref.m[same])
            assert np.array_equal(st.v[same], ref.v[same])


@pytest.mark.parametrize("wd", [0.0, 0.01, 0.1])
def test_matches_torch_adamw_single_tensor(wd):
    # torch's single-tensor AdamW (foreach=False) on CPU fp32 is the library
    # special case: R = 1, scale 1. It forms m by lerp and v by addcmul, so
    # the two may differ by an ulp per step.
    rng = np.random.default_rng(5)
    P, steps = 4099, 7
    x = rng.normal(0, 0.02, P).astype(np.float32)
    st = O.State(x, O.BF16)
    fsm = O.make_fsm(O.SCALE_NONE)
    w = torch.nn.Parameter(torch.from_numpy(x.copy()))
    opt = torch.optim.AdamW([w], lr=HP["lr"], betas=(HP["beta1"], HP["beta2"]), eps=HP["eps"],
                            weight_decay=wd, foreach=False, fused=False)
    for _ in range(steps):
        gh = O.float_to_half(rng.normal(0, 1e-2, P).astype(np.float32), O.BF16)
        O.step(st, gh[None, :], hp(weight_decay=wd), fsm)
        w.grad = torch.from_numpy(O.half_to_float(gh, O.BF16))
        opt.step()
    ref = w.detach().numpy()
    s = opt.state[w]
    assert np.all(np.abs(st.master - ref) <= 1e-6 * np.abs(ref) + 1e-9)
    # m and v can nearly cancel, so their bound is a few ulps of the gradient
    # scale (|g| < 0.06, g^2 < 4e-3), far below what a dropped term would move
    assert np.all(np.abs(st.m - s["exp_avg"].numpy()) <= 1e-5 * np.abs(st.m) + 2e-8)
    assert np.all(np.abs(st.v - s["exp_avg_sq"].numpy()) <= 1e-5 * np.abs(st.v) + 1e-12)
    # the half parameter is the rounded master
    assert np.array_equal(st.param, torch_param_bf16(st.master))


def torch_param_bf16(x):
    return torch.from_numpy(x).to(torch.bfloat16).view(torch.int16).numpy().view(np.uint16)


def test_step_count_and_bias_correction_progress():
    # t advances by one per applied step; at t = 1 the bias-corrected moments
    # are g and g^2, so every coordinate moves by -lr g / (|g| + eps), i.e. by
    # about lr against the sign of its gradient.
    rng = np.random.default_rng(9)
    P = 1000
    x = rng.normal(0, 0.02, P).astype(np.float32)
    g = rng.normal(0, 1e-2, P).astype(np.float32)
    gh = O.float_to_half(g, O.FP16)
    gf = O.half_to_float(gh, O.FP16)
    st = O.State(x, O.FP16)
    fsm = O.make_fsm(O.SCALE_NONE)
    O.step(st, gh[None, :], hp(weight_decay=0.0), fsm)
    d = st.master.astype(np.float64) - x
    nz = gf != 0
    gd = gf.astype(np.float64)
    want = -HP["lr"] * gd / (np.abs(gd) + HP["eps"])
    assert np.all(np.abs(d - want) < 2e-8)  # a few float ulps of |p| ~ 0.1
    assert np.all(np.abs(d[nz]) > 0.9 * HP["lr"] * (np.abs(gd[nz]) > 1e-6))
    assert fsm.t == 1
