"""Pins for the oracle's gradient accumulation and global-norm clipping
(oracle_step_ex). Neither is on the pages; the readings are stated in
zero_oracle.c. The pins: torch.nn.utils.clip_grad_norm_ followed by
torch.optim.AdamW (single tensor) as the library special case; invariance of
k identical micro-batches under divisor k; the accumulated norm against a
numpy float64 sum; closed forms for m and v after one clipped step; and an
inactive clip leaving the step unchanged bit for bit."""
import numpy as np
import pytest
import torch

import oracle as O

HP = O.AdamW(1e-3, 0.9, 0.999, 1e-8, 0.01)
TORCH = {O.BF16: torch.bfloat16, O.FP16: torch.float16}


def decode(h, dtype):
    return torch.from_numpy(np.ascontiguousarray(h).view(np.int16)).view(TORCH[dtype]).float().numpy()


@pytest.mark.parametrize("max_norm", [0.05, 0.5, 1e9])
def test_clip_matches_torch_clip_grad_norm_then_adamw(max_norm):
    rng = np.random.default_rng(8)
    P, steps = 3001, 5
    x = rng.normal(0, 0.02, P).astype(np.float32)
    st = O.State(x, O.BF16)
    fsm = O.make_fsm(O.SCALE_NONE)
    w = torch.nn.Parameter(torch.from_numpy(x.copy()))
    opt = torch.optim.AdamW([w], lr=HP.lr, betas=(HP.beta1, HP.beta2), eps=HP.eps,
                            weight_decay=HP.weight_decay, foreach=False, fused=False)
    for _ in range(steps):
        gh = O.float_to_half(rng.normal(0, 1e-2, P).astype(np.float32), O.BF16)
        O.step_ex(st, gh[None, None, :], HP, fsm, 1.0, max_norm)
        w.grad = torch.from_numpy(decode(gh, O.BF16))
        total = torch.nn.utils.clip_grad_norm_([w], max_norm)
        assert abs(float(total) ** 2 - fsm.grad_norm_sq) <= 1e-5 * fsm.grad_norm_sq
        opt.step()
    ref = w.detach().numpy()
    assert np.all(np.abs(st.master - ref) <= 2e-6 * np.abs(ref) + 1e-9)


@pytest.mark.parametrize("k", [2, 4, 8])
@pytest.mark.parametrize("dtype", [O.BF16, O.FP16])
def test_identical_micro_batches_with_divisor_k_equal_one_step(k, dtype):
    # k equal micro-batch sums add exactly (power-of-two k, few significant
    # bits), and dividing by R*k*scale is exact, so the step is bit-identical
    rng = np.random.default_rng(k)
    R, P = 4, 999
    x = rng.normal(0, 0.02, P).astype(np.float32)
    g = O.float_to_half(rng.normal(0, 1e-2, (R, P)).astype(np.float32), dtype)
    one, acc = O.State(x, dtype), O.State(x, dtype)
    f1, fk = O.make_fsm(O.SCALE_STATIC, 16.0), O.make_fsm(O.SCALE_STATIC, 16.0)
    O.step(one, g, HP, f1)
    O.step_ex(acc, np.stack([g] * k), HP, fk, float(k), 0.0)
    for a in ("master", "m", "v", "param"):
        assert np.array_equal(getattr(one, a), getattr(acc, a))
    assert f1.grad_norm_sq == fk.grad_norm_sq


def test_accumulated_norm_matches_numpy():
    rng = np.random.default_rng(3)
    n, R, P = 3, 2, 2000
    g = O.float_to_half(rng.standard_t(3, (n, R, P)).astype(np.float32) * 1e-2, O.FP16)
    st = O.State(np.zeros(P, np.float32), O.FP16)
    fsm = O.make_fsm(O.SCALE_STATIC, 8.0)
    O.step_ex(st, g, HP, fsm, 3.0, 0.0)
    f = decode(g, O.FP16)
    acc = f[0, 0] + f[0, 1]
    for mu in range(1, n):
        acc = acc + (f[mu, 0] + f[mu, 1])
    inv = np.float32(1.0 / ((R * 3.0) * 8.0))
    gg = (acc * inv).astype(np.float64)
    want = np.sum(gg * gg)
    assert abs(fsm.grad_norm_sq - want) <= 1e-12 * want


def test_first_clipped_step_moments_closed_form():
    # at t = 1, m = (1 - b1) g c and v = (1 - b2) (g c)^2 with
    # c = max_norm / (||g|| + 1e-6) when that is below 1
    rng = np.random.default_rng(5)
    P = 500
    gh = O.float_to_half(rng.normal(0, 1e-1, P).astype(np.float32), O.FP16)
    g = decode(gh, O.FP16).astype(np.float64)
    norm = np.sqrt(np.sum(g * g))
    max_norm = 0.25 * norm
    c = max_norm / (norm + 1e-6)
    st = O.State(np.zeros(P, np.float32), O.FP16)
    fsm = O.make_fsm(O.SCALE_NONE)
    O.step_ex(st, gh[None, None, :], HP, fsm, 1.0, max_norm)
    assert np.allclose(st.m, (1 - HP.beta1) * g * c, rtol=2e-6, atol=1e-12)
    assert np.allclose(st.v, (1 - HP.beta2) * (g * c) ** 2, rtol=2e-6, atol=1e-16)
    assert abs(fsm.grad_norm_sq - norm ** 2) <= 1e-6 * norm ** 2  # recorded before clipping


def test_clip_coefficient_carries_its_epsilon_at_tiny_norms():
    # with ||g|| ~ 1e-7 the 1e-6 in c = max_norm / (||g|| + 1e-6) dominates
    rng = np.random.default_rng(9)
    P = 100
    gh = O.float_to_half((rng.normal(0, 1e-8, P)).astype(np.float32), O.BF16)
    g = decode(gh, O.BF16).astype(np.float64)
    norm = np.sqrt(np.sum(g * g))
    max_norm = 0.5 * norm
    c = max_norm / (norm + 1e-6)
    assert c < 0.1  # far from max_norm / norm = 0.5
    st = O.State(np.zeros(P, np.float32), O.BF16)
    fsm = O.make_fsm(O.SCALE_NONE)
    O.step_ex(st, gh[None, None, :], HP, fsm, 1.0, max_norm)
    assert np.allclose(st.m, (1 - HP.beta1) * g * c, rtol=2e-6, atol=0)


def test_inactive_clip_changes_nothing():
    rng = np.random.default_rng(6)
    R, P = 2, 700
    x = rng.normal(0, 0.02, P).astype(np.float32)
    g = O.float_to_half(rng.normal(0, 1e-2, (R, P)).astype(np.float32), O.BF16)
    a, b = O.State(x, O.BF16), O.State(x, O.BF16)
    fa, fb = O.make_fsm(O.SCALE_NONE), O.make_fsm(O.SCALE_NONE)
    O.step(a, g, HP, fa)
    O.step_ex(b, g[None], HP, fb, 1.0, 1e6)
    for name in ("master", "m", "v", "param"):
        assert np.array_equal(getattr(a, name), getattr(b, name))


def test_overflow_in_any_micro_batch_skips():
    rng = np.random.default_rng(7)
    n, R, P = 3, 2, 100
    g = O.float_to_half(rng.normal(0, 1e-2, (n, R, P)).astype(np.float32) * 64, O.FP16)
    g[1, 0, 17] = 0x7C00
    st = O.State(rng.normal(0, 0.02, P).astype(np.float32), O.FP16)
    before = st.copy()
    fsm = O.make_fsm(O.SCALE_DYNAMIC, 64.0, interval=10)
    assert O.step_ex(st, g, HP, fsm, 3.0, 1.0)
    assert fsm.scale == 32.0 and fsm.t == 0
    assert np.array_equal(st.master, before.master)


@pytest.mark.parametrize("max_norm", [0.0, 0.05, 1e9])
@pytest.mark.parametrize("dtype", [O.BF16, O.FP16])
def test_step_on_a_sample_with_the_whole_norm_equals_the_whole_step(max_norm, dtype):
    # given the whole model's norm, each element's step depends on its own
    # inputs only: a sample stepped with that norm has the whole step's bytes
    rng = np.random.default_rng(40 + dtype)
    n, R, P = 2, 3, 5000
    x = rng.normal(0, 0.02, P).astype(np.float32)
    whole = O.State(x, dtype)
    fw = O.make_fsm(O.SCALE_STATIC, 4.0)
    idx = np.sort(rng.choice(P, 300, replace=False))
    part = O.State(x[idx].copy(), dtype)
    fp = O.make_fsm(O.SCALE_STATIC, 4.0)
    for _ in range(3):
        g = O.float_to_half(rng.normal(0, 1e-2, (n, R, P)).astype(np.float32) * 4.0, dtype)
        O.step_ex(whole, g, HP, fw, 2.0, max_norm)
        O.step_ex_sample(part, g[:, :, idx], HP, fp, 2.0, max_norm, fw.grad_norm_sq)
        for a in ("master", "m", "v"):
            assert np.array_equal(getattr(whole, a)[idx].view(np.uint32), getattr(part, a).view(np.uint32)), a
        assert np.array_equal(whole.param[idx], part.param)
        assert fp.grad_norm_sq == fw.grad_norm_sq and fp.t == fw.t
    # the sample's own norm instead: clipping with it changes the result
    if max_norm == 0.05:
        own = O.State(x[idx].copy(), dtype)
        fo = O.make_fsm(O.SCALE_STATIC, 4.0)
        g = O.float_to_half(rng.normal(0, 1e-2, (n, R, P)).astype(np.float32) * 4.0, dtype)
        O.step_ex(own, g[:, :, idx], HP, fo, 2.0, max_norm)
        alt = O.State(x[idx].copy(), dtype)
        fa = O.make_fsm(O.SCALE_STATIC, 4.0)
        O.step_ex_sample(alt, g[:, :, idx], HP, fa, 2.0, max_norm, fo.grad_norm_sq * 16.0)
        assert not np.array_equal(own.master, alt.master)


def test_step_on_a_sample_with_its_own_norm_is_step_ex():
    rng = np.random.default_rng(9)
    R, P = 2, 777
    x = rng.normal(0, 0.02, P).astype(np.float32)
    g = O.float_to_half(rng.normal(0, 1e-2, (1, R, P)).astype(np.float32), O.FP16)
    a, b = O.State(x, O.FP16), O.State(x, O.FP16)
    fa, fb = O.make_fsm(O.SCALE_DYNAMIC, 2.0), O.make_fsm(O.SCALE_DYNAMIC, 2.0)
    O.step_ex(a, g, HP, fa, 1.0, 0.01)
    O.step_ex_sample(b, g, HP, fb, 1.0, 0.01, fa.grad_norm_sq)
    for k in ("master", "m", "v", "param"):
        assert np.array_equal(getattr(a, k), getattr(b, k))
