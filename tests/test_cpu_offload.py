"""zero_cpu_step (ZeRO-Offload: the optimizer step on CPU cores) against the
oracle, bit for bit. Host only: these run without a GPU."""
import numpy as np
import pytest

import oracle as O
import zero_partitioned_mixed_reduce_b200 as Z

HP = dict(lr=1e-3, beta1=0.9, beta2=0.999, eps=1e-8, weight_decay=0.01)
OHP = O.AdamW(1e-3, 0.9, 0.999, 1e-8, 0.01)


class Offload:
    """Host shards of one plan, driven by zero_cpu_step, beside the oracle."""

    def __init__(self, numels, R, dtype, align, mode, scale=256.0, interval=3, seed=0):
        self.rng = np.random.default_rng(seed)
        self.lay = O.Layout(numels, R, align)
        self.plan = Z.Plan(numels, None, R, dtype, align, 0)
        self.R, self.dtype, self.mode = R, dtype, mode
        self.idx = self.lay.flat_index()
        P, T, S = self.lay.P, self.lay.T, self.lay.S
        x = self.rng.normal(0, 0.02, P).astype(np.float32)
        self.ost = O.State(x, dtype)
        flat = np.zeros(T, np.float32)
        flat[self.idx] = x
        pflat = np.zeros(T, np.uint16)
        pflat[self.idx] = self.ost.param
        self.master = [flat[r * S:(r + 1) * S].copy() for r in range(R)]
        self.m = [np.zeros(S, np.float32) for _ in range(R)]
        self.v = [np.zeros(S, np.float32) for _ in range(R)]
        self.param = [pflat[r * S:(r + 1) * S].copy() for r in range(R)]
        self.acc = [np.zeros(S, np.float32) for _ in range(R)]
        self.fsm = O.make_fsm(mode, scale=scale if mode else 1.0, interval=interval)
        self.cfg = dict(mode=mode, growth_interval=interval)
        self.ls = dict(scale=scale if mode else 1.0, cur=0, good=0, t=0)

    def step(self, n_micro=1, divisor=1.0, clip=0.0, inject=None, nthreads=0, flags=0):
        P, S = self.lay.P, self.lay.S
        g = O.float_to_half(
            (self.rng.normal(0, 1e-2, (n_micro, self.R, P)) * self.fsm.scale).astype(np.float32),
            self.dtype)
        if inject:
            g[inject] = 0x7C00 if self.dtype == O.FP16 else 0x7F80
        acc = None
        for mu in range(n_micro):
            s, _ = O.allreduce_sum(g[mu], self.dtype)
            acc = s if acc is None else acc + s
        flat = np.zeros(self.lay.T, np.float32)
        flat[self.idx] = acc
        for r in range(self.R):
            self.acc[r][:] = flat[r * S:(r + 1) * S]
        self.ls = Z.zero_cpu_step(self.plan.handle, self.cfg, self.ls, HP, self.acc, self.master,
                                  self.m, self.v, self.param, divisor, clip, nthreads, flags)
        O.step_ex(self.ost, g, OHP, self.fsm, divisor, clip)

    def compare(self):
        cat = lambda xs: np.concatenate(xs)[self.idx]
        for name, a, b in (("master", cat(self.master), self.ost.master), ("m", cat(self.m), self.ost.m),
                           ("v", cat(self.v), self.ost.v)):
            assert np.array_equal(a.view(np.uint32), b.view(np.uint32)), name
        assert np.array_equal(cat(self.param), self.ost.param)
        f, o = self.ls, self.fsm
        assert (f["t"], f["good"], f["last_overflow"], f["last_skipped"]) == \
               (o.t, o.good, o.last_overflow, o.last_skipped)
        assert np.float32(f["scale"]) == np.float32(o.scale)
        if np.isfinite(o.grad_norm_sq):
            assert abs(f["grad_norm_sq"] - o.grad_norm_sq) <= 1e-9 * o.grad_norm_sq
        else:
            assert not np.isfinite(f["grad_norm_sq"])


@pytest.mark.parametrize("R", [1, 2, 3, 8])
@pytest.mark.parametrize("dtype", [O.BF16, O.FP16])
@pytest.mark.parametrize("mode", [O.SCALE_NONE, O.SCALE_STATIC, O.SCALE_DYNAMIC])
@pytest.mark.parametrize("align", [1, 8])
def test_cpu_step_matches_oracle(R, dtype, mode, align):
    rng = np.random.default_rng(R * 10 + dtype)
    numels = rng.integers(1, 50_000, 5).tolist()
    o = Offload(numels, R, dtype, align, mode, seed=R + 7 * mode)
    for _ in range(3):
        o.step()
        o.compare()


@pytest.mark.parametrize("n_micro,divisor,clip", [(2, 2.0, 0.0), (3, 3.0, 1e-3), (1, 1.0, 1e9)])
def test_cpu_step_accumulation_and_clipping(n_micro, divisor, clip):
    o = Offload([120_000, 77, 3], 4, O.BF16, 8, O.SCALE_NONE, seed=3)
    for _ in range(3):
        o.step(n_micro, divisor, clip)
        o.compare()


def test_cpu_step_skips_on_overflow_and_recovers():
    o = Offload([30_000, 500], 2, O.FP16, 8, O.SCALE_DYNAMIC, scale=1024.0, interval=2, seed=5)
    o.step()
    o.compare()
    before = [x.copy() for x in o.master]
    o.step(inject=(0, 1, 123))
    o.compare()
    assert o.ls["last_skipped"] == 1 and o.ls["scale"] == 512.0
    assert all(np.array_equal(a, b) for a, b in zip(before, o.master))
    for _ in range(3):
        o.step()
        o.compare()


def test_thread_count_does_not_change_the_state():
    a = Offload([200_000, 1234], 4, O.FP16, 8, O.SCALE_DYNAMIC, seed=9)
    b = Offload([200_000, 1234], 4, O.FP16, 8, O.SCALE_DYNAMIC, seed=9)
    for _ in range(2):
        a.step(nthreads=1)
        b.step(nthreads=7)
    for x, y in zip(a.master + a.m + a.v, b.master + b.m + b.v):
        assert np.array_equal(x.view(np.uint32), y.view(np.uint32))
    for x, y in zip(a.param, b.param):
        assert np.array_equal(x, y)
    assert abs(a.ls["grad_norm_sq"] - b.ls["grad_norm_sq"]) <= 1e-12 * a.ls["grad_norm_sq"]


@pytest.mark.parametrize("dtype", [O.BF16, O.FP16])
def test_half_encoding_over_many_bit_patterns(dtype):
    # lr = 0 and wd = 0 leave master unchanged, so param must equal the
    # oracle's encoding of arbitrary fp32 values, subnormal and overflowing ones included
    rng = np.random.default_rng(12)
    n = 1 << 21
    bits = rng.integers(0, 1 << 32, n, dtype=np.uint64).astype(np.uint32)
    special = np.array([0x00000001, 0x33000000, 0x33000001, 0x337FFFFF, 0x387FE000, 0x387FF000,
                        0x38800000, 0x477FEFFF, 0x477FF000, 0x7F7FFFFF, 0x80000001, 0xB3800000,
                        0x00800000, 0x007FFFFF, 0x7F800000, 0xFF800000], np.uint32)
    bits[:special.size] = special
    x = bits.view(np.float32)
    x = np.where(np.isnan(x), np.float32(0.5), x).astype(np.float32)
    plan = Z.Plan([n], None, 1, dtype, 8, 0)
    master = [x.copy()]
    param = [np.zeros(n, np.uint16)]
    zeros = [np.zeros(n, np.float32) for _ in range(3)]
    hp = dict(lr=0.0, beta1=0.9, beta2=0.999, eps=1e-8, weight_decay=0.0)
    Z.zero_cpu_step(plan.handle, dict(mode=0), dict(scale=1.0, cur=0, good=0, t=0), hp, [zeros[0]],
                    master, [zeros[1]], [zeros[2]], param)
    assert np.array_equal(master[0].view(np.uint32), x.view(np.uint32))
    assert np.array_equal(param[0], O.float_to_half(x, dtype))


def test_cpu_step_argument_errors():
    plan = Z.Plan([100], None, 2, O.BF16, 8, 0)
    buf = [np.zeros(plan.S, np.float32) for _ in range(2)]
    half = [np.zeros(plan.S, np.uint16) for _ in range(2)]
    with pytest.raises(Z.ZeroError):
        Z.zero_cpu_step(plan.handle, dict(mode=0), dict(scale=1.0, t=0), HP, buf, buf, buf, buf, half,
                        grad_divisor=0.5)
    with pytest.raises(Z.ZeroError):
        Z.zero_cpu_step(plan.handle, dict(mode=0), dict(scale=1.0, t=0),
                        dict(HP, beta1=1.0), buf, buf, buf, buf, half)


@pytest.mark.parametrize("dtype", [O.BF16, O.FP16])
@pytest.mark.parametrize("mode", [O.SCALE_NONE, O.SCALE_DYNAMIC])
@pytest.mark.parametrize("clip", [0.0, 1e-3])
def test_split_cpu_step_equals_cpu_step(dtype, mode, clip):
    # scan, then the update in uneven ranges in shuffled order, then commit:
    # the same bytes and loss-scale state as zero_cpu_step (and the oracle)
    a = Offload([200_000, 77, 4096], 4, dtype, 8, mode, seed=21)
    b = Offload([200_000, 77, 4096], 4, dtype, 8, mode, seed=21)
    rng = np.random.default_rng(3)
    for step in range(4):
        inject = (0, 1, 123) if (step == 2 and mode == O.SCALE_DYNAMIC) else None
        a.step(1, 1.0, clip, inject)
        a.compare()
        # b: the same gradients as a drew (same seed sequence), split path
        g = O.float_to_half((b.rng.normal(0, 1e-2, (1, b.R, b.lay.P)) * b.fsm.scale).astype(np.float32), dtype)
        if inject:
            g[inject] = 0x7C00 if dtype == O.FP16 else 0x7F80
        s_, _ = O.allreduce_sum(g[0], dtype)
        flat = np.zeros(b.lay.T, np.float32)
        flat[b.idx] = s_
        S = b.lay.S
        for r in range(b.R):
            b.acc[r][:] = flat[r * S:(r + 1) * S]
        d = Z.zero_cpu_scan(b.plan.handle, b.cfg, b.ls, b.acc, 1.0, clip)
        cuts = np.sort(rng.choice(np.arange(1, S), 5, replace=False))
        ranges = list(zip(np.concatenate([[0], cuts]), np.concatenate([cuts, [S]])))
        rng.shuffle(ranges)
        for lo, hi in ranges:
            Z.zero_cpu_update(b.plan.handle, b.ls, HP, d, b.acc, b.master, b.m, b.v, b.param, int(lo), int(hi))
        b.ls = Z.zero_cpu_commit(b.cfg, b.ls, d)
        O.step_ex(b.ost, g, OHP, b.fsm, 1.0, clip)
        b.compare()
        for x, y in zip(a.master + a.m + a.v, b.master + b.m + b.v):
            assert np.array_equal(x.view(np.uint32), y.view(np.uint32))
        for x, y in zip(a.param, b.param):
            assert np.array_equal(x, y)


def test_cpu_update_range_errors():
    plan = Z.Plan([100], None, 2, O.BF16, 8, 0)
    buf = [np.zeros(plan.S, np.float32) for _ in range(2)]
    half = [np.zeros(plan.S, np.uint16) for _ in range(2)]
    ls = dict(scale=1.0, t=0)
    d = Z.zero_cpu_scan(plan.handle, dict(mode=0), ls, buf)
    with pytest.raises(Z.ZeroError) as e:
        Z.zero_cpu_update(plan.handle, ls, HP, d, buf, buf, buf, buf, half, 0, plan.S + 1)
    assert e.value.status == Z.ZERO_ERR_RANGE
    with pytest.raises(Z.ZeroError):
        Z.zero_cpu_update(plan.handle, ls, HP, d, buf, buf, buf, buf, half, 5, 4)


def test_concurrent_cpu_steps_from_two_host_threads():
    # the library keeps one pool of worker threads; a step that finds it busy
    # runs on threads of its own. Both ways give the bytes of a lone step.
    import threading
    base = Offload([300_000, 4099], 4, O.BF16, 8, O.SCALE_DYNAMIC, seed=5)
    base.step()
    init = [[x.copy() for x in xs] for xs in (base.acc, base.master, base.m, base.v, base.param)]

    def run(out, k):
        acc, master, m, v, param = [[x.copy() for x in xs] for xs in init]
        ls = dict(base.ls)
        for _ in range(k):
            ls = Z.zero_cpu_step(base.plan.handle, base.cfg, ls, HP, acc, master, m, v, param, 1.0, 0.0, 4)
        out.append((master, m, v, param, ls))

    lone = []
    run(lone, 6)
    results = [[] for _ in range(3)]
    threads = [threading.Thread(target=run, args=(results[i], 6)) for i in range(3)]
    for t in threads:
        t.start()
    for t in threads:
        t.join()
    for res in results:
        (master, m, v, param, ls), = res
        for x, y in zip(master + m + v, lone[0][0] + lone[0][1] + lone[0][2]):
            assert np.array_equal(x.view(np.uint32), y.view(np.uint32))
        for x, y in zip(param, lone[0][3]):
            assert np.array_equal(x, y)
        assert ls == lone[0][4]


def test_random_configurations_match_oracle():
    # property check over random configurations: tensor lists, R, dtype,
    # alignment, loss-scale mode, micro-batches with their divisor, clipping,
    # thread count; every step bit for bit against the oracle. Sizes straddle
    # the one-thread threshold (65,536 elements) and the 2,048-element blocks.
    from hypothesis import HealthCheck, given, settings, strategies as st

    @settings(max_examples=25, deadline=None, suppress_health_check=list(HealthCheck))
    @given(numels=st.lists(st.integers(1, 40_000), min_size=1, max_size=5),
           R=st.integers(1, 6), dtype=st.sampled_from([O.BF16, O.FP16]), align=st.sampled_from([1, 8]),
           mode=st.sampled_from([O.SCALE_NONE, O.SCALE_STATIC, O.SCALE_DYNAMIC]),
           n_micro=st.integers(1, 3), clip=st.sampled_from([0.0, 1e-3, 1e9]),
           nthreads=st.sampled_from([0, 1, 3]), seed=st.integers(0, 2**16))
    def check(numels, R, dtype, align, mode, n_micro, clip, nthreads, seed):
        o = Offload(numels, R, dtype, align, mode, seed=seed)
        for _ in range(2):
            o.step(n_micro, float(n_micro), clip, None, nthreads)
            o.compare()

    check()


@pytest.mark.parametrize("R,dtype", [(1, O.FP16), (3, O.BF16), (8, O.FP16)])
def test_dynamic_step_known_clean_runs_in_one_pass(R, dtype):
    # ZERO_STEP_CLEAN: the caller knows no accumulator overflowed (the GPU's
    # flag), so a DYNAMIC step needs no scan first; the result is the oracle's
    o = Offload([40_000, 17, 9999], R, dtype, 8, O.SCALE_DYNAMIC, interval=2, seed=R + 90)
    for s in range(4):
        o.step(divisor=2.0 if s == 2 else 1.0, flags=Z.ZERO_STEP_CLEAN)
        o.compare()
    assert o.fsm.t == 4 and o.fsm.scale == 1024.0  # grew twice at interval 2


def test_clean_claim_contradicted_is_refused():
    o = Offload([30_000, 5], 2, O.FP16, 8, O.SCALE_DYNAMIC, seed=95)
    o.step()
    before = dict(o.ls)
    with pytest.raises(Z.ZeroError) as e:
        o.step(inject=(0, 1, 7), flags=Z.ZERO_STEP_CLEAN)
    assert e.value.status == Z.ZERO_ERR_STATE
    assert o.ls == before  # the loss-scale state did not advance


def test_cpu_step_rejects_gpu_step_flags():
    o = Offload([1000], 1, O.BF16, 8, O.SCALE_NONE, seed=96)
    with pytest.raises(Z.ZeroError) as e:
        o.step(flags=Z.ZERO_STEP_PUSH_PARAMS)
    assert e.value.status == Z.ZERO_ERR_INVALID_ARG
