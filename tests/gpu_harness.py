"""Helpers for the GPU parity tests: guard-banded device buffers, seeded
inputs shared by both sides, and comparison against the oracle.

Every device buffer handed to the library is a view into a larger
allocation whose guard bands (GUARD elements on each side) hold a canary
pattern; `check_guards` verifies after every launch that no kernel wrote
outside its buffer.
"""
import numpy as np
import torch

import oracle as O
import zero_partitioned_mixed_reduce_b200 as Z
import synth

GUARD = 64  # elements; keeps 32-byte alignment for fp32 and 16-byte for half
CANARY_F32 = 0x7FBADBAD  # a NaN pattern no kernel writes
CANARY_U16 = 0x7DAD

HALF = {0: torch.bfloat16, 1: torch.float16}


class Guarded:
    """Buffers of n elements with canary guard bands."""

    def __init__(self):
        self.allocs = []

    def f32(self, n):
        base = torch.empty(n + 2 * GUARD, dtype=torch.int32, device="cuda")
        base.fill_(CANARY_F32)
        self.allocs.append((base, "f32"))
        return base[GUARD:GUARD + n].view(torch.float32)

    def half(self, n, dtype):
        base = torch.empty(n + 2 * GUARD, dtype=torch.int16, device="cuda")
        base.fill_(np.int16(np.uint16(CANARY_U16).view(np.int16)))
        self.allocs.append((base, "u16"))
        return base[GUARD:GUARD + n].view(HALF[dtype])

    def check(self):
        torch.cuda.synchronize()
        for base, kind in self.allocs:
            head, tail = base[:GUARD], base[-GUARD:]
            if kind == "f32":
                ok = bool((head == CANARY_F32).all()) and bool((tail == CANARY_F32).all())
            else:
                c = int(np.uint16(CANARY_U16).view(np.int16))
                ok = bool((head == c).all()) and bool((tail == c).all())
            assert ok, "a kernel wrote into a guard band"


def u16(t: torch.Tensor) -> np.ndarray:
    return t.detach().contiguous().view(torch.int16).cpu().numpy().view(np.uint16)


def f32bits(a: np.ndarray) -> np.ndarray:
    return np.ascontiguousarray(a, np.float32).view(np.uint32)


class Case:
    """One parity case: a tensor list, R, dtype, alignment, loss-scale mode and
    path ("inplace", "pingpong", "twopass", "twopass_pp": two-pass with
    ping-pong state, "fused_acc": ping-pong state plus accumulators for the
    fused last micro-batch), run for a few steps on the GPU and in the oracle
    on the same bytes."""

    def __init__(self, numels, R, dtype, align=8, mode=O.SCALE_NONE, init_scale=1.0, interval=1000,
                 path="pingpong", bucket_elems=0, layer_ids=None, sigma=1e-2, seed=5, hp=None):
        self.wl = synth.custom_workload(numels, R, dtype, mode, init_scale, interval, sigma,
                                        layer_ids=layer_ids, bucket_elems=bucket_elems, index=seed)
        self.R, self.dtype, self.mode, self.path = R, dtype, mode, path
        self.init_scale, self.interval = init_scale, interval
        self.hp = hp or self.wl["hp"]
        self.lay = O.Layout(numels, R, align, bucket_elems, layer_ids)
        self.plan = Z.Plan(numels, layer_ids, R, dtype, align, bucket_elems)
        self.idx = self.lay.flat_index()
        S, T = self.plan.S, self.plan.T
        self.g = Guarded()
        sets = 2 if path in ("pingpong", "twopass_pp", "fused_acc") else 1
        self.sets = sets
        self.master = [[self.g.f32(S) for _ in range(R)] for _ in range(sets)]
        self.m = [[self.g.f32(S) for _ in range(R)] for _ in range(sets)]
        self.v = [[self.g.f32(S) for _ in range(R)] for _ in range(sets)]
        self.param = [[self.g.half(S, dtype) for _ in range(R)] for _ in range(sets)]
        self.acc = ([self.g.f32(S) for _ in range(R)]
                    if path.startswith("twopass") or path == "fused_acc" else None)
        self.grads = [self.g.half(T, dtype) for _ in range(R)]
        self.handle = Z.StateHandle(
            [dict(master=self.master[k], m=self.m[k], v=self.v[k], param=self.param[k])
             for k in range(sets)], self.acc)
        # initial state: fp32 master ~N(0, 0.02), half param = torch cast of it
        x = synth.flat_master(self.wl, "cpu")
        p0 = x.to(HALF[dtype])
        self.ostate = O.State(x.numpy(), dtype, u16(p0))
        mpad = self.plan.pack(x, fill=0.0)
        ppad = self.plan.pack(p0, fill=0)
        for k in range(sets):
            for r in range(R):
                sl = slice(r * S, (r + 1) * S)
                self.master[k][r].copy_(mpad[sl])
                self.param[k][r].copy_(ppad[sl])
                self.m[k][r].zero_()
                self.v[k][r].zero_()
        self.ofsm = O.make_fsm(mode, scale=init_scale if mode != O.SCALE_NONE else 1.0,
                               interval=interval)
        self.ctx = Z.zero_ctx_create(self.plan.handle, mode, init_scale, interval)
        self.step_no = 0

    def close(self):
        if self.ctx:
            Z.zero_ctx_destroy(self.ctx)
            self.ctx = None

    def make_grads(self, inject=None):
        """Seeded replicas at the current loss scale; returns (R, P) uint16."""
        scale = self.ofsm.scale if self.mode != O.SCALE_NONE else 1.0
        rows = [synth.flat_grads(self.wl, self.step_no, r, scale, "cpu") for r in range(self.R)]
        g = np.stack([u16(t) for t in rows])
        if inject:
            for (r, e, bits) in inject:
                g[r, e] = bits
        return g

    def step(self, inject=None):
        self.step_no += 1
        g = self.make_grads(inject)
        # GPU inputs: padded replicas (padding zero)
        for r in range(self.R):
            gp = np.zeros(self.plan.T, np.uint16)
            gp[self.idx] = g[r]
            self.grads[r].view(torch.int16).copy_(torch.from_numpy(gp.view(np.int16)))
        if self.path.startswith("twopass"):
            for b in range(len(self.plan.buckets)):
                Z.zero_reduce_scatter_bucket(self.ctx, b, self.grads, self.acc)
            Z.zero_step(self.ctx, self.hp, self.handle, None)
        else:
            Z.zero_step(self.ctx, self.hp, self.handle, self.grads)
        skipped = O.step(self.ostate, g, O.AdamW(**{k: self.hp[k] for k in
                                                    ("lr", "beta1", "beta2", "eps",
                                                     "weight_decay")}), self.ofsm)
        self.g.check()
        return skipped

    def step_noalloc(self, inject=None):
        """The two-pass step through zero_step_noalloc (all scratch in the
        library's static array, no context; the loss-scale state lives on
        the host in self.noalloc_ls) on set 0, against the oracle."""
        assert self.path == "inplace"
        self.step_no += 1
        g = self.make_grads(inject)
        for r in range(self.R):
            gp = np.zeros(self.plan.T, np.uint16)
            gp[self.idx] = g[r]
            self.grads[r].view(torch.int16).copy_(torch.from_numpy(gp.view(np.int16)))
        if not hasattr(self, "noalloc_ls"):
            self.noalloc_ls = dict(scale=self.init_scale if self.mode != O.SCALE_NONE else 1.0,
                                   cur=0, good=0, t=0)
        cfg = dict(mode=self.mode, growth_interval=self.interval, growth_factor=2.0,
                   backoff_factor=0.5, min_scale=1.0)
        self.noalloc_ls = Z.zero_step_noalloc(self.plan.handle, cfg, self.noalloc_ls, self.hp, self.grads,
                                              self.master[0], self.m[0], self.v[0], self.param[0])
        skipped = O.step(self.ostate, g, O.AdamW(**{k: self.hp[k] for k in
                                                    ("lr", "beta1", "beta2", "eps",
                                                     "weight_decay")}), self.ofsm)
        self.g.check()
        return skipped

    def step_ex(self, n_micro, grad_divisor=1.0, max_grad_norm=0.0, inject=None, rs_norm=False,
                whole=False, groups=None):
        """Two-pass step over n_micro accumulated micro-batches, optionally
        clipped; inject: (micro, rank, element, bits) tuples. rs_norm: the
        last micro-batch's reduce-scatters record the clipping norm
        (ZERO_RS_NORM) and the step sums their shares; whole: one
        reduce-scatter over the whole range per micro-batch; groups: (first,
        count) runs of consecutive buckets, one zero_reduce_scatter_buckets
        call each."""
        assert self.path.startswith("twopass")
        norm_flag = Z.ZERO_RS_NORM if rs_norm else 0
        if rs_norm:
            Z.zero_ctx_set_grad_divisor(self.ctx, grad_divisor)
        self.step_no += 1
        scale = self.ofsm.scale if self.mode != O.SCALE_NONE else 1.0
        micro = []
        for mu in range(n_micro):
            rows = [synth.flat_grads(self.wl, self.step_no * 100 + mu, r, scale, "cpu")
                    for r in range(self.R)]
            micro.append(np.stack([u16(t) for t in rows]))
        g = np.stack(micro)
        for (mu, r, e, bits) in inject or []:
            g[mu, r, e] = bits
        for mu in range(n_micro):
            for r in range(self.R):
                gp = np.zeros(self.plan.T, np.uint16)
                gp[self.idx] = g[mu, r]
                self.grads[r].view(torch.int16).copy_(torch.from_numpy(gp.view(np.int16)))
            flags = (Z.ZERO_RS_ACCUMULATE if mu else 0) | (norm_flag if mu == n_micro - 1 else 0)
            if groups is not None:
                for first, count in groups:
                    Z.zero_reduce_scatter_buckets(self.ctx, first, count, self.grads, self.acc, flags)
                continue
            for b in ([-1] if whole else range(len(self.plan.buckets))):
                Z.zero_reduce_scatter_bucket_ex(self.ctx, b, self.grads, self.acc, flags)
        Z.zero_step_ex(self.ctx, self.hp, self.handle, None, grad_divisor, max_grad_norm,
                       flags=Z.ZERO_STEP_NORM_FROM_RS if rs_norm else 0)
        skipped = O.step_ex(self.ostate, g, O.AdamW(**{k: self.hp[k] for k in
                                                       ("lr", "beta1", "beta2", "eps",
                                                        "weight_decay")}),
                            self.ofsm, grad_divisor, max_grad_norm)
        self.g.check()
        return skipped

    def step_fused_ex(self, grad_divisor=1.0, max_grad_norm=0.0, inject=None):
        """Fused step (zero_step_ex with the replicas) with a grad divisor
        and optional global-norm clipping; inject: (rank, element, bits)."""
        assert self.path in ("inplace", "pingpong")
        self.step_no += 1
        g = self.make_grads(inject)
        for r in range(self.R):
            gp = np.zeros(self.plan.T, np.uint16)
            gp[self.idx] = g[r]
            self.grads[r].view(torch.int16).copy_(torch.from_numpy(gp.view(np.int16)))
        Z.zero_step_ex(self.ctx, self.hp, self.handle, self.grads, grad_divisor, max_grad_norm)
        skipped = O.step_ex(self.ostate, g[None], O.AdamW(**{k: self.hp[k] for k in
                                                             ("lr", "beta1", "beta2", "eps",
                                                              "weight_decay")}),
                            self.ofsm, grad_divisor, max_grad_norm)
        self.g.check()
        return skipped

    def step_overlap(self, n_micro=1, grad_divisor=1.0, max_grad_norm=0.0, busy=None, rs_norm=False,
                     per_call=1):
        """Two-pass step whose reduce-scatters are issued by the overlap
        scheduler: each tensor's gradients are written on the caller's stream
        (after `busy` work, standing in for backward) in reverse tensor order,
        then reported ready; join; step. rs_norm: the last micro-batch's
        reduce-scatters record the clipping norm. per_call: tensors reported
        per zero_grads_ready call (a call that completes consecutive buckets
        reduces them in one launch)."""
        assert self.path.startswith("twopass")
        if rs_norm:
            Z.zero_ctx_set_grad_divisor(self.ctx, grad_divisor)
        self.step_no += 1
        scale = self.ofsm.scale if self.mode != O.SCALE_NONE else 1.0
        micro = []
        for mu in range(n_micro):
            rows = [synth.flat_grads(self.wl, self.step_no * 100 + mu, r, scale, "cpu")
                    for r in range(self.R)]
            micro.append(np.stack([u16(t) for t in rows]))
        g = np.stack(micro)
        starts = np.concatenate([[0], np.cumsum(self.lay.numels)[:-1]])
        dev = [torch.from_numpy(g[mu].view(np.int16)).cuda() for mu in range(n_micro)]
        torch.cuda.synchronize()
        for r in range(self.R):
            self.grads[r].zero_()
        nt = len(self.lay.numels)
        for mu in range(n_micro):
            for hi in range(nt, 0, -per_call):
                lo = max(0, hi - per_call)
                if busy is not None:
                    busy()
                for k in range(lo, hi):
                    off, n, st = int(self.lay.offsets[k]), int(self.lay.numels[k]), int(starts[k])
                    for r in range(self.R):
                        self.grads[r].view(torch.int16)[off:off + n].copy_(dev[mu][r, st:st + n])
                flags = (Z.ZERO_RS_ACCUMULATE if mu else 0) | \
                    (Z.ZERO_RS_NORM if rs_norm and mu == n_micro - 1 else 0)
                Z.zero_grads_ready(self.ctx, lo, hi - lo, self.grads, self.acc, flags,
                                   torch.cuda.current_stream())
            Z.zero_grads_join(self.ctx, torch.cuda.current_stream())
        Z.zero_step_ex(self.ctx, self.hp, self.handle, None, grad_divisor, max_grad_norm,
                       torch.cuda.current_stream(), flags=Z.ZERO_STEP_NORM_FROM_RS if rs_norm else 0)
        skipped = O.step_ex(self.ostate, g, O.AdamW(**{k: self.hp[k] for k in
                                                       ("lr", "beta1", "beta2", "eps",
                                                        "weight_decay")}),
                            self.ofsm, grad_divisor, max_grad_norm)
        self.g.check()
        return skipped

    def step_sharded(self, splits, inject=None):
        """The fused step done shard range by shard range (zero_step_shard),
        the per-range totals summed as a cross-rank all-reduce would, then
        zero_step_commit. splits: list of (owner_lo, owner_hi)."""
        self.step_no += 1
        g = self.make_grads(inject)
        for r in range(self.R):
            gp = np.zeros(self.plan.T, np.uint16)
            gp[self.idx] = g[r]
            self.grads[r].view(torch.int16).copy_(torch.from_numpy(gp.view(np.int16)))
        partials = [torch.full((2,), -1.0, dtype=torch.float64, device="cuda") for _ in splits]
        for (lo, hi), part in zip(splits, partials):
            Z.zero_step_shard(self.ctx, self.hp, self.handle, self.grads, lo, hi, part)
        reduced = torch.stack(partials).sum(0)
        Z.zero_step_commit(self.ctx, reduced)
        skipped = O.step(self.ostate, g, O.AdamW(**{k: self.hp[k] for k in
                                                    ("lr", "beta1", "beta2", "eps",
                                                     "weight_decay")}), self.ofsm)
        self.g.check()
        return skipped, [p.cpu().numpy() for p in partials]

    def step_fused_accum(self, n_micro, grad_divisor=1.0, inject=None):
        """Accumulation whose last micro-batch is fused into the step
        (ZERO_STEP_ADD_ACC): micro-batches 0..n-2 reduce-scattered into the
        accumulators, the last read straight from the replicas.
        inject: (micro, rank, element, bits)."""
        assert self.path == "fused_acc" and n_micro >= 2
        self.step_no += 1
        scale = self.ofsm.scale if self.mode != O.SCALE_NONE else 1.0
        g = np.stack([np.stack([u16(synth.flat_grads(self.wl, self.step_no * 100 + mu, r, scale, "cpu"))
                                for r in range(self.R)]) for mu in range(n_micro)])
        for (mu, r, e, bits) in inject or []:
            g[mu, r, e] = bits
        for mu in range(n_micro):
            for r in range(self.R):
                gp = np.zeros(self.plan.T, np.uint16)
                gp[self.idx] = g[mu, r]
                self.grads[r].view(torch.int16).copy_(torch.from_numpy(gp.view(np.int16)))
            if mu < n_micro - 1:
                for b in range(len(self.plan.buckets)):
                    Z.zero_reduce_scatter_bucket_ex(self.ctx, b, self.grads, self.acc,
                                                    Z.ZERO_RS_ACCUMULATE if mu else 0)
        Z.zero_step_ex(self.ctx, self.hp, self.handle, self.grads, grad_divisor, 0.0,
                       flags=Z.ZERO_STEP_ADD_ACC)
        skipped = O.step_ex(self.ostate, g, O.AdamW(**{k: self.hp[k] for k in
                                                       ("lr", "beta1", "beta2", "eps",
                                                        "weight_decay")}),
                            self.ofsm, grad_divisor, 0.0)
        self.g.check()
        return skipped

    def step_sharded_ex(self, splits, n_micro=1, grad_divisor=1.0, max_grad_norm=0.0, inject=None,
                        rs_norm=False):
        """The multi-rank step emulated shard range by shard range, with the
        cross-rank sums done here: fused (path "pingpong"/"inplace") or
        two-pass (paths "twopass*": per micro-batch and bucket,
        zero_reduce_scatter_shard for each range), optional global-norm
        clipping (zero_grad_norm_shard per range, summed), then
        zero_step_shard_ex per range and one zero_step_commit.
        inject: (micro, rank, element, bits). rs_norm (two-pass, clipped): each
        range's last reduce-scatters take its norm share (ZERO_RS_NORM), summed
        by zero_grad_norm_shard from the shares before the next range's
        reduce-scatters reuse the context's slots."""
        self.step_no += 1
        scale = self.ofsm.scale if self.mode != O.SCALE_NONE else 1.0
        g = np.stack([np.stack([u16(synth.flat_grads(self.wl, self.step_no * 100 + mu, r, scale, "cpu"))
                                for r in range(self.R)]) for mu in range(n_micro)])
        for (mu, r, e, bits) in inject or []:
            g[mu, r, e] = bits
        twopass = self.path.startswith("twopass")
        add_acc = self.path == "fused_acc" and n_micro > 1  # last micro-batch fused into the step
        assert twopass or add_acc or n_micro == 1
        dev = lambda: torch.zeros(2, dtype=torch.float64, device="cuda")
        rs_norm = rs_norm and twopass and max_grad_norm > 0
        if rs_norm:
            Z.zero_ctx_set_grad_divisor(self.ctx, grad_divisor)
        shares = []
        for mu in range(n_micro):
            for r in range(self.R):
                gp = np.zeros(self.plan.T, np.uint16)
                gp[self.idx] = g[mu, r]
                self.grads[r].view(torch.int16).copy_(torch.from_numpy(gp.view(np.int16)))
            if twopass or (add_acc and mu < n_micro - 1):
                last = rs_norm and mu == n_micro - 1
                for lo, hi in splits:
                    acc = [self.acc[o] if lo <= o < hi else None for o in range(self.R)]
                    flags = (Z.ZERO_RS_ACCUMULATE if mu else 0) | (Z.ZERO_RS_NORM if last else 0)
                    for b in range(len(self.plan.buckets)):
                        Z.zero_reduce_scatter_shard(self.ctx, b, self.grads, acc, lo, hi, flags)
                    if last:
                        part = dev()
                        Z.zero_grad_norm_shard(self.ctx, None, None, lo, hi, part, grad_divisor)
                        shares.append(part)
        norm = None
        if rs_norm:
            norm = torch.stack(shares).sum(0)[:1].contiguous()  # the cross-rank all-reduce
        elif max_grad_norm > 0:
            parts = []
            for lo, hi in splits:
                part = dev()
                if twopass:
                    acc = [self.acc[o] if lo <= o < hi else None for o in range(self.R)]
                    Z.zero_grad_norm_shard(self.ctx, None, acc, lo, hi, part, grad_divisor)
                else:
                    Z.zero_grad_norm_shard(self.ctx, self.grads, None, lo, hi, part, grad_divisor)
                parts.append(part)
            norm = torch.stack(parts).sum(0)[:1].contiguous()  # the cross-rank all-reduce
        partials = []
        for lo, hi in splits:
            part = dev()
            Z.zero_step_shard_ex(self.ctx, self.hp, self.handle, None if twopass else self.grads, lo, hi,
                                 part, grad_divisor, max_grad_norm, norm,
                                 flags=Z.ZERO_STEP_ADD_ACC if add_acc else 0)
            partials.append(part)
        Z.zero_step_commit(self.ctx, torch.stack(partials).sum(0))
        skipped = O.step_ex(self.ostate, g, O.AdamW(**{k: self.hp[k] for k in
                                                       ("lr", "beta1", "beta2", "eps",
                                                        "weight_decay")}),
                            self.ofsm, grad_divisor, max_grad_norm)
        self.g.check()
        return skipped

    def gpu_fsm(self):
        return Z.zero_loss_scale(self.ctx)

    def gpu_state(self, cur=None):
        cur = self.gpu_fsm()["cur"] if cur is None else cur
        k = cur if self.sets == 2 else 0
        idx = self.idx
        cat = lambda bufs: torch.cat([b for b in bufs]).cpu()
        master = cat(self.master[k]).numpy()[idx]
        m = cat(self.m[k]).numpy()[idx]
        v = cat(self.v[k]).numpy()[idx]
        param = u16(torch.cat(self.param[k]))[idx]
        pads = np.ones(self.plan.T, bool)
        pads[idx] = False
        return dict(master=master, m=m, v=v, param=param, cur=cur,
                    pad_master=cat(self.master[k]).numpy()[pads],
                    pad_param=u16(torch.cat(self.param[k]))[pads])

    def compare(self, exact=True, fsm=None):
        """Assert parity with the oracle after the last step; fsm: the
        loss-scale state to check (default: the context's)."""
        f = self.gpu_fsm() if fsm is None else fsm
        o = self.ofsm
        assert (f["t"], f["good"], f["last_overflow"], f["last_skipped"]) == \
               (o.t, o.good, o.last_overflow, o.last_skipped), (f, o.t, o.good)
        assert np.float32(f["scale"]) == np.float32(o.scale)
        if np.isfinite(o.grad_norm_sq):
            assert abs(f["grad_norm_sq"] - o.grad_norm_sq) <= 1e-9 * abs(o.grad_norm_sq) + 1e-300
        else:
            assert not np.isfinite(f["grad_norm_sq"])
        s = self.gpu_state(f["cur"])
        st = self.ostate
        for name in ("master", "m", "v"):
            a, b = s[name], getattr(st, name)
            fin = np.isfinite(b)
            assert np.array_equal(np.isfinite(a), fin), name
            rel = np.abs(a[fin].astype(np.float64) - b[fin]) / np.maximum(np.abs(b[fin]), 1e-30)
            assert rel.size == 0 or rel.max() <= 1e-5, (name, rel.max())
            if exact:
                assert np.array_equal(f32bits(a[fin]), f32bits(b[fin])), \
                    (name, int(np.sum(f32bits(a[fin]) != f32bits(b[fin]))))
        pa, pb = s["param"].astype(np.int32), st.param.astype(np.int32)
        nan_b = half_is_nan(st.param, self.dtype)
        assert np.array_equal(half_is_nan(s["param"], self.dtype), nan_b)
        # within 1 ulp: same sign and adjacent encodings
        d = np.abs(pa[~nan_b] - pb[~nan_b])
        assert d.size == 0 or d.max() <= 1
        if exact:
            assert np.array_equal(pa[~nan_b], pb[~nan_b])
        # padding stays zero
        assert np.all(s["pad_master"] == 0) and np.all(s["pad_param"] == 0)
        return s


def half_is_nan(h: np.ndarray, dtype: int) -> np.ndarray:
    """NaN encodings: all-ones exponent with a non-zero significand."""
    h = h.astype(np.uint32)
    if dtype == O.FP16:
        return ((h & 0x7C00) == 0x7C00) & ((h & 0x03FF) != 0)
    return ((h & 0x7F80) == 0x7F80) & ((h & 0x007F) != 0)
