"""GPU parity at the full workload sizes, in the launch configuration the
benchmark times. The whole step runs on the GPU; the oracle recomputes a
sample of elements one by one from the same input bytes (the step is
elementwise once the global overflow decision is known, and the sample
always contains the injected overflow element, while no other element can
overflow by construction). Properties checked at full size: the layout
matches the oracle's, the squared gradient norm matches a float64 torch
recomputation, and each gathered layer equals the concatenated shards.
"""
import gc

import numpy as np
import pytest
import torch

import oracle as O

pytestmark = pytest.mark.gpu

if torch.cuda.is_available():
    import zero_partitioned_mixed_reduce_b200 as Z
    import synth
    from gpu_harness import u16, f32bits

HALF = {0: torch.bfloat16, 1: torch.float16}


def layout_matches(plan, lay):
    assert (plan.P, plan.L, plan.S, plan.T) == (lay.P, lay.L, lay.S, lay.T)
    assert plan.offsets == lay.offsets.tolist()
    assert plan.buckets == lay.buckets and plan.layers == lay.layers


def write_flat(shards, S, off, values):
    """Copy `values` into the sharded flat buffer at flat offset `off`."""
    n = values.numel()
    pos = 0
    while pos < n:
        r, j = divmod(off + pos, S)
        k = min(n - pos, S - j)
        shards[r][j:j + k].copy_(values[pos:pos + k])
        pos += k


def read_flat(shards, S, padded_idx):
    """Gather elements at padded flat indices from a sharded buffer (to CPU)."""
    idx = torch.from_numpy(padded_idx)
    r = idx // S
    out = torch.empty(len(padded_idx), dtype=shards[0].dtype)
    for rr in torch.unique(r).tolist():
        sel = (r == rr).nonzero().flatten()
        j = (idx[sel] - rr * S).to(shards[0].device)
        out[sel] = shards[rr].index_select(0, j).cpu()
    return out


class Workload:
    """path: "pingpong", "inplace", "twopass", or "twopass_clip" (two-pass,
    global-norm clipping at `clip` with the norm taken by the reduce-scatters;
    the oracle steps the sample with the whole model's norm)."""

    def __init__(self, name, path, sample=1 << 16, clip=0.0, extra=None):
        self.wl = wl = synth.workload(name) if isinstance(name, str) else name
        self.path, self.clip = path, clip
        self.R, self.dtype = wl["R"], wl["dtype"]
        self.lay = O.Layout(wl["numels"], wl["R"], 8, wl["bucket_elems"], wl["layer_ids"])
        self.plan = Z.Plan(wl["numels"], wl["layer_ids"], wl["R"], wl["dtype"], 8,
                           wl["bucket_elems"])
        layout_matches(self.plan, self.lay)
        self.S, self.T = self.plan.S, self.plan.T
        sets = 2 if path == "pingpong" else 1
        self.state = Z.ShardedState(self.plan, sets=sets, with_acc=path.startswith("twopass"))
        starts = np.concatenate([[0], np.cumsum(wl["numels"])[:-1]])
        # sample of unpadded indices: random, every tensor's first and last
        # element, the neighbours of every shard boundary, the injection point
        rng = np.random.default_rng(17)
        P = self.lay.P
        s = [rng.integers(0, P, sample), starts, starts + np.array(wl["numels"]) - 1]
        for r in range(1, self.R):
            b = r * self.S
            # nearest unpadded elements on both sides of the boundary
            k = np.searchsorted(self.lay.offsets, b, side="right") - 1
            for kk in (k, min(k + 1, len(starts) - 1)):
                s.append(np.array([starts[kk], starts[kk] + wl["numels"][kk] - 1]))
        inj = wl["inject"]
        if inj:
            s.append(np.array([starts[inj["tensor"]] + inj["element"]]))
        if extra is not None:
            s.append(np.asarray(extra))
        self.u = np.unique(np.concatenate(s).astype(np.int64))
        kk = np.searchsorted(starts, self.u, side="right") - 1
        self.p = (self.lay.offsets[kk] + (self.u - starts[kk])).astype(np.int64)
        # initial state, tensor by tensor on the GPU
        sh = self.state
        for k, (n, off) in enumerate(zip(wl["numels"], self.plan.offsets)):
            x = synth.tensor_master(n, wl["index"], k, "cuda")
            for kset in range(sets):
                write_flat(sh.master[kset], self.S, off, x)
                write_flat(sh.param[kset], self.S, off, x.to(HALF[self.dtype]))
        torch.cuda.synchronize()
        m0 = read_flat(sh.master[0], self.S, self.p).numpy()
        p0 = u16(read_flat(sh.param[0], self.S, self.p))
        self.ostate = O.State(m0, self.dtype, p0)
        self.ofsm = O.make_fsm(wl["mode"], scale=wl["init_scale"] if wl["mode"] else 1.0,
                               interval=wl["interval"])
        self.ctx = Z.zero_ctx_create(self.plan.handle, wl["mode"], wl["init_scale"],
                                     wl["interval"])
        self.grads = [torch.zeros(self.T, dtype=HALF[self.dtype], device="cuda")
                      for _ in range(self.R)]
        self.step_no = 0
        hp = wl["hp"]
        self.ohp = O.AdamW(hp["lr"], hp["beta1"], hp["beta2"], hp["eps"], hp["weight_decay"])

    def close(self):
        Z.zero_ctx_destroy(self.ctx)
        del self.state, self.grads
        gc.collect()
        torch.cuda.empty_cache()

    def fill_grads(self):
        wl = self.wl
        scale = self.ofsm.scale if wl["mode"] != O.SCALE_NONE else 1.0
        for r in range(self.R):
            for k, (n, off) in enumerate(zip(wl["numels"], self.plan.offsets)):
                self.grads[r][off:off + n] = synth.tensor_grads(
                    n, wl["dist"], wl["sigma"], scale, wl["dtype"], wl["index"], self.step_no,
                    r, k, "cuda")
        inj = wl["inject"]
        if inj and inj["step"] == self.step_no:
            off = self.plan.offsets[inj["tensor"]] + inj["element"]
            self.grads[inj["rank"]][off] = float("inf")

    def reference_norm(self, scale):
        """float64 torch recomputation of sum((sum_r g_r * (1/(R scale)))^2)."""
        inv = np.float32(1.0 / (self.R * scale))
        total = 0.0
        CH = 1 << 28
        for a in range(0, self.T, CH):
            acc = self.grads[0][a:a + CH].float()
            for r in range(1, self.R):
                acc = acc + self.grads[r][a:a + CH].float()
            g = (acc * float(inv)).double()
            total += float((g * g).sum())
        return total

    def step(self):
        self.step_no += 1
        self.fill_grads()
        scale_before = self.ofsm.scale if self.wl["mode"] != O.SCALE_NONE else 1.0
        sample_g = np.stack([u16(self.grads[r].index_select(0, torch.from_numpy(self.p).cuda()))
                             for r in range(self.R)])
        hp = self.wl["hp"]
        if self.path == "twopass":
            for b in range(len(self.plan.buckets)):
                Z.zero_reduce_scatter_bucket(self.ctx, b, self.grads, self.state.acc)
            Z.zero_step(self.ctx, hp, self.state.handle, None)
        elif self.path == "twopass_clip":
            for b in range(len(self.plan.buckets)):
                Z.zero_reduce_scatter_bucket_ex(self.ctx, b, self.grads, self.state.acc, Z.ZERO_RS_NORM)
            Z.zero_step_ex(self.ctx, hp, self.state.handle, None, 1.0, self.clip,
                           flags=Z.ZERO_STEP_NORM_FROM_RS)
        else:
            Z.zero_step(self.ctx, hp, self.state.handle, self.grads)
        ref_norm = self.reference_norm(scale_before)
        if self.path == "twopass_clip":
            O.step_ex_sample(self.ostate, sample_g[None], self.ohp, self.ofsm, 1.0, self.clip, ref_norm)
        else:
            O.step(self.ostate, sample_g, self.ohp, self.ofsm)
        return ref_norm

    def check(self, ref_norm):
        f = Z.zero_loss_scale(self.ctx)
        o = self.ofsm
        assert (f["t"], f["good"], f["last_overflow"], f["last_skipped"]) == \
               (o.t, o.good, o.last_overflow, o.last_skipped)
        assert np.float32(f["scale"]) == np.float32(o.scale)
        if np.isfinite(ref_norm):
            assert abs(f["grad_norm_sq"] - ref_norm) <= 1e-9 * ref_norm
        else:
            assert not np.isfinite(f["grad_norm_sq"])
        k = f["cur"] if self.state.sets == 2 else 0
        sh = self.state
        for name in ("master", "m", "v"):
            a = read_flat(getattr(sh, name)[k], self.S, self.p).numpy()
            b = getattr(self.ostate, name)
            assert np.array_equal(f32bits(a), f32bits(b)), \
                (name, int(np.sum(f32bits(a) != f32bits(b))))
        a = u16(read_flat(sh.param[k], self.S, self.p))
        assert np.array_equal(a, self.ostate.param)
        return f


def run(name, path, gather=False, steps=None, clip=0.0, extra=None):
    w = Workload(name, path, clip=clip, extra=extra)
    try:
        for _ in range(steps or w.wl["steps"]):
            ref = w.step()
            f = w.check(ref)
            if gather:
                k = f["cur"] if w.state.sets == 2 else 0
                flat = torch.cat(w.state.param[k])
                for l, (lo, hi) in enumerate(w.plan.layers):
                    out = torch.empty(hi - lo, dtype=HALF[w.dtype], device="cuda")
                    Z.zero_gather_layer(w.ctx, l, w.state.handle, out)
                    assert torch.equal(out.view(torch.int16), flat[lo:hi].view(torch.int16)), l
                # the same layers gathered in buckets of up to 64 layers per launch
                nl = len(w.plan.layers)
                for first in range(0, nl, 64):
                    ls = range(first, min(nl, first + 64))
                    outs = [torch.empty(w.plan.layers[l][1] - w.plan.layers[l][0],
                                        dtype=HALF[w.dtype], device="cuda") for l in ls]
                    Z.zero_gather_layers(w.ctx, first, outs, w.state.handle)
                    for o, l in zip(outs, ls):
                        lo, hi = w.plan.layers[l]
                        assert torch.equal(o.view(torch.int16), flat[lo:hi].view(torch.int16)), l
                    del outs
                del flat
        return w.ofsm
    finally:
        w.close()


def test_tiny_full_compare():
    # the small workload is compared element for element over every step
    from gpu_harness import Case
    wl = synth.workload("tiny")
    c = Case(wl["numels"], wl["R"], wl["dtype"], 8, wl["mode"], wl["init_scale"],
             path="inplace", sigma=wl["sigma"], layer_ids=wl["layer_ids"], seed=wl["index"])
    try:
        for _ in range(wl["steps"]):
            c.step()
            c.compare()
    finally:
        c.close()


def test_gpt2s_dynamic_with_injected_inf():
    fsm = run("gpt2s", "pingpong", gather=True)
    assert fsm.t == 9 and fsm.scale == 2.0 ** 15  # step 3 skipped and backed off


def test_gpt2s_two_pass_buckets():
    run("gpt2s", "twopass", steps=4)


def test_gpt2s_two_pass_clipped_with_the_norm_from_the_reduce_scatters():
    # the unscaled gradient's norm is about 0.4 here: a 0.1 threshold clips
    # every applied step; step 3's injected inf is still skipped
    fsm = run("gpt2s", "twopass_clip", steps=4, clip=0.1)
    assert fsm.t == 3 and fsm.scale == 2.0 ** 15
    assert fsm.grad_norm_sq > 0.1 ** 2


def test_d1p3b_with_layer_gathers():
    run("d1p3b", "inplace", gather=True)


def test_llama3b_two_pass_50M_buckets():
    run("llama3b", "twopass")


def test_llama3b_fused_pingpong_with_layer_gathers():
    # the benchmark's default configuration: 3,606,752,256 params, R = 4, bf16,
    # the fused step on ping-pong state (130 GB resident), and every layer gathered
    run("llama3b", "pingpong", gather=True)


def test_irregular_r16():
    run("irr_r16", "pingpong", gather=True)


def test_irregular_r2():
    run("irr_r2", "pingpong")


def test_shard_longer_than_2_to_the_32_staged_step():
    # R = 1 with a shard of 2^32 + 8 elements (69 GB in place): the staged
    # kernel's tile index, shard offset and tile length pass 2^32, so every
    # element past it must be updated; the sample covers the last 4104 elements
    # (the last tile holds 8) besides random ones across the whole shard, and
    # both layers (the second ends past 2^32) are gathered and compared whole
    n = 1 << 31
    wl = synth.custom_workload([n, n + 8], 1, 0, synth.NONE, 1.0, 1000, sigma=1e-4, index=31)
    wl["steps"] = 2
    p = Z.Plan(wl["numels"], None, 1, 0, 8, 0)
    tile, tps, _ = Z.zero_plan_step_tiles(p.handle)
    assert p.S == (1 << 32) + 8 and (tps - 1) * tile == 1 << 32
    del p
    run(wl, "inplace", gather=True, extra=np.arange((1 << 32) - 4096, (1 << 32) + 8))


def test_shard_longer_than_2_to_the_32_two_pass_step():
    # the same shard of 2^32 + 8 elements on the two-pass path: one
    # reduce-scatter into the fp32 accumulator, then the staged step from the
    # accumulator, whose tiles pass 2^32 like the fused step's (86 GB on the
    # device); the sample covers the last 4104 elements again
    n = 1 << 31
    wl = synth.custom_workload([n, n + 8], 1, 0, synth.NONE, 1.0, 1000, sigma=1e-4, index=32)
    wl["steps"] = 2
    run(wl, "twopass", extra=np.arange((1 << 32) - 4096, (1 << 32) + 8))
