"""ZeRO-Offload on the GPU: gradients reduce-scattered on the GPU, copied to
pinned host memory, the optimizer step run by zero_cpu_step on CPU threads,
and the half parameters copied back -- run serialized and with the one-step
delayed parameter update (the CPU step of step s overlapping step s+1's GPU
work). The optimizer sees the same gradients either way, so the host state
and the GPU parameters must equal the oracle's bit for bit."""
import threading

import numpy as np
import pytest
import torch

import oracle as O

pytestmark = pytest.mark.gpu

if torch.cuda.is_available():
    import zero_partitioned_mixed_reduce_b200 as Z
    import synth
    from gpu_harness import u16

HALF = {0: torch.bfloat16, 1: torch.float16}


class OffloadRun:
    def __init__(self, numels, R, dtype, mode, scale=512.0, interval=3):
        self.wl = synth.custom_workload(numels, R, dtype, mode, scale, interval, sigma=1e-2, index=31)
        self.lay = O.Layout(numels, R, 8)
        self.plan = Z.Plan(numels, None, R, dtype, 8, 0)
        self.R, self.dtype, self.mode = R, dtype, mode
        S, T = self.plan.S, self.plan.T
        self.idx = self.lay.flat_index()
        x = synth.flat_master(self.wl, "cpu")
        p0 = x.to(HALF[dtype])
        self.ost = O.State(x.numpy(), dtype, u16(p0))
        self.fsm = O.make_fsm(mode, scale=scale if mode else 1.0, interval=interval)
        mflat = self.plan.pack(x, fill=0.0)
        pflat = self.plan.pack(p0, fill=0)
        pin = lambda t: t.pin_memory()
        self.master = [pin(mflat[r * S:(r + 1) * S].clone()) for r in range(R)]
        self.m = [pin(torch.zeros(S)) for _ in range(R)]
        self.v = [pin(torch.zeros(S)) for _ in range(R)]
        self.param_host = [pin(pflat[r * S:(r + 1) * S].clone()) for r in range(R)]
        self.acc_host = [[pin(torch.zeros(S)) for _ in range(R)] for _ in range(2)]  # double buffer
        self.param_gpu = [self.param_host[r].cuda() for r in range(R)]
        self.acc_gpu = [torch.zeros(S, device="cuda") for _ in range(R)]
        self.grads = [torch.zeros(T, dtype=HALF[dtype], device="cuda") for _ in range(R)]
        self.ctx = Z.zero_ctx_create(self.plan.handle, mode, scale, interval)
        self.cfg = dict(mode=mode, growth_interval=interval)
        self.ls = dict(scale=scale if mode else 1.0, cur=0, good=0, t=0)
        self.copy = torch.cuda.Stream()
        self.step_no = 0
        self.up_ev = None
        self.pipelined = False
        self.hp = self.wl["hp"]
        self.ohp = O.AdamW(*(self.hp[k] for k in ("lr", "beta1", "beta2", "eps", "weight_decay")))

    def gpu_half(self, slot):
        """GPU part of a step: grads, reduce-scatter, D2H of the accumulators
        into host buffer `slot`. Returns the event marking the copy."""
        self.step_no += 1
        scale = self.ls_scale_for_grads
        g = np.stack([u16(synth.flat_grads(self.wl, self.step_no, r, scale, "cpu")) for r in range(self.R)])
        for r in range(self.R):
            gp = np.zeros(self.plan.T, np.uint16)
            gp[self.idx] = g[r]
            self.grads[r].view(torch.int16).copy_(torch.from_numpy(gp.view(np.int16)))
        Z.zero_reduce_scatter_bucket(self.ctx, -1, self.grads, self.acc_gpu)
        ev = torch.cuda.Event()
        ev.record()
        self.copy.wait_event(ev)
        with torch.cuda.stream(self.copy):
            for r in range(self.R):
                self.acc_host[slot][r].copy_(self.acc_gpu[r], non_blocking=True)
        done = torch.cuda.Event()
        done.record(self.copy)
        # the next reduce-scatter may not overwrite the accumulators mid-copy
        torch.cuda.current_stream().wait_event(done)
        return g, done

    def cpu_half(self, slot, done):
        done.synchronize()
        if self.up_ev is not None:
            self.up_ev.synchronize()  # the last upload has finished reading param_host
        if not self.pipelined:
            self.ls = Z.zero_cpu_step(self.plan.handle, self.cfg, self.ls, self.hp, self.acc_host[slot],
                                      self.master, self.m, self.v, self.param_host, nthreads=0)
            return
        # scan, then the update range by range, each range uploaded while the next updates
        S = self.plan.S
        dec = Z.zero_cpu_scan(self.plan.handle, self.cfg, self.ls, self.acc_host[slot])
        for i in range(5):
            lo, hi = S * i // 5, S * (i + 1) // 5
            Z.zero_cpu_update(self.plan.handle, self.ls, self.hp, dec, self.acc_host[slot], self.master,
                              self.m, self.v, self.param_host, lo, hi)
            with torch.cuda.stream(self.copy):
                for r in range(self.R):
                    self.param_gpu[r][lo:hi].copy_(self.param_host[r][lo:hi], non_blocking=True)
        self.ls = Z.zero_cpu_commit(self.cfg, self.ls, dec)
        self.pipe_ev = torch.cuda.Event()
        self.pipe_ev.record(self.copy)

    def upload(self):
        if self.pipelined:  # the ranges are already queued
            self.up_ev = self.pipe_ev
            return
        with torch.cuda.stream(self.copy):
            for r in range(self.R):
                self.param_gpu[r].copy_(self.param_host[r], non_blocking=True)
        self.up_ev = torch.cuda.Event()
        self.up_ev.record(self.copy)

    def run(self, steps, delayed):
        """With delayed=True the CPU step of step s runs in a thread while the
        GPU half of step s+1 is issued (one-step delayed parameter update)."""
        pending = None
        for s in range(steps):
            if self.mode == O.SCALE_DYNAMIC and delayed and pending is not None:
                # the next step's backward must know the loss scale: wait for the
                # previous decision, as the host loop of a delayed update does
                pending[0].join()
                self.upload()
                pending = None
            self.ls_scale_for_grads = self.ls["scale"] if self.mode else 1.0
            g, done = self.gpu_half(s % 2)
            O.step(self.ost, g, self.ohp, self.fsm)
            if pending is not None:
                pending[0].join()
                self.upload()
            th = threading.Thread(target=self.cpu_half, args=(s % 2, done))
            th.start()
            if delayed:
                pending = (th,)
            else:
                th.join()
                self.upload()
        if pending is not None:
            pending[0].join()
            self.upload()
        torch.cuda.synchronize()

    def compare(self):
        cat = lambda xs: torch.cat(xs).numpy()[self.idx]
        for name, a, b in (("master", cat(self.master), self.ost.master), ("m", cat(self.m), self.ost.m),
                           ("v", cat(self.v), self.ost.v)):
            assert np.array_equal(a.view(np.uint32), b.view(np.uint32)), name
        assert np.array_equal(u16(torch.cat(self.param_gpu))[self.idx], self.ost.param)
        assert (self.ls["t"], self.ls["last_skipped"]) == (self.fsm.t, self.fsm.last_skipped)
        assert np.float32(self.ls["scale"]) == np.float32(self.fsm.scale)

    def close(self):
        Z.zero_ctx_destroy(self.ctx)


@pytest.mark.parametrize("delayed", [False, True])
@pytest.mark.parametrize("pipelined", [False, True])
@pytest.mark.parametrize("R,dtype,mode", [(2, O.BF16, O.SCALE_NONE), (8, O.FP16, O.SCALE_DYNAMIC),
                                          (3, O.FP16, O.SCALE_STATIC)])
def test_offload_pipeline_matches_oracle(delayed, pipelined, R, dtype, mode):
    o = OffloadRun([200_001, 77, 4096, 3], R, dtype, mode)
    o.pipelined = pipelined
    try:
        o.run(5, delayed)
        o.compare()
    finally:
        o.close()


def test_take_overflow_hands_the_flag_to_the_cpu_step():
    # the reduce-scatters' overflow flag, taken and cleared, lets a DYNAMIC
    # CPU step run in one pass (ZERO_STEP_CLEAN) when it reads 0; an inf sets
    # it, and the scan-first step then skips as the oracle does
    run = OffloadRun([30_000, 13, 4099], 2, O.FP16, O.SCALE_DYNAMIC, interval=2)
    flag = torch.zeros(1, dtype=torch.int32, device="cuda")
    try:
        for step in range(1, 5):
            run.step_no += 1
            g = np.stack([u16(synth.flat_grads(run.wl, run.step_no, r, run.fsm.scale, "cpu"))
                          for r in range(run.R)])
            if step == 2:
                g[1, 5] = 0x7C00
            for r in range(run.R):
                gp = np.zeros(run.plan.T, np.uint16)
                gp[run.idx] = g[r]
                run.grads[r].view(torch.int16).copy_(torch.from_numpy(gp.view(np.int16)))
            Z.zero_reduce_scatter_bucket(run.ctx, -1, run.grads, run.acc_gpu)
            Z.zero_take_overflow(run.ctx, flag)
            for r in range(run.R):
                run.acc_host[0][r].copy_(run.acc_gpu[r])
            f = int(flag.item())
            assert f == (1 if step == 2 else 0), step
            Z.zero_take_overflow(run.ctx, flag)
            assert int(flag.item()) == 0  # taken: cleared
            run.ls = Z.zero_cpu_step(run.plan.handle, run.cfg, run.ls, run.hp, run.acc_host[0], run.master,
                                     run.m, run.v, run.param_host, flags=0 if f else Z.ZERO_STEP_CLEAN)
            O.step(run.ost, g, run.ohp, run.fsm)
            cat = lambda xs: torch.cat(xs).numpy()[run.idx]
            assert np.array_equal(cat(run.master).view(np.uint32), run.ost.master.view(np.uint32)), step
            assert np.array_equal(u16(torch.cat(run.param_host))[run.idx], run.ost.param), step
            assert (run.ls["t"], run.ls["last_skipped"], run.ls["scale"]) == \
                (run.fsm.t, run.fsm.last_skipped, run.fsm.scale), step
    finally:
        Z.zero_ctx_destroy(run.ctx)


@pytest.mark.parametrize("divisor", [1.0, 2.0])
def test_clipped_offload_step_reads_the_host_accumulators_once(divisor):
    # with clipping the CPU step needs the global norm before its first
    # update; the reduce-scatters take it on the device as they write the
    # accumulators (ZERO_RS_NORM, the context holding the host's loss scale
    # and the step's divisor), zero_take_overflow hands over the flag, and
    # zero_cpu_decide turns the two into the decision: zero_cpu_update then
    # reads every host accumulator once, with no scan first
    run = OffloadRun([30_000, 13, 4099], 4, O.FP16, O.SCALE_DYNAMIC, interval=2)
    flag = torch.zeros(1, dtype=torch.int32, device="cuda")
    part = torch.zeros(2, dtype=torch.float64, device="cuda")
    acc_list = list(run.acc_gpu)
    S, R = run.plan.S, run.R
    clip = 1e-3  # below the gradients' norm: every applied step clips
    Z.zero_ctx_set_grad_divisor(run.ctx, divisor)
    try:
        for step in range(1, 6):
            run.step_no += 1
            g = np.stack([u16(synth.flat_grads(run.wl, run.step_no, r, run.fsm.scale, "cpu")) for r in range(R)])
            if step == 3:
                g[2, 17] = 0x7C00
            for r in range(R):
                gp = np.zeros(run.plan.T, np.uint16)
                gp[run.idx] = g[r]
                run.grads[r].view(torch.int16).copy_(torch.from_numpy(gp.view(np.int16)))
            Z.zero_loss_scale(run.ctx, Z.ZERO_LOSS_SCALE_SET, run.ls)  # the host's scale on the device
            Z.zero_reduce_scatter_shard(run.ctx, -1, run.grads, acc_list, 0, R, Z.ZERO_RS_NORM)
            Z.zero_grad_norm_shard(run.ctx, None, None, 0, R, part, divisor)
            Z.zero_take_overflow(run.ctx, flag)
            for r in range(R):
                run.acc_host[0][r].copy_(run.acc_gpu[r])
            reduced = (float(part[0].item()), float(flag.item()))
            dec = Z.zero_cpu_decide(run.plan.handle, run.cfg, run.ls, reduced, divisor, clip)
            Z.zero_cpu_update(run.plan.handle, run.ls, run.hp, dec, run.acc_host[0], run.master, run.m, run.v,
                              run.param_host, 0, S)
            run.ls = Z.zero_cpu_commit(run.cfg, run.ls, dec)
            O.step_ex(run.ost, g[None], run.ohp, run.fsm, divisor, clip)
            assert bool(dec.skip) == (step == 3)
            if step != 3:
                assert dec.clip < 1.0
                assert abs(dec.grad_norm_sq - run.fsm.grad_norm_sq) <= 1e-9 * run.fsm.grad_norm_sq
            cat = lambda xs: torch.cat(xs).numpy()[run.idx]
            for name, a, b in (("master", cat(run.master), run.ost.master), ("m", cat(run.m), run.ost.m),
                               ("v", cat(run.v), run.ost.v)):
                assert np.array_equal(a.view(np.uint32), b.view(np.uint32)), (name, step)
            assert np.array_equal(u16(torch.cat(run.param_host))[run.idx], run.ost.param), step
            assert (run.ls["t"], run.ls["last_skipped"], run.ls["scale"]) == \
                (run.fsm.t, run.fsm.last_skipped, run.fsm.scale), step
    finally:
        Z.zero_ctx_destroy(run.ctx)
