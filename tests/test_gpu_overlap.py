"""GPU tests of the overlap / prefetch scheduler (zero_grads_ready /
zero_grads_join and zero_prefetch_begin / zero_layer_acquire /
zero_layer_release). The caller's stream is kept busy with matmuls so that
the communication stream runs ahead of it; any missing ordering (a
reduce-scatter reading gradients not yet written, a ring slot refilled before
its release) changes the results, which must equal the oracle's bit for bit."""
import numpy as np
import pytest
import torch

import oracle as O

pytestmark = pytest.mark.gpu

if torch.cuda.is_available():
    import zero_partitioned_mixed_reduce_b200 as Z
    from gpu_harness import Case, u16


def make_busy(n=1024, reps=4):
    a = torch.randn(n, n, device="cuda", dtype=torch.bfloat16)

    def busy():
        x = a
        for _ in range(reps):
            x = x @ a
        return x
    return busy


@pytest.mark.parametrize("R,dtype", [(2, O.FP16), (4, O.BF16), (8, O.FP16)])
@pytest.mark.parametrize("n_micro", [1, 2])
@pytest.mark.parametrize("comm_sms", [0, 1, 5])
def test_overlapped_reduce_scatter_matches_oracle(R, dtype, n_micro, comm_sms):
    # comm_sms caps the grid of the communication kernels; results must not
    # depend on it
    numels = [70_001, 13, 4096, 7, 999, 30_000, 5]
    mode = O.SCALE_DYNAMIC if dtype == O.FP16 else O.SCALE_NONE
    c = Case(numels, R, dtype, 8, mode, init_scale=256.0, interval=3, path="twopass",
             bucket_elems=20_000)
    busy = make_busy()
    Z.zero_sched_set_comm_sms(c.ctx, comm_sms)
    try:
        for _ in range(3):
            c.step_overlap(n_micro, float(n_micro), 0.0 if R != 4 else 0.5, busy)
            c.compare()
    finally:
        c.close()


@pytest.mark.parametrize("R,dtype", [(4, O.BF16), (8, O.FP16)])
@pytest.mark.parametrize("n_micro", [1, 3])
@pytest.mark.parametrize("comm_sms", [0, 2])
def test_overlapped_reduce_scatter_with_norm_matches_oracle(R, dtype, n_micro, comm_sms):
    # clipping whose norm the overlapped reduce-scatters take (ZERO_RS_NORM on
    # the last micro-batch): the step reads no accumulator before updating
    numels = [70_001, 13, 4096, 7, 999, 30_000, 5]
    mode = O.SCALE_DYNAMIC if dtype == O.FP16 else O.SCALE_NONE
    c = Case(numels, R, dtype, 8, mode, init_scale=256.0, interval=3, path="twopass",
             bucket_elems=20_000)
    busy = make_busy()
    Z.zero_sched_set_comm_sms(c.ctx, comm_sms)
    try:
        for clip in (1e-3, 1e9, 2e-3):
            c.step_overlap(n_micro, float(n_micro), clip, busy, rs_norm=True)
            c.compare()
    finally:
        c.close()


@pytest.mark.parametrize("per_call", [3, 8])
@pytest.mark.parametrize("rs_norm", [False, True])
def test_reports_of_several_tensors_coalesce_and_match_oracle(per_call, rs_norm):
    # a call that completes several consecutive buckets reduces them in one
    # launch; the result is the oracle's either way
    numels = [70_001, 13, 4096, 7, 999, 30_000, 5, 12_000, 800]
    c = Case(numels, 8, O.FP16, 8, O.SCALE_DYNAMIC, init_scale=256.0, interval=3, path="twopass",
             bucket_elems=5_000)
    busy = make_busy()
    try:
        for n_micro in (1, 2):
            c.step_overlap(n_micro, float(n_micro), 1e-3 if rs_norm else 0.0, busy, rs_norm=rs_norm,
                           per_call=per_call)
            c.compare()
    finally:
        c.close()


def test_grads_join_refuses_missing_and_repeated_reports():
    c = Case([100, 200, 300], 2, O.BF16, 8, O.SCALE_NONE, path="twopass", bucket_elems=250)
    try:
        Z.zero_grads_ready(c.ctx, 2, 1, c.grads, c.acc)
        with pytest.raises(Z.ZeroError) as e:
            Z.zero_grads_ready(c.ctx, 2, 1, c.grads, c.acc)
        assert e.value.status == 7
        with pytest.raises(Z.ZeroError) as e:
            Z.zero_grads_join(c.ctx)
        assert e.value.status == 7 and "not reported" in str(e.value)
        Z.zero_grads_ready(c.ctx, 0, 2, c.grads, c.acc)
        Z.zero_grads_join(c.ctx)
        with pytest.raises(Z.ZeroError) as e:
            Z.zero_grads_ready(c.ctx, 2, 2, c.grads, c.acc)
        assert e.value.status == 5
    finally:
        c.close()


@pytest.mark.parametrize("direction", [1, -1])
@pytest.mark.parametrize("nbufs,depth", [(1, 0), (2, 1), (3, 2), (4, 1)])
@pytest.mark.parametrize("align", [1, 8])
@pytest.mark.parametrize("comm_sms", [0, 2])
def test_prefetch_ring_delivers_every_layer(direction, nbufs, depth, align, comm_sms):
    numels = [3001, 17, 8, 2048, 5, 700, 1, 9000, 64, 3, 40_000, 11]
    layer_ids = [0, 0, 1, 1, 2, 2, 3, 4, 5, 5, 6, 7]
    c = Case(numels, 4, O.FP16, align, O.SCALE_DYNAMIC, 64.0, path="pingpong", layer_ids=layer_ids)
    Z.zero_sched_set_comm_sms(c.ctx, comm_sms)
    busy = make_busy(reps=8)
    try:
        for _ in range(2):
            c.step()
        c.compare()
        flat = np.zeros(c.plan.T, np.uint16)
        flat[c.idx] = c.ostate.param
        L = c.lay.layers
        biggest = max(hi - lo for lo, hi in L)
        bufs = [torch.full((biggest + 8,), -1, dtype=torch.int16, device="cuda") for _ in range(nbufs)]
        by_addr = {b.data_ptr(): b for b in bufs}
        stream = torch.cuda.current_stream()
        order = range(len(L)) if direction > 0 else reversed(range(len(L)))
        for rnd in range(2):  # two passes over the same ring
            Z.zero_prefetch_begin(c.ctx, c.handle, bufs, depth, direction, stream)
            got = {}
            for l in order if rnd == 0 else (range(len(L)) if direction > 0 else reversed(range(len(L)))):
                addr = Z.zero_layer_acquire(c.ctx, l, stream)
                busy()  # the ring slot must not be refilled while this work is queued
                lo, hi = L[l]
                got[l] = by_addr[addr][:hi - lo].clone()
                Z.zero_layer_release(c.ctx, l, stream)
            torch.cuda.synchronize()
            for l, (lo, hi) in enumerate(L):
                assert np.array_equal(u16(got[l]), flat[lo:hi]), (rnd, l)
        # a new pass must be taken in order: a layer beyond the ring is refused
        assert nbufs < len(L)
        Z.zero_prefetch_begin(c.ctx, c.handle, bufs, depth, direction, stream)
        with pytest.raises(Z.ZeroError) as e:
            Z.zero_layer_acquire(c.ctx, len(L) - 1 if direction > 0 else 0, stream)
        assert e.value.status == 7
        with pytest.raises(Z.ZeroError):
            Z.zero_prefetch_begin(c.ctx, c.handle, bufs, nbufs, direction, stream)  # depth == nbufs
    finally:
        c.close()


def test_prefetch_follows_the_step_that_produced_the_parameters():
    # the step is queued behind busy work and not synchronized before
    # zero_prefetch_begin: the gathers must still see the updated parameters
    c = Case([5000, 3000, 2000], 2, O.BF16, 8, O.SCALE_NONE, path="pingpong",
             layer_ids=[0, 1, 2])
    busy = make_busy(reps=8)
    hp = O.AdamW(*(c.hp[k] for k in ("lr", "beta1", "beta2", "eps", "weight_decay")))
    try:
        bufs = [torch.empty(5008, dtype=torch.int16, device="cuda") for _ in range(3)]
        by_addr = {b.data_ptr(): b for b in bufs}
        stream = torch.cuda.current_stream()
        for _ in range(3):
            c.step_no += 1
            g = c.make_grads()
            staged = [torch.from_numpy(np.ascontiguousarray(g[r]).view(np.int16)).cuda()
                      for r in range(c.R)]
            torch.cuda.synchronize()
            busy()
            for r in range(c.R):
                gp = torch.zeros(c.plan.T, dtype=torch.int16, device="cuda")
                gp[torch.from_numpy(c.idx).cuda()] = staged[r]
                c.grads[r].view(torch.int16).copy_(gp)
            Z.zero_step(c.ctx, c.hp, c.handle, c.grads, stream)
            Z.zero_prefetch_begin(c.ctx, c.handle, bufs, 2, 1, stream)
            outs = []
            for l in range(3):
                addr = Z.zero_layer_acquire(c.ctx, l, stream)
                lo, hi = c.lay.layers[l]
                outs.append(by_addr[addr][:hi - lo].clone())
                Z.zero_layer_release(c.ctx, l, stream)
            O.step(c.ostate, g, hp, c.ofsm)
            torch.cuda.synchronize()
            flat = np.zeros(c.plan.T, np.uint16)
            flat[c.idx] = c.ostate.param
            for l, (lo, hi) in enumerate(c.lay.layers):
                assert np.array_equal(u16(outs[l]), flat[lo:hi]), l
        c.compare()
    finally:
        c.close()
