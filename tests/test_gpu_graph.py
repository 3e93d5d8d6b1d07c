"""The step captured once into a CUDA graph and replayed. Every decision of
the step (overflow, skip, loss scale, which ping-pong set is current, the
step count behind the bias corrections) lives on the device, so replaying
one captured launch sequence must give the oracle's state bit for bit,
skipped steps included. The bias-correction table is reserved before the
capture; a capture that would have to grow it is refused on the host, and a
replay that outruns it is reported, not read past."""
import numpy as np
import pytest
import torch

import oracle as O

pytestmark = pytest.mark.gpu

if torch.cuda.is_available():
    import zero_partitioned_mixed_reduce_b200 as Z
    from gpu_harness import Case

FP16_INF = 0x7C00


def _capture(fn):
    """Capture fn(stream) into a CUDA graph on a side stream. The library
    allocates nothing during a step, so no warm-up run precedes the capture."""
    s = torch.cuda.Stream()
    s.wait_stream(torch.cuda.current_stream())
    g = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g, stream=s):
        fn(torch.cuda.current_stream())
    torch.cuda.current_stream().wait_stream(s)
    return g


def _write_grads(c, inject=None):
    """Next step's gradient replicas into the captured (static) buffers; also
    returns them for the oracle."""
    c.step_no += 1
    g = c.make_grads(inject)
    for r in range(c.R):
        gp = np.zeros(c.plan.T, np.uint16)
        gp[c.idx] = g[r]
        c.grads[r].view(torch.int16).copy_(torch.from_numpy(gp.view(np.int16)))
    return g


def _ohp(c):
    return O.AdamW(**{k: c.hp[k] for k in ("lr", "beta1", "beta2", "eps", "weight_decay")})


@pytest.mark.parametrize("R,dtype", [(1, O.BF16), (2, O.FP16), (8, O.FP16), (3, O.BF16)])
def test_replayed_fused_step_matches_oracle(R, dtype):
    mode = O.SCALE_DYNAMIC
    c = Case([70_001, 4096, 13, 9_000], R, dtype, mode=mode, init_scale=2048.0, interval=2,
             path="pingpong", seed=61)
    try:
        Z.zero_ctx_reserve_steps(c.ctx, 16, c.hp["beta1"], c.hp["beta2"])
        graph = _capture(lambda s: Z.zero_step(c.ctx, c.hp, c.handle, c.grads, s))
        bad = FP16_INF if dtype == O.FP16 else 0x7F80
        # step 3 overflows: skipped, scale halves, the ping-pong set stays
        for k in range(7):
            inject = [(R - 1, 5, bad)] if k == 2 else None
            g = _write_grads(c, inject)
            graph.replay()
            skipped = O.step(c.ostate, g, _ohp(c), c.ofsm)
            assert skipped == (k == 2)
            c.g.check()
            c.compare()
    finally:
        c.close()


@pytest.mark.parametrize("rs_norm", [False, True])
def test_replayed_two_pass_step_with_clipping_matches_oracle(rs_norm):
    # rs_norm: the reduce-scatters take the clipping norm; their per-bucket
    # counters re-arm themselves, so every replay sums fresh shares
    c = Case([50_000, 333, 8_192], 4, O.BF16, mode=O.SCALE_NONE, path="twopass",
             bucket_elems=20_000, seed=62)
    try:
        Z.zero_ctx_reserve_steps(c.ctx, 8, c.hp["beta1"], c.hp["beta2"])
        nb = len(c.plan.buckets)

        def step(s):
            for b in range(nb):
                Z.zero_reduce_scatter_bucket_ex(c.ctx, b, c.grads, c.acc, Z.ZERO_RS_NORM if rs_norm else 0, s)
            Z.zero_step_ex(c.ctx, c.hp, c.handle, None, 1.0, 1e-3, s,
                           flags=Z.ZERO_STEP_NORM_FROM_RS if rs_norm else 0)

        graph = _capture(step)
        for _ in range(4):
            g = _write_grads(c)
            graph.replay()
            O.step_ex(c.ostate, g[None], _ohp(c), c.ofsm, 1.0, 1e-3)
            c.g.check()
            c.compare()
    finally:
        c.close()


def test_replayed_step_and_gather_match_oracle():
    layers = [0, 0, 1, 2, 2]
    c = Case([10_000, 77, 30_001, 4_000, 123], 2, O.FP16, mode=O.SCALE_DYNAMIC, init_scale=512.0,
             interval=3, path="pingpong", layer_ids=layers, seed=63)
    try:
        Z.zero_ctx_reserve_steps(c.ctx, 8, c.hp["beta1"], c.hp["beta2"])
        L = c.lay.layers
        outs = [torch.zeros(int(hi - lo), dtype=torch.int16, device="cuda") for lo, hi in L]

        def step(s):
            Z.zero_step(c.ctx, c.hp, c.handle, c.grads, s)
            Z.zero_gather_layers(c.ctx, 0, outs, c.handle, s)

        graph = _capture(step)
        for k in range(5):
            g = _write_grads(c, [(0, 9, FP16_INF)] if k == 1 else None)
            graph.replay()
            O.step(c.ostate, g, _ohp(c), c.ofsm)
            s = c.compare()
            # the gathered layers are the current parameters, layer by layer
            full = np.zeros(c.plan.T, np.uint16)
            full[c.idx] = s["param"]
            got = np.concatenate([o.cpu().numpy().view(np.uint16) for o in outs])
            want = np.concatenate([full[lo:hi] for lo, hi in L])
            assert np.array_equal(got, want)
    finally:
        c.close()


def test_capture_that_must_grow_the_table_is_refused():
    c = Case([5_000], 2, O.BF16, path="pingpong", seed=64)
    try:
        s = torch.cuda.Stream()
        s.wait_stream(torch.cuda.current_stream())
        g = torch.cuda.CUDAGraph()
        with pytest.raises(Z.ZeroError):
            with torch.cuda.graph(g, stream=s):
                Z.zero_step(c.ctx, c.hp, c.handle, c.grads, torch.cuda.current_stream())
        torch.cuda.synchronize()
        # nothing was launched: the context still steps normally afterwards
        c.step()
        c.compare()
    finally:
        c.close()


def test_replay_beyond_the_reserve_is_reported():
    c = Case([1_000], 1, O.BF16, path="pingpong", seed=65)
    try:
        Z.zero_ctx_reserve_steps(c.ctx, 4, c.hp["beta1"], c.hp["beta2"])
        graph = _capture(lambda s: Z.zero_step(c.ctx, c.hp, c.handle, c.grads, s))
        _write_grads(c)
        # the smallest table holds 1024 entries; t + 1 reaches it on replay 1024
        for _ in range(1023):
            graph.replay()
        torch.cuda.synchronize()
        assert Z.zero_loss_scale(c.ctx)["t"] == 1023
        graph.replay()
        torch.cuda.synchronize()
        with pytest.raises(Z.ZeroError):
            Z.zero_loss_scale(c.ctx)
        c.g.check()
    finally:
        c.close()


@pytest.mark.parametrize("mode", [O.SCALE_DYNAMIC, O.SCALE_NONE])
def test_replayed_overlapped_step_matches_oracle(mode):
    # the scheduler's cross-stream work (reduce-scatters on the communication
    # stream as tensors are reported ready, then the join) captured with the
    # gradient writes and the step into one graph
    numels = [30_000, 77, 5_000, 12_001, 9]
    R = 4
    c = Case(numels, R, O.FP16, mode=mode, init_scale=256.0, interval=2, path="twopass",
             bucket_elems=15_000, seed=66)
    try:
        c.step_overlap()  # first use creates the scheduler's stream and events
        c.compare()
        Z.zero_ctx_reserve_steps(c.ctx, 8, c.hp["beta1"], c.hp["beta2"])
        P = c.lay.P
        starts = np.concatenate([[0], np.cumsum(c.lay.numels)[:-1]])
        dev = torch.zeros((R, P), dtype=torch.int16, device="cuda")

        def step(s):
            for r in range(R):
                c.grads[r].zero_()
            for k in reversed(range(len(numels))):
                off, n, st = int(c.lay.offsets[k]), int(c.lay.numels[k]), int(starts[k])
                for r in range(R):
                    c.grads[r].view(torch.int16)[off:off + n].copy_(dev[r, st:st + n])
                Z.zero_grads_ready(c.ctx, k, 1, c.grads, c.acc, 0, s)
            Z.zero_grads_join(c.ctx, s)
            Z.zero_step_ex(c.ctx, c.hp, c.handle, None, 1.0, 0.0, s)

        graph = _capture(step)
        for k in range(4):
            c.step_no += 1
            g = c.make_grads([(1, 40, 0x7C00)] if k == 1 else None)
            dev.copy_(torch.from_numpy(g.view(np.int16)))
            graph.replay()
            skipped = O.step(c.ostate, g, _ohp(c), c.ofsm)
            assert skipped == (k == 1 and mode == O.SCALE_DYNAMIC)
            c.g.check()
            c.compare()
    finally:
        c.close()


def test_replayed_zero3_training_step_matches_oracle():
    # a whole ZeRO-3 step in one graph: forward through the look-ahead gather
    # ring, backward through it in reverse with each layer's gradients written
    # and reported (reduce-scatters on the communication stream), the join and
    # the step; replays must follow the oracle, and every gathered layer must
    # equal the parameters of the step before
    numels = [30_000, 77, 5_000, 12_001, 9, 4_096]
    layer_ids = [0, 0, 1, 2, 2, 3]
    R = 4
    c = Case(numels, R, O.FP16, mode=O.SCALE_DYNAMIC, init_scale=256.0, interval=2, path="twopass_pp",
             bucket_elems=15_000, layer_ids=layer_ids, seed=67)
    try:
        c.step_overlap()  # first use creates the scheduler's stream and events
        c.compare()
        Z.zero_ctx_reserve_steps(c.ctx, 8, c.hp["beta1"], c.hp["beta2"])
        L = c.lay.layers
        nl = len(L)
        biggest = max(hi - lo for lo, hi in L)
        ring = [torch.empty(biggest + 8, dtype=torch.int16, device="cuda") for _ in range(2)]
        seen = [torch.empty(hi - lo, dtype=torch.int16, device="cuda") for lo, hi in L]
        by_addr = {b.data_ptr(): b for b in ring}
        P = c.lay.P
        starts = np.concatenate([[0], np.cumsum(c.lay.numels)[:-1]])
        first_t = [layer_ids.index(l) for l in range(nl)]
        count_t = [layer_ids.count(l) for l in range(nl)]
        dev = torch.zeros((R, P), dtype=torch.int16, device="cuda")

        def step(s):
            Z.zero_prefetch_begin(c.ctx, c.handle, ring, 1, 1, s)
            for l in range(nl):  # forward: use (here: keep a copy of) each gathered layer
                buf = by_addr[Z.zero_layer_acquire(c.ctx, l, s)]
                seen[l].copy_(buf[:L[l][1] - L[l][0]])
                Z.zero_layer_release(c.ctx, l, s)
            for r in range(R):
                c.grads[r].zero_()
            Z.zero_prefetch_begin(c.ctx, c.handle, ring, 1, -1, s)
            for l in reversed(range(nl)):  # backward: gradients of the layer's tensors
                Z.zero_layer_acquire(c.ctx, l, s)
                for k in range(first_t[l], first_t[l] + count_t[l]):
                    off, n, st = int(c.lay.offsets[k]), int(c.lay.numels[k]), int(starts[k])
                    for r in range(R):
                        c.grads[r].view(torch.int16)[off:off + n].copy_(dev[r, st:st + n])
                Z.zero_layer_release(c.ctx, l, s)
                Z.zero_grads_ready(c.ctx, first_t[l], count_t[l], c.grads, c.acc, 0, s)
            Z.zero_grads_join(c.ctx, s)
            Z.zero_step_ex(c.ctx, c.hp, c.handle, None, 1.0, 0.0, s)

        graph = _capture(step)
        for k in range(4):
            before = c.gpu_state()["param"]
            c.step_no += 1
            g = c.make_grads([(2, 100, 0x7C00)] if k == 2 else None)
            dev.copy_(torch.from_numpy(g.view(np.int16)))
            graph.replay()
            torch.cuda.synchronize()
            full = np.zeros(c.plan.T, np.uint16)
            full[c.idx] = before
            for l, (lo, hi) in enumerate(L):
                assert np.array_equal(seen[l].cpu().numpy().view(np.uint16), full[lo:hi]), (k, l)
            skipped = O.step(c.ostate, g, _ohp(c), c.ofsm)
            assert skipped == (k == 2)
            c.g.check()
            c.compare()
    finally:
        c.close()
