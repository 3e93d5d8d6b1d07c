"""Per-call tracing (zero_trace_start / zero_trace_read / zero_trace_stop):
every traced call's device time, in call order, with its bucket or layer;
nothing recorded while a stream is captured; a full trace counts the calls it
dropped; a short read buffer consumes nothing."""
import math

import pytest
import torch

import oracle as O

pytestmark = pytest.mark.gpu

if torch.cuda.is_available():
    import zero_partitioned_mixed_reduce_b200 as Z
    from gpu_harness import Case


def test_trace_records_every_call_in_order():
    c = Case([70_001, 13, 4096, 7, 999], 4, O.FP16, 8, O.SCALE_DYNAMIC, init_scale=256.0, path="twopass_pp",
             bucket_elems=5000, layer_ids=[0, 0, 1, 1, 2])
    nb, nl = len(c.plan.buckets), len(c.plan.layers)
    try:
        with pytest.raises(Z.ZeroError) as e:
            Z.zero_trace_read(c.ctx)
        assert e.value.status == Z.ZERO_ERR_STATE
        Z.zero_trace_start(c.ctx, 64)
        c.step_ex(2, 2.0, 1e-3, rs_norm=True)  # 2 x nb reduce-scatters, then the step
        c.compare()
        outs = [torch.empty(hi - lo, dtype=torch.float16, device="cuda") for lo, hi in c.plan.layers]
        Z.zero_gather_layers(c.ctx, 0, outs, c.handle)
        Z.zero_gather_layer(c.ctx, 1, c.handle, outs[1])
        recs, dropped = Z.zero_trace_read(c.ctx)
        assert dropped == 0
        want = ([("reduce_scatter", b) for b in range(nb)] * 2 + [("step", -1), ("gather", 0), ("gather", 1)])
        assert [(n, a) for n, a, _ in recs] == want
        assert all(math.isfinite(ms) and ms > 0.0 for _, _, ms in recs)
        # read empties the trace
        assert Z.zero_trace_read(c.ctx) == ([], 0)
        Z.zero_trace_stop(c.ctx)
        with pytest.raises(Z.ZeroError):
            Z.zero_trace_read(c.ctx)
    finally:
        c.close()


def test_trace_capacity_short_reads_and_capture():
    c = Case([50_000, 333, 8_192], 2, O.BF16, mode=O.SCALE_NONE, path="twopass", bucket_elems=20_000)
    nb = len(c.plan.buckets)
    try:
        Z.zero_trace_start(c.ctx, 2)
        for b in range(nb):
            Z.zero_reduce_scatter_bucket(c.ctx, b, c.grads, c.acc)
        Z.zero_step(c.ctx, c.hp, c.handle, None)
        # room for one record of two: nothing is consumed
        with pytest.raises(Z.ZeroError) as e:
            Z.zero_trace_read(c.ctx, max_records=1)
        assert e.value.status == Z.ZERO_ERR_RANGE
        recs, dropped = Z.zero_trace_read(c.ctx)
        assert len(recs) == 2 and dropped == nb + 1 - 2
        # calls captured into a CUDA graph are not traced, nor are replays
        Z.zero_trace_start(c.ctx, 16)
        Z.zero_ctx_reserve_steps(c.ctx, 8, c.hp["beta1"], c.hp["beta2"])
        s = torch.cuda.Stream()
        s.wait_stream(torch.cuda.current_stream())
        g = torch.cuda.CUDAGraph()
        with torch.cuda.graph(g, stream=s):
            for b in range(nb):
                Z.zero_reduce_scatter_bucket(c.ctx, b, c.grads, c.acc, torch.cuda.current_stream())
        torch.cuda.current_stream().wait_stream(s)
        g.replay()
        torch.cuda.synchronize()
        assert Z.zero_trace_read(c.ctx) == ([], 0)
        del g
        with pytest.raises(Z.ZeroError) as e:
            Z.zero_trace_start(c.ctx, 0)
        assert e.value.status == Z.ZERO_ERR_INVALID_ARG
        Z.zero_trace_stop(c.ctx)
    finally:
        c.close()


def test_trace_sees_the_scheduler_launches():
    c = Case([70_001, 13, 4096, 7, 999, 30_000, 5], 4, O.BF16, 8, O.SCALE_NONE, path="twopass",
             bucket_elems=20_000, layer_ids=[0, 0, 1, 1, 2, 2, 3])
    nb, nl = len(c.plan.buckets), len(c.plan.layers)
    try:
        Z.zero_trace_start(c.ctx, 256)
        c.step_overlap(1, 1.0, 0.0, None)  # one report per tensor, reverse order
        c.compare()
        recs, _ = Z.zero_trace_read(c.ctx)
        rs = [a for n, a, _ in recs if n == "reduce_scatter"]
        assert sorted(rs) == list(range(nb)) and recs[-1][0] == "step"
        # a forward pass through the look-ahead ring
        bufs = [torch.empty(max(hi - lo for lo, hi in c.plan.layers), dtype=torch.bfloat16, device="cuda")
                for _ in range(2)]
        Z.zero_prefetch_begin(c.ctx, c.handle, bufs, 1, 1, torch.cuda.current_stream())
        for layer in range(nl):
            Z.zero_layer_acquire(c.ctx, layer, torch.cuda.current_stream())
            Z.zero_layer_release(c.ctx, layer, torch.cuda.current_stream())
        recs, _ = Z.zero_trace_read(c.ctx)
        assert [(n, a) for n, a, _ in recs] == [("gather", l) for l in range(nl)]
        Z.zero_trace_stop(c.ctx)
    finally:
        c.close()
