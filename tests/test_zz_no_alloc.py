"""zero_step_noalloc: the step for callers that cannot allocate device memory.

Some callers of this library may not call cudaMalloc: a process whose GPU
memory is owned by another allocator that has already reserved it, or a
training loop that must not allocate or free once it runs (cudaFree
synchronizes the whole device, and an allocation can fail mid-run). For them
zero_step_noalloc runs the two-pass step with all of its scratch in a static
device array inside the library and no context. These tests check, through
the C ABI, on two and more calls in a row:
  - the model state and loss-scale state equal the context-based two-pass
    path (zero_reduce_scatter_bucket over the whole range + zero_step from
    the accumulators) bit for bit, and the gradient norm within the parity
    tests' bound, including a model whose padded length is exactly the
    static scratch's limit and an overflow under static and dynamic scaling;
  - the same state equals the oracle's step on the same bytes;
  - the calls after the first allocate no device memory.

The file is named so that pytest collects it last.
"""
import numpy as np
import pytest
import torch

import oracle as O

pytestmark = pytest.mark.gpu

HALF = {0: torch.bfloat16, 1: torch.float16}
MAX = 4194304  # ZERO_NOALLOC_MAX_ELEMS
# a two-tensor list whose padded length at R = 16 is exactly MAX: L = 4,194,298
# (the second tensor starts at the 8-aligned 4,194,208), S = 262,144
AT_LIMIT = [MAX - 100, 90]


def _state(plan, master0, param0, device="cuda"):
    S, R = plan.S, plan.R
    st = {f: [torch.zeros(S, dtype=torch.float32, device=device) for _ in range(R)]
          for f in ("master", "m", "v")}
    st["param"] = [torch.zeros(S, dtype=HALF[plan.dtype], device=device) for _ in range(R)]
    for r in range(R):
        st["master"][r].copy_(master0[r * S:(r + 1) * S])
        st["param"][r].copy_(param0[r * S:(r + 1) * S])
    return st


def _bits(ts):
    return torch.cat([t.contiguous().view(torch.int16 if t.element_size() == 2 else torch.int32)
                      for t in ts]).cpu().numpy()


# (numels, R, dtype, mode, the call whose replica 1 carries an inf)
CASES = [
    ([70_001, 13, 4096, 777, 5], 4, 1, 2, 2),  # fp16, dynamic: call 2 is skipped and backs off
    ([70_001, 13, 4096, 777, 5], 4, 0, 1, None),  # bf16, static scale
    ([70_001, 13, 4096, 777, 5], 4, 0, 0, None),  # bf16, no scaling
    (AT_LIMIT, 16, 0, 1, 2),  # at the size limit; static mode applies the non-finite step
]


@pytest.mark.parametrize("numels,R,dtype,mode,inf_call", CASES)
def test_noalloc_matches_context_two_pass(numels, R, dtype, mode, inf_call):
    import zero_partitioned_mixed_reduce_b200 as Z
    import synth

    plan = Z.Plan(numels, None, R, dtype, 8, 0)
    assert plan.T <= Z.ZERO_NOALLOC_MAX_ELEMS == MAX
    if numels is AT_LIMIT:
        assert plan.T == MAX
    wl = synth.custom_workload(numels, R, dtype, mode, 256.0, 3, sigma=1e-2, index=77)
    x = plan.pack(synth.flat_master(wl, "cuda"))
    p0 = x.to(HALF[dtype])
    ref, new = _state(plan, x, p0), _state(plan, x, p0)
    acc = [torch.zeros(plan.S, dtype=torch.float32, device="cuda") for _ in range(R)]
    handle = Z.StateHandle([dict(master=ref["master"], m=ref["m"], v=ref["v"],
                                 param=ref["param"])], acc)
    init = 256.0 if mode else 1.0
    ctx = Z.zero_ctx_create(plan.handle, mode, init, 3)
    cfg = dict(mode=mode, growth_interval=3, growth_factor=2.0, backoff_factor=0.5, min_scale=1.0)
    ls = dict(scale=init, cur=0, good=0, t=0)
    calls = (1, 2, 3)
    # every input of every call exists before the first call, so that nothing
    # else allocates device memory between the calls; the replicas are drawn
    # at the initial scale (the skipped call's backoff does not change them)
    grads = {c: [plan.pack(synth.flat_grads(wl, c, r, init, "cuda")) for r in range(R)] for c in calls}
    if inf_call:
        grads[inf_call][1][plan.offsets[-1] + 3] = float("inf")
    free = {}
    try:
        for call in calls:
            Z.zero_reduce_scatter_bucket(ctx, -1, grads[call], acc)
            Z.zero_step(ctx, wl["hp"], handle, None)
            want = Z.zero_loss_scale(ctx)
            torch.cuda.synchronize()
            free[call] = torch.cuda.mem_get_info()[0]
            ls = Z.zero_step_noalloc(plan.handle, cfg, ls, wl["hp"], grads[call], new["master"],
                                     new["m"], new["v"], new["param"])
            torch.cuda.synchronize()
            if call > 1:
                # the second and later calls take no device memory: the static
                # array was reserved by the first call's set-up, if not before
                assert torch.cuda.mem_get_info()[0] == free[call], (call, free[call])
            for f in ("master", "m", "v", "param"):
                assert np.array_equal(_bits(ref[f]), _bits(new[f])), (call, f)
            for k in ("t", "good", "last_overflow", "last_skipped", "cur"):
                assert ls[k] == want[k], (call, k, ls[k], want[k])
            if mode:
                assert ls["scale"] == want["scale"]
            a, b = ls["grad_norm_sq"], want["grad_norm_sq"]
            if np.isfinite(b):
                assert abs(a - b) <= 1e-9 * abs(b)
            else:
                assert not np.isfinite(a)
        if mode == 2:
            assert ls["last_overflow"] == 0 and ls["t"] == 2 and ls["scale"] == 128.0
        if mode == 1 and inf_call:
            assert want["last_overflow"] == 0 and want["t"] == 3  # static mode never skips
    finally:
        Z.zero_ctx_destroy(ctx)


@pytest.mark.parametrize("numels,R,dtype,align,mode", [
    ([70_001, 13, 4096, 777, 5], 3, 1, 1, 2),  # R = 3, packed tensors, dynamic scaling with a skip
    (AT_LIMIT, 16, 0, 8, 1),  # at the size limit, static scaling with an overflow
])
def test_noalloc_matches_the_oracle(numels, R, dtype, align, mode):
    from gpu_harness import Case
    c = Case(numels, R, dtype, align, mode, init_scale=256.0, interval=2, path="inplace", seed=R + 40)
    inf = 0x7C00 if dtype == O.FP16 else 0x7F80
    try:
        for call in (1, 2, 3):
            c.step_noalloc(inject=[(1, 17, inf)] if call == 2 else None)
            c.compare(fsm=c.noalloc_ls)
        if mode == O.SCALE_DYNAMIC:
            assert c.noalloc_ls["t"] == 2 and c.noalloc_ls["scale"] == 128.0
        else:
            assert c.noalloc_ls["t"] == 3 and c.noalloc_ls["last_skipped"] == 0
    finally:
        c.close()


def test_noalloc_rejects_models_beyond_its_scratch():
    import zero_partitioned_mixed_reduce_b200 as Z
    plan = Z.Plan([Z.ZERO_NOALLOC_MAX_ELEMS + 1], None, 1, 0, 8, 0)
    dummy = [torch.zeros(8, device="cuda")]
    with pytest.raises(Z.ZeroError) as e:
        Z.zero_step_noalloc(plan.handle, dict(mode=0), dict(scale=1.0, cur=0, good=0, t=0),
                            dict(lr=1e-3, beta1=0.9, beta2=0.999, eps=1e-8, weight_decay=0.0),
                            dummy, dummy, dummy, dummy, dummy)
    assert e.value.status == 5 and "static scratch" in str(e.value)
