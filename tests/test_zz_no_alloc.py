"""zero_step_noalloc: the step for callers that cannot allocate device memory.

Some callers of this library may not call cudaMalloc: a process whose GPU
memory is owned by another allocator that has already reserved it, or a
training loop that must not allocate or free once it runs (cudaFree
synchronizes the whole device, and an allocation can fail mid-run). For them
zero_step_noalloc runs the two-pass step with all of its scratch in a static
device array inside the library and no context. These tests check, through
the C ABI, that two calls in a row give the same model state and loss-scale
state as the context-based two-pass path (zero_reduce_scatter_bucket over the
whole range + zero_step from the accumulators), bit for bit on the model
state and within the parity tests' bound on the gradient norm.

The file is named so that pytest collects it last.
"""
import numpy as np
import pytest
import torch

pytestmark = pytest.mark.gpu

HALF = {0: torch.bfloat16, 1: torch.float16}


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


@pytest.mark.parametrize("dtype,mode", [(1, 2), (0, 1), (0, 0)])
def test_noalloc_matches_context_two_pass(dtype, mode):
    import zero_partitioned_mixed_reduce_b200 as Z
    import synth

    numels, R = [70_001, 13, 4096, 777, 5], 4
    plan = Z.Plan(numels, None, R, dtype, 8, 0)
    assert plan.T <= Z.ZERO_NOALLOC_MAX_ELEMS
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
    try:
        for call in (1, 2):
            grads = [plan.pack(synth.flat_grads(wl, call, r, ls["scale"] if mode else 1.0, "cuda"))
                     for r in range(R)]
            if call == 2 and mode == 2:  # the second call overflows and must be skipped
                grads[1][plan.offsets[2] + 9] = float("inf")
            Z.zero_reduce_scatter_bucket(ctx, -1, grads, acc)
            Z.zero_step(ctx, wl["hp"], handle, None)
            want = Z.zero_loss_scale(ctx)
            ls = Z.zero_step_noalloc(plan.handle, cfg, ls, wl["hp"], grads, new["master"],
                                     new["m"], new["v"], new["param"])
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
            assert ls["last_skipped"] == 1 and ls["scale"] == 128.0 and ls["t"] == 1
    finally:
        Z.zero_ctx_destroy(ctx)


def test_noalloc_rejects_models_beyond_its_scratch():
    import zero_partitioned_mixed_reduce_b200 as Z
    plan = Z.Plan([Z.ZERO_NOALLOC_MAX_ELEMS + 1], None, 1, 0, 8, 0)
    dummy = [torch.zeros(8, device="cuda")]
    with pytest.raises(Z.ZeroError) as e:
        Z.zero_step_noalloc(plan.handle, dict(mode=0), dict(scale=1.0, cur=0, good=0, t=0),
                            dict(lr=1e-3, beta1=0.9, beta2=0.999, eps=1e-8, weight_decay=0.0),
                            dummy, dummy, dummy, dummy, dummy)
    assert e.value.status == 5 and "static scratch" in str(e.value)
