"""A one-GPU ZeRO step through the Python binding, as a user writes it.

R = 8 simulated data-parallel ranks on one GPU, fp16 gradients, dynamic loss
scaling, ping-pong state: build the partition plan, load the fp32 master
weights into the shards, run the fused reduce-scatter + AdamW + cast step,
read the loss-scale state and gather one layer (ZeRO-3). Every call is a
thin binding of the C ABI function of the same name.

    python -m zero_partitioned_mixed_reduce_b200.example
"""
import torch

import zero_partitioned_mixed_reduce_b200 as Z


def one_gpu_step():
    numels, layers = [768 * 3072, 3072, 3072 * 768, 768], [0, 0, 1, 1]
    plan = Z.Plan(numels, layers, R=8, dtype=Z.ZERO_FP16, tensor_align=8, bucket_elems=25_000_000)
    state = Z.ShardedState(plan, sets=2)                  # two sets: ping-pong state
    x = torch.randn(sum(numels), device="cuda") * 0.02    # fp32 master weights, unpadded
    state.load(plan.pack(x), plan.pack(x.half()))
    ctx = Z.zero_ctx_create(plan.handle, Z.ZERO_SCALE_DYNAMIC, 65536.0, 1000)
    grads = [torch.zeros(plan.T, dtype=torch.float16, device="cuda") for _ in range(8)]
    hp = dict(lr=1e-3, beta1=0.9, beta2=0.999, eps=1e-8, weight_decay=0.01)
    # each rank's backward writes its replica into grads[r] (flat layout, padding zero)
    for g in grads:
        g[:plan.L].normal_(0.0, 1e-4 * 65536.0)
    Z.zero_step(ctx, hp, state.handle, grads)              # fused reduce-scatter + AdamW + cast
    ls = Z.zero_loss_scale(ctx)                            # scale, t, skipped, grad_norm_sq, cur
    lo, hi = plan.layers[1]
    out = torch.empty(hi - lo, dtype=torch.float16, device="cuda")
    Z.zero_gather_layer(ctx, 1, state.handle, out)         # ZeRO-3 gather of layer 1
    Z.zero_ctx_destroy(ctx)
    return plan, state, ls, out


if __name__ == "__main__":
    _, _, ls, out = one_gpu_step()
    print(ls, out.shape)
