"""Worker for tests/test_gpu_dist.py, launched with torch.distributed.run:
DistributedZero (one process per GPU, NCCL, CUDA IPC peer mappings) against the
oracle. Prints "ok" on rank 0 when every step matched."""
import datetime
import os
import sys

import numpy as np
import torch
import torch.distributed as dist

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
sys.path.insert(0, ROOT)

import oracle as O  # noqa: E402
import zero_partitioned_mixed_reduce_b200 as Z  # noqa: E402
import synth  # noqa: E402
from zero_partitioned_mixed_reduce_b200.dist import DistributedZero  # noqa: E402


def u16(t):
    return t.contiguous().view(torch.int16).cpu().numpy().view(np.uint16)


def main():
    # ZB_DIST_BACKEND=gloo runs the ranks as processes sharing this machine's
    # GPUs (several ranks on one GPU): their buffers are still shared through
    # CUDA IPC, and the ordering all-reduces go through gloo, which blocks on
    # the host; no kernel ever waits for another rank's
    backend = os.environ.get("ZB_DIST_BACKEND", "nccl")
    torch.cuda.set_device(int(os.environ.get("LOCAL_RANK", "0")) % torch.cuda.device_count())
    dist.init_process_group(backend, timeout=datetime.timedelta(seconds=120))
    rank, world = dist.get_rank(), dist.get_world_size()
    numels, layer_ids = [70_001, 13, 4096, 999], [0, 0, 1, 1]
    dz = DistributedZero(numels, layer_ids, Z.ZERO_FP16, Z.ZERO_SCALE_DYNAMIC, 256.0, 3, push_params=True)
    wl = synth.custom_workload(numels, world, Z.ZERO_FP16, Z.ZERO_SCALE_DYNAMIC, 256.0, 3, sigma=1e-2,
                               layer_ids=layer_ids, index=55)
    lay = O.Layout(numels, world, 8, 0, layer_ids)
    idx = lay.flat_index()
    x = synth.flat_master(wl, "cpu")
    p0 = x.to(torch.float16)
    dz.load(dz.plan.pack(x.cuda()), dz.plan.pack(p0.cuda()))
    ost = O.State(x.numpy(), O.FP16, u16(p0))
    fsm = O.make_fsm(O.SCALE_DYNAMIC, scale=256.0, interval=3)
    hp = wl["hp"]
    ohp = O.AdamW(*(hp[k] for k in ("lr", "beta1", "beta2", "eps", "weight_decay")))
    S = dz.plan.S
    side = torch.cuda.Stream()
    for step in range(1, 6):
        g = np.stack([u16(synth.flat_grads(wl, step, r, fsm.scale, "cpu")) for r in range(world)])
        if step == 3:
            g[world - 1, 5] = 0x7C00
        gp = np.zeros(dz.plan.T, np.uint16)
        gp[idx] = g[rank]
        dz.grads.view(torch.int16).copy_(torch.from_numpy(gp.view(np.int16)))
        if step == 2:  # a side stream made current: kernels and collectives follow it
            side.wait_stream(torch.cuda.current_stream())
            with torch.cuda.stream(side):
                dz.step(hp)
            torch.cuda.current_stream().wait_stream(side)
        elif step == 4:  # a side stream passed in
            side.wait_stream(torch.cuda.current_stream())
            dz.step(hp, stream=side)
            torch.cuda.current_stream().wait_stream(side)
        else:
            dz.step(hp)
        O.step(ost, g, ohp, fsm)
        f = dz.loss_scale()
        assert (f["t"], f["last_skipped"], f["scale"]) == (fsm.t, fsm.last_skipped, fsm.scale), (step, f)
        flat = np.zeros(dz.plan.T, np.float32)
        flat[idx] = ost.master
        mine = dz.current("master").cpu().numpy()
        assert np.array_equal(mine.view(np.uint32), flat[rank * S:(rank + 1) * S].view(np.uint32)), step
        # the parameters every rank's step pushed: the whole model on every rank
        pfull = np.zeros(dz.plan.T, np.uint16)
        pfull[idx] = ost.param
        assert np.array_equal(u16(dz.full_params()), pfull), step
    # ZeRO-3 gather from every rank's shard
    pflat = np.zeros(dz.plan.T, np.uint16)
    pflat[idx] = ost.param
    for l, (lo, hi) in enumerate(lay.layers):
        out = torch.empty(hi - lo, dtype=torch.float16, device="cuda")
        dz.gather_layer(l, out)
        torch.cuda.synchronize()
        assert np.array_equal(u16(out), pflat[lo:hi]), l
    # the same layers bucketed, and through the look-ahead ring
    outs = [torch.empty(hi - lo, dtype=torch.float16, device="cuda") for lo, hi in lay.layers]
    dz.gather_layers(0, outs)
    torch.cuda.synchronize()
    for l, (lo, hi) in enumerate(lay.layers):
        assert np.array_equal(u16(outs[l]), pflat[lo:hi]), l
    biggest = max(hi - lo for lo, hi in lay.layers)
    bufs = [torch.empty(biggest + 8, dtype=torch.float16, device="cuda") for _ in range(2)]
    by_addr = {b.data_ptr(): b for b in bufs}
    dz.prefetch_begin(bufs, 1, 1)
    for l, (lo, hi) in enumerate(lay.layers):
        buf = by_addr[dz.layer_acquire(l)]
        torch.cuda.synchronize()
        assert np.array_equal(u16(buf[:hi - lo]), pflat[lo:hi]), l
        dz.layer_release(l)
    dz.close()
    check_accumulate_and_clip(rank, world)
    # the same with the clipping norm taken by the reduce-scatters (divisor 2:
    # the two-micro-batch steps use the shares, the others the accumulator)
    check_accumulate_and_clip(rank, world, norm_divisor=2.0)
    dist.barrier()
    dist.destroy_process_group()
    if rank == 0:
        print("ok")


def check_accumulate_and_clip(rank, world, norm_divisor=None):
    """Two-pass steps over accumulated micro-batches and fused steps, with
    global-norm clipping, against the oracle's step_ex."""
    numels = [50_001, 77, 3000]
    dz = DistributedZero(numels, None, Z.ZERO_BF16, Z.ZERO_SCALE_NONE, bucket_elems=20_000, accumulate=True,
                         norm_divisor=norm_divisor)
    wl = synth.custom_workload(numels, world, Z.ZERO_BF16, Z.ZERO_SCALE_NONE, 1.0, 1000, sigma=1e-2,
                               index=56)
    lay = O.Layout(numels, world, 8)
    idx = lay.flat_index()
    x = synth.flat_master(wl, "cpu")
    p0 = x.to(torch.bfloat16)
    dz.load(dz.plan.pack(x.cuda()), dz.plan.pack(p0.cuda()))
    ost = O.State(x.numpy(), O.BF16, u16(p0))
    fsm = O.make_fsm(O.SCALE_NONE)
    hp = wl["hp"]
    ohp = O.AdamW(*(hp[k] for k in ("lr", "beta1", "beta2", "eps", "weight_decay")))
    S = dz.plan.S

    def write(g):
        gp = np.zeros(dz.plan.T, np.uint16)
        gp[idx] = g[rank]
        dz.grads.view(torch.int16).copy_(torch.from_numpy(gp.view(np.int16)))

    for step in range(1, 7):
        clip = 1e-3 if step % 2 else 0.0
        if step >= 5:  # three micro-batches, the last passed to the fused step
            micro = [np.stack([u16(synth.flat_grads(wl, step * 10 + mu, r, 1.0, "cpu")) for r in range(world)])
                     for mu in range(3)]
            for g in micro[:2]:
                write(g)
                dz.reduce_scatter()
            write(micro[2])
            dz.step(hp, max_grad_norm=clip)
            O.step_ex(ost, np.stack(micro), ohp, fsm, 3.0, clip)
        elif step <= 2:  # two micro-batches, accumulated
            micro = [np.stack([u16(synth.flat_grads(wl, step * 10 + mu, r, 1.0, "cpu")) for r in range(world)])
                     for mu in range(2)]
            for g in micro:
                write(g)
                dz.reduce_scatter()
            dz.step_accumulated(hp, max_grad_norm=clip)
            O.step_ex(ost, np.stack(micro), ohp, fsm, 2.0, clip)
        else:  # fused
            g = np.stack([u16(synth.flat_grads(wl, step * 10, r, 1.0, "cpu")) for r in range(world)])
            write(g)
            dz.step(hp, max_grad_norm=clip)
            O.step_ex(ost, g[None], ohp, fsm, 1.0, clip)
        f = dz.loss_scale()
        assert f["t"] == fsm.t, (step, f)
        assert abs(f["grad_norm_sq"] - fsm.grad_norm_sq) <= 1e-9 * fsm.grad_norm_sq, step
        flat = np.zeros(dz.plan.T, np.float32)
        flat[idx] = ost.master
        mine = dz.current("master").cpu().numpy()
        assert np.array_equal(mine.view(np.uint32), flat[rank * S:(rank + 1) * S].view(np.uint32)), step

    def check_master(step):
        flat = np.zeros(dz.plan.T, np.float32)
        flat[idx] = ost.master
        mine = dz.current("master").cpu().numpy()
        assert np.array_equal(mine.view(np.uint32), flat[rank * S:(rank + 1) * S].view(np.uint32)), step

    # overlapped with a backward pass: each tensor's gradients are written on
    # the compute stream in reverse order and reported; buckets reduce-scatter
    # on the communication stream as they complete
    starts = np.concatenate([[0], np.cumsum(numels)[:-1]])
    for step in range(7, 10):
        clip = 1e-3 if step == 8 else 0.0
        micro = [np.stack([u16(synth.flat_grads(wl, step * 10 + mu, r, 1.0, "cpu")) for r in range(world)])
                 for mu in range(2)]
        for mu, g in enumerate(micro):
            dev = torch.from_numpy(g[rank].view(np.int16)).cuda()
            for k in reversed(range(len(numels))):
                off, n, st = int(lay.offsets[k]), numels[k], int(starts[k])
                dz.grads.view(torch.int16)[off:off + n].copy_(dev[st:st + n])
                if step != 9:
                    dz.grads_ready(k)
            if step == 9:
                # every tensor reported at once: the buckets go as one run
                dz.grads_ready(0, len(numels))
            dz.join()
        dz.step_accumulated(hp, max_grad_norm=clip)
        O.step_ex(ost, np.stack(micro), ohp, fsm, 2.0, clip)
        assert dz.loss_scale()["t"] == fsm.t, step
        check_master(step)
    dz.close()


if __name__ == "__main__":
    main()
