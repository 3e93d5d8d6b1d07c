"""ZeRO-Offload across processes: each rank holds only its own shards in host
memory, scans them (zero_cpu_scan_shard), the ranks all-reduce the two totals
over gloo, each forms the same decision (zero_cpu_decide), updates its shards
(zero_cpu_update_shard) and commits. The result equals the oracle's
unpartitioned step, bit for bit, on every rank. Host only."""
import os
import socket

import numpy as np
import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp

import oracle as O
import zero_partitioned_mixed_reduce_b200 as Z

HP = dict(lr=1e-3, beta1=0.9, beta2=0.999, eps=1e-8, weight_decay=0.01)
OHP = O.AdamW(1e-3, 0.9, 0.999, 1e-8, 0.01)
NUMELS = [90_001, 13, 4096, 77_777]


def inputs(R, dtype, mode, steps, n_micro, seed):
    """Seeded master weights and per-step micro-batch replicas (both sides)."""
    rng = np.random.default_rng(seed)
    P = sum(NUMELS)
    x = rng.normal(0, 0.02, P).astype(np.float32)
    grads = [O.float_to_half((rng.normal(0, 1e-2, (n_micro, R, P)) * 64.0).astype(np.float32), dtype)
             for _ in range(steps)]
    if mode == O.SCALE_DYNAMIC:
        grads[1][0, R - 1, P - 5] = 0x7C00 if dtype == O.FP16 else 0x7F80  # step 2 overflows
    return x, grads


def run_rank(rank, world, port, dtype, mode, clip, n_micro, nthreads, out_dir):
    dist.init_process_group("gloo", init_method=f"tcp://127.0.0.1:{port}", rank=rank, world_size=world)
    try:
        R = world
        steps = 3
        lay = O.Layout(NUMELS, R, 8)
        plan = Z.Plan(NUMELS, None, R, dtype, 8, 0)
        S, idx = plan.S, lay.flat_index()
        x, grads = inputs(R, dtype, mode, steps, n_micro, seed=77)
        flat = np.zeros(lay.T, np.float32)
        flat[idx] = x
        ost = O.State(x, dtype)
        pflat = np.zeros(lay.T, np.uint16)
        pflat[idx] = ost.param
        sl = slice(rank * S, (rank + 1) * S)
        own = lambda arr: [arr if r == rank else None for r in range(R)]
        master, m, v = flat[sl].copy(), np.zeros(S, np.float32), np.zeros(S, np.float32)
        param, acc = pflat[sl].copy(), np.zeros(S, np.float32)
        cfg = dict(mode=mode, growth_interval=2)
        ls = dict(scale=64.0 if mode else 1.0, cur=0, good=0, t=0)
        fsm = O.make_fsm(mode, scale=64.0 if mode else 1.0, interval=2)
        for s in range(steps):
            g = grads[s]
            # this rank's accumulator: the rank-order sum of every micro-batch
            total = None
            for mu in range(n_micro):
                part, _ = O.allreduce_sum(g[mu], dtype)
                total = part if total is None else total + part
            full = np.zeros(lay.T, np.float32)
            full[idx] = total
            acc[:] = full[sl]
            kw = dict(grad_divisor=float(n_micro), max_grad_norm=clip)
            nrm, ovf = Z.zero_cpu_scan_shard(plan.handle, cfg, ls, own(acc), rank, rank + 1, nthreads=nthreads, **kw)
            red = torch.tensor([nrm, ovf], dtype=torch.float64)
            dist.all_reduce(red)
            d = Z.zero_cpu_decide(plan.handle, cfg, ls, red.tolist(), **kw)
            Z.zero_cpu_update_shard(plan.handle, ls, HP, d, own(acc), own(master), own(m), own(v), own(param),
                                    rank, rank + 1, nthreads)
            ls = Z.zero_cpu_commit(cfg, ls, d)
            O.step_ex(ost, g, OHP, fsm, float(n_micro), clip)
            assert (ls["t"], ls["good"], ls["last_skipped"]) == (fsm.t, fsm.good, fsm.last_skipped), s
            assert np.float32(ls["scale"]) == np.float32(fsm.scale)
            if np.isfinite(fsm.grad_norm_sq):
                assert abs(ls["grad_norm_sq"] - fsm.grad_norm_sq) <= 1e-9 * fsm.grad_norm_sq
            want = np.zeros(lay.T, np.float32)
            for name, got in (("master", master), ("m", m), ("v", v)):
                want[:] = 0
                want[idx] = getattr(ost, name)
                assert np.array_equal(got.view(np.uint32), want[sl].view(np.uint32)), (name, s)
            wp = np.zeros(lay.T, np.uint16)
            wp[idx] = ost.param
            assert np.array_equal(param, wp[sl]), s
        open(os.path.join(out_dir, f"ok{rank}"), "w").write("ok")
    finally:
        dist.destroy_process_group()


def free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


@pytest.mark.parametrize("world", [2, 3])
@pytest.mark.parametrize("dtype,mode,clip,n_micro", [(O.FP16, O.SCALE_DYNAMIC, 0.0, 1),
                                                     (O.BF16, O.SCALE_NONE, 1e-3, 2),
                                                     (O.FP16, O.SCALE_STATIC, 1e9, 3)])
def test_offload_across_ranks_matches_oracle(world, dtype, mode, clip, n_micro, tmp_path):
    mp.start_processes(run_rank, args=(world, free_port(), dtype, mode, clip, n_micro, 2, str(tmp_path)),
                       nprocs=world, join=True, start_method="spawn")
    assert sorted(os.listdir(tmp_path)) == [f"ok{r}" for r in range(world)]


def test_split_scan_and_update_equal_the_one_process_step():
    # one process, every owner range in turn: the same bytes as zero_cpu_step
    R, dtype, mode = 4, O.FP16, O.SCALE_DYNAMIC
    plan = Z.Plan(NUMELS, None, R, dtype, 8, 0)
    lay = O.Layout(NUMELS, R, 8)
    S, idx = plan.S, lay.flat_index()
    x, grads = inputs(R, dtype, mode, 3, 2, seed=5)
    flat = np.zeros(lay.T, np.float32)
    flat[idx] = x
    sets = []
    for _ in range(2):
        sets.append(dict(master=[flat[r * S:(r + 1) * S].copy() for r in range(R)],
                         m=[np.zeros(S, np.float32) for _ in range(R)], v=[np.zeros(S, np.float32) for _ in range(R)],
                         param=[np.zeros(S, np.uint16) for _ in range(R)], acc=[np.zeros(S, np.float32) for _ in range(R)],
                         ls=dict(scale=64.0, cur=0, good=0, t=0)))
    cfg = dict(mode=mode, growth_interval=2)
    for s in range(3):
        total = None
        for mu in range(2):
            part, _ = O.allreduce_sum(grads[s][mu], dtype)
            total = part if total is None else total + part
        full = np.zeros(lay.T, np.float32)
        full[idx] = total
        for st in sets:
            for r in range(R):
                st["acc"][r][:] = full[r * S:(r + 1) * S]
        a = sets[0]
        a["ls"] = Z.zero_cpu_step(plan.handle, cfg, a["ls"], HP, a["acc"], a["master"], a["m"], a["v"], a["param"],
                                  2.0, 1e-3, 3)
        b = sets[1]
        ranges = [(0, 1), (1, 3), (3, 4)]
        parts = [Z.zero_cpu_scan_shard(plan.handle, cfg, b["ls"], b["acc"], lo, hi, 2.0, 1e-3, 3) for lo, hi in ranges]
        red = (sum(p[0] for p in parts), sum(p[1] for p in parts))
        d = Z.zero_cpu_decide(plan.handle, cfg, b["ls"], red, 2.0, 1e-3)
        for lo, hi in ranges:
            Z.zero_cpu_update_shard(plan.handle, b["ls"], HP, d, b["acc"], b["master"], b["m"], b["v"], b["param"],
                                    lo, hi, 3)
        b["ls"] = Z.zero_cpu_commit(cfg, b["ls"], d)
        for k in ("master", "m", "v"):
            for x1, x2 in zip(a[k], b[k]):
                assert np.array_equal(x1.view(np.uint32), x2.view(np.uint32)), (k, s)
        for x1, x2 in zip(a["param"], b["param"]):
            assert np.array_equal(x1, x2)
        assert (a["ls"]["t"], a["ls"]["scale"], a["ls"]["good"]) == (b["ls"]["t"], b["ls"]["scale"], b["ls"]["good"])


def test_shard_call_errors():
    plan = Z.Plan([1000], None, 2, O.BF16, 8, 0)
    S = plan.S
    acc = [np.zeros(S, np.float32), None]
    cfg = dict(mode=O.SCALE_NONE)
    ls = dict(scale=1.0, cur=0, good=0, t=0)
    for lo, hi in ((1, 1), (-1, 1), (0, 3)):
        with pytest.raises(Z.ZeroError) as e:
            Z.zero_cpu_scan_shard(plan.handle, cfg, ls, acc, lo, hi)
        assert e.value.status == Z.ZERO_ERR_RANGE
    with pytest.raises(Z.ZeroError) as e:  # an owned accumulator missing
        Z.zero_cpu_scan_shard(plan.handle, cfg, ls, acc, 0, 2)
    assert e.value.status == Z.ZERO_ERR_INVALID_ARG
    with pytest.raises(Z.ZeroError) as e:
        Z.zero_cpu_decide(plan.handle, cfg, ls, (1.0, -1.0))
    assert e.value.status == Z.ZERO_ERR_INVALID_ARG
