#!/usr/bin/env python
"""Benchmark of the ZeRO data-parallel hot path on B200.

One step = one pass of the whole path over one batch of synthetic
gradients: the fused reduce-scatter + unscale + overflow check + AdamW +
cast kernel over every shard (ping-pong state), the device-side loss-scale
update, and the ZeRO-3 gather of every layer into a contiguous buffer. The
partition plan is built once, before timing.

Default workload: the Llama-style 3B-shaped parameter list (3,606,752,256
params, 255 tensors, 28 layers, d=3072, SwiGLU 8192, GQA 24/8 heads, vocab
128256, untied embeddings), R=4 simulated ranks, bf16 gradients
1e-4 * Student-t(3), no loss scaling. The step touches about 137 GB of HBM,
far more than the 126 MB L2. `--workload gpt2s|d1p3b|irr_r2|irr_r16|tiny`
selects the other configurations.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl ours|reference]

With N > 1 (under torch.distributed.run) the job runs the real multi-GPU
ZeRO step (DistributedZero): rank o owns shard o of the workload, its fused
step reads the other ranks' gradient replicas over NVLink, and the ZeRO-3
gathers read every rank's parameter shard; the time is the maximum over
ranks. `--replicas` runs N independent single-GPU copies instead. The step
and the gathers are captured once into CUDA graphs through the C ABI and
replayed (`--eager` issues every launch instead). `--impl reference` times
the CPU oracle on host cores on a bounded sample of the same workload, and
reports the same `config`. ZB_BENCH_BACKEND=gloo runs a multi-rank job with
several ranks sharing a GPU (a functional test of that path, not a
measurement).
"""
import argparse
import datetime
import hashlib
import json
import os
import statistics
import sys
import time

import numpy as np
import torch

ROOT = os.path.dirname(os.path.abspath(__file__))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)

METRIC = "params updated/sec per ZeRO step and achieved HBM GB/s vs B200 peak, 1 GPU"
FALLBACK_HBM_GBS = 6650.0
NOMINAL_HBM_GBS = 8000.0  # B200 HBM3e, the spec figure (the measured copy is the roofline peak)


def parse_args(argv=None):
    ap = argparse.ArgumentParser(description=__doc__.splitlines()[1])
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=100)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--impl", choices=["ours", "reference"], default="ours")
    ap.add_argument("--workload", default="llama3b")
    ap.add_argument("--path", choices=["auto", "pingpong", "inplace", "twopass", "twopass_pingpong"],
                    default="auto",
                    help="fused step (ping-pong or in-place state) or the two-pass path "
                         "(in-place or ping-pong state)")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--no-e2e", action="store_true")
    ap.add_argument("--accum", type=int, default=1,
                    help="micro-batches accumulated per step (the last fused into the step, or "
                         "all reduce-scattered on the two-pass path)")
    ap.add_argument("--clip", type=float, default=0.0,
                    help="global-norm clipping threshold (> 0: on; fused path for R <= 4, "
                         "two-pass path otherwise)")
    ap.add_argument("--clip-norm", choices=["rs", "pass"], default="rs",
                    help="two-pass path with clipping: the last micro-batch's reduce-scatters take "
                         "the norm (rs), or a separate read-only pass over the accumulators (pass)")
    ap.add_argument("--gather-bucket", type=int, default=32 << 20,
                    help="gather consecutive layers in one launch up to this many elements "
                         "(0: one launch per layer)")
    ap.add_argument("--overlap", action="store_true",
                    help="measure the overlap scheduler on a synthetic training step instead")
    ap.add_argument("--tokens", type=int, default=4096,
                    help="tokens per synthetic GEMM in --overlap mode")
    ap.add_argument("--bucket-elems", type=int, default=None,
                    help="override the workload's reduce-scatter bucket size")
    ap.add_argument("--carveout", type=int, default=0,
                    help="SMs kept free of the synthetic GEMMs in --overlap mode")
    ap.add_argument("--comm-sms", type=int, default=0,
                    help="SMs the scheduler's communication kernels may fill in --overlap mode "
                         "(0: all)")
    ap.add_argument("--offload", action="store_true",
                    help="measure ZeRO-Offload (CPU AdamW, with and without the delayed update)")
    ap.add_argument("--rs-sweep", action="store_true",
                    help="time the bucketed reduce-scatter against bucket size instead")
    ap.add_argument("--rs-sizes", default="0,1000000,5000000,25000000,50000000,100000000,200000000",
                    help="bucket sizes (elements; 0: one bucket for the whole model) for --rs-sweep")
    ap.add_argument("--dist", action="store_true",
                    help="the real multi-GPU ZeRO step over the job's GPUs (DistributedZero), also at "
                         "N = 1 (the default whenever N > 1)")
    ap.add_argument("--zero2", action="store_true",
                    help="sharded step: ZeRO-1/2 parameters (every rank keeps the whole model, which each "
                         "rank's step pushes to every rank) instead of the ZeRO-3 layer gathers")
    ap.add_argument("--replicas", action="store_true",
                    help="with N > 1: N independent single-GPU copies of the workload (no collective on "
                         "the data path) instead of the sharded multi-GPU step")
    ap.add_argument("--rs-group", type=int, default=25 << 20,
                    help="two-pass path: consecutive buckets reduce-scattered in one launch up to this "
                         "many elements (0: one launch per bucket)")
    ap.add_argument("--graph", dest="graph", action="store_true", default=True,
                    help="(default) capture the step and the gathers once into CUDA graphs, "
                         "through the C ABI, and replay them")
    ap.add_argument("--eager", dest="graph", action="store_false",
                    help="issue every launch through the C ABI instead of replaying CUDA graphs")
    ap.add_argument("--first-tensors", type=int, default=0,
                    help="use only the first N tensors of the workload (small profiling cases)")
    ap.add_argument("--tensors", default="",
                    help="use only tensors LO:HI of the workload's list (small profiling cases)")
    args = ap.parse_args(argv)
    args.tensor_range = None
    if args.tensors:
        lo, hi = (int(x) for x in args.tensors.split(":"))
        args.tensor_range = (lo, hi)
    elif args.first_tensors:
        args.tensor_range = (0, args.first_tensors)
    return args


def restrict(wl, rng):
    """The workload cut to tensors [lo, hi) of its list (layer ids renumbered
    from 0); rng None keeps it whole."""
    if rng is None:
        return wl
    lo, hi = rng
    wl["numels"] = wl["numels"][lo:hi]
    if wl["layer_ids"]:
        ids = wl["layer_ids"][lo:hi]
        wl["layer_ids"] = [i - ids[0] for i in ids]
    if wl.get("inject") and not (lo <= wl["inject"]["tensor"] < hi):
        wl["inject"] = None
    elif wl.get("inject"):
        wl["inject"] = dict(wl["inject"], tensor=wl["inject"]["tensor"] - lo)
    return wl


# ---- distributed plumbing ---------------------------------------------------

def dist_init():
    """One process per GPU: NCCL when there are GPUs, gloo otherwise.
    ZB_BENCH_BACKEND=gloo keeps gloo with GPUs, so that several ranks can
    share one GPU in a functional test of the multi-rank path (rank r on GPU
    r mod the GPU count); such a run measures nothing."""
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    if world > 1:
        import torch.distributed as dist
        backend = os.environ.get("ZB_BENCH_BACKEND") or ("nccl" if torch.cuda.is_available() else "gloo")
        if torch.cuda.is_available():
            torch.cuda.set_device(local % torch.cuda.device_count())
        dist.init_process_group(backend, timeout=datetime.timedelta(seconds=300))
    elif torch.cuda.is_available():
        torch.cuda.set_device(local)
    return world, rank, local


def barrier(world):
    if world > 1:
        import torch.distributed as dist
        dist.barrier()


def aggregate(ms_local, units_local, world):
    """Max of the per-rank times and sum of the per-rank units (whole job)."""
    if world == 1:
        return ms_local, units_local
    import torch.distributed as dist
    dev = "cuda" if dist.get_backend() == "nccl" else "cpu"
    t = torch.tensor([ms_local], dtype=torch.float64, device=dev)
    u = torch.tensor([units_local], dtype=torch.float64, device=dev)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    dist.all_reduce(u, op=dist.ReduceOp.SUM)
    return float(t.item()), float(u.item())


# ---- clocks -----------------------------------------------------------------

class ClockSampler:
    """SM clock and clock-event (throttle) reasons sampled through NVML from a
    background thread every ~2 ms while the timed region runs."""

    REASONS = {0x4: "sw_power_cap", 0x8: "hw_slowdown", 0x20: "sw_thermal_slowdown",
               0x40: "hw_thermal_slowdown", 0x80: "hw_power_brake_slowdown"}

    def __init__(self, device_index):
        self.dev = device_index
        self.samples = []
        self.thread = None
        self.stop_flag = False
        self.nvml = None

    def _handle(self):
        import pynvml as N
        N.nvmlInit()
        self.nvml = N
        try:
            uuid = str(torch.cuda.get_device_properties(self.dev).uuid)
            return N.nvmlDeviceGetHandleByUUID("GPU-" + uuid)
        except Exception:
            return N.nvmlDeviceGetHandleByIndex(self.dev)

    def _run(self, h):
        N = self.nvml
        get_reasons = getattr(N, "nvmlDeviceGetCurrentClocksEventReasons", None) or \
            N.nvmlDeviceGetCurrentClocksThrottleReasons
        while not self.stop_flag:
            try:
                sm = N.nvmlDeviceGetClockInfo(h, N.NVML_CLOCK_SM)
                rs = get_reasons(h)
                self.samples.append((sm, rs))
            except Exception:
                pass
            time.sleep(0.002)

    def start(self):
        import threading
        try:
            h = self._handle()
            self.max_mhz = self.nvml.nvmlDeviceGetMaxClockInfo(h, self.nvml.NVML_CLOCK_SM)
        except Exception:
            self.thread = None
            return
        self.thread = threading.Thread(target=self._run, args=(h,), daemon=True)
        self.thread.start()

    def stop(self):
        if self.thread is None:
            return None
        self.stop_flag = True
        self.thread.join(timeout=5)
        if not self.samples:
            return None
        sm = [s for s, _ in self.samples]
        reasons = sorted({name for _, rs in self.samples for bit, name in self.REASONS.items()
                          if rs & bit})
        return {"sm_mhz": statistics.median(sm), "sm_max_mhz": self.max_mhz, "reasons": reasons,
                "samples": len(sm), "source": "nvml"}


# ---- peaks and profile-derived traffic --------------------------------------

def hbm_peak():
    try:
        with open(os.path.join(ROOT, "MEASURED_PEAKS.json")) as f:
            return float(json.load(f)["hbm_gbs"]), "measured"
    except (OSError, KeyError, ValueError):
        return FALLBACK_HBM_GBS, "fallback"


def kernels_sha():
    """Hash of the step kernels' source (kernels.cu and its device header)."""
    h = hashlib.sha256()
    for name in ("kernels.cu", "device_common.cuh"):
        with open(os.path.join(ROOT, "zero_partitioned_mixed_reduce_b200", "csrc", name), "rb") as f:
            h.update(f.read())
    return h.hexdigest()[:16]


def profiled_traffic(kernel, workload):
    """DRAM bytes per launch from the committed ncu summary, if it was taken
    on the current kernel source; else None."""
    p = os.path.join(ROOT, "profiles", "traffic.txt")
    if not os.path.exists(p):
        return None
    sha = kernels_sha()
    for line in open(p):
        t = line.split()
        if len(t) >= 4 and not line.startswith("#") and t[0] == kernel and t[1] == workload \
                and t[2] == sha:
            return float(t[3])
    return None


# ---- the workload -------------------------------------------------------------

def workload_label(name, wl, tensor_range=None):
    """The workload as both arms name it in their `config`."""
    part = f" (tensors {tensor_range[0]}:{tensor_range[1]})" if tensor_range else ""
    return (f"{name}{part}: {len(wl['numels'])} tensors, P={sum(wl['numels'])}, R={wl['R']} "
            f"simulated ranks, {'fp16' if wl['dtype'] else 'bf16'} grads, "
            f"loss scale mode {wl['mode']}")


def job_config(args, world, wl, R, T, S, n_layers, sharded):
    """The workload a command line measures, as every arm of that command
    line reports it in `config` (the GPU arms take T, S and the layer count
    from the library's plan, the reference arm from the oracle's layout; they
    agree bit for bit). How an arm runs it goes elsewhere in its line.
    sharded: the DistributedZero job (one shard per rank), else one GPU or
    independent replicas."""
    label = workload_label(args.workload, wl, args.tensor_range)
    if sharded:
        label = label.split(", R=")[0] + f", sharded over {world} rank(s), one per GPU"
        par = f"dp{world}: {world} GPU(s), one shard each"
        moved, per = (2 * R + 26) * S, "per rank"
    else:
        par = "1 GPU" if world == 1 else f"{world} independent replicas (--replicas)"
        moved, per = (2 * R + 26) * T, "per GPU"
    return {"workload": label, "R": R, "P": sum(wl["numels"]), "T": T, "S": S, "n_layers": n_layers,
            "l2": f"inputs larger than L2: every step reads and writes at least (2R + 26) x "
                  f"{'S' if sharded else 'T'} = {moved / 1e9:.1f} GB {per} (L2 126 MB)",
            "parallelism": par}


def bucket_runs(buckets, group):
    """Consecutive buckets, as (first, count), in launches of up to `group`
    elements (a larger bucket alone); group 0: one launch per bucket.
    Consecutive buckets are one contiguous flat range."""
    runs, first, size = [], 0, 0
    for b, (lo, hi) in enumerate(buckets):
        n = hi - lo
        if b > first and (group <= 0 or size + n > group):
            runs.append((first, b - first))
            first, size = b, 0
        size += n
    if buckets:
        runs.append((first, len(buckets) - first))
    return runs


class Bench:
    def __init__(self, name, path, tensor_range=None, gather_bucket=32 << 20, accum=1, clip=0.0,
                 bucket_elems=None, clip_norm="rs", rs_group=25 << 20):
        import zero_partitioned_mixed_reduce_b200 as Z
        import synth
        self.Z, self.synth = Z, synth
        self.wl = wl = synth.workload(name)
        if bucket_elems is not None:
            wl["bucket_elems"] = bucket_elems
        restrict(wl, tensor_range)
        self.R, self.dtype = wl["R"], wl["dtype"]
        self.accum, self.clip = accum, clip
        if path == "auto":
            # accumulation fuses its last micro-batch into the step unless
            # clipping needs the full sum first
            if (accum > 1 and clip > 0) or (clip > 0 and wl["R"] > 4):
                path = "twopass"
            else:
                # ping-pong state measured 2-3 % faster than in place at R = 4 and 8
                # (the writes never alias the lines being read); it doubles the
                # fp32 state, which every workload here fits
                path = "pingpong"
        self.twopass = path.startswith("twopass")
        # the two-pass clip norm from the reduce-scatters, or a separate pass
        self.rs_norm = self.twopass and clip > 0 and clip_norm == "rs"
        if accum > 1 and clip > 0 and not self.twopass:
            raise SystemExit("--accum with --clip needs the two-pass path")
        self.path = path
        self.plan = Z.Plan(wl["numels"], wl["layer_ids"], wl["R"], wl["dtype"], 8,
                           wl["bucket_elems"])
        self.P, self.T, self.S, self.L = self.plan.P, self.plan.T, self.plan.S, self.plan.L
        # reduce-scatters of consecutive buckets grouped into launches, as a
        # caller whose backward has written them issues them
        self.rs_runs = bucket_runs(self.plan.buckets, rs_group)
        # the two-pass step measured the same in place as ping-pong, so it
        # keeps one state set
        sets = 2 if path in ("pingpong", "twopass_pingpong") else 1
        self.state = Z.ShardedState(self.plan, sets=sets, with_acc=self.twopass or accum > 1)
        half = Z.state.HALF[wl["dtype"]]
        # initial fp32 master ~N(0, 0.02) and its half copy, tensor by tensor
        for k, (n, off) in enumerate(zip(wl["numels"], self.plan.offsets)):
            x = synth.tensor_master(n, wl["index"], k, "cuda")
            for kset in range(sets):
                self._write(self.state.master[kset], off, x)
                self._write(self.state.param[kset], off, x.to(half))
        # one batch of gradients at the initial loss scale, padding zero
        scale = wl["init_scale"] if wl["mode"] != synth.NONE else 1.0
        self.grads = []
        for r in range(self.R):
            g = torch.zeros(self.T, dtype=half, device="cuda")
            for k, (n, off) in enumerate(zip(wl["numels"], self.plan.offsets)):
                g[off:off + n] = synth.tensor_grads(n, wl["dist"], wl["sigma"], scale,
                                                    wl["dtype"], wl["index"], 1, r, k, "cuda")
            self.grads.append(g)
        self.ctx = Z.zero_ctx_create(self.plan.handle, wl["mode"], wl["init_scale"],
                                     wl["interval"])
        if self.rs_norm:
            Z.zero_ctx_set_grad_divisor(self.ctx, float(accum))
        self.max_layer = max(hi - lo for lo, hi in self.plan.layers)
        # gather buckets: consecutive layers up to gather_bucket elements (a larger
        # layer alone), at most 64 per launch; each layer lands in its own
        # 16-byte-aligned slice of one reusable bucket buffer
        self.gather_buckets = []
        if gather_bucket > 0:
            first, size, offs = 0, 0, []
            for l, (lo, hi) in enumerate(self.plan.layers):
                n = hi - lo
                if offs and (size + n > gather_bucket or len(offs) == Z.ZERO_GATHER_MAX_LAYERS):
                    self.gather_buckets.append((first, offs, size))
                    first, size, offs = l, 0, []
                offs.append(size)
                size += (n + 7) // 8 * 8
            self.gather_buckets.append((first, offs, size))
            cap = max(b[2] for b in self.gather_buckets)
        else:
            cap = self.max_layer
        self.layer_buf = torch.empty(cap, dtype=half, device="cuda")
        base = self.layer_buf.data_ptr()
        self.gather_outs = [[base + 2 * o for o in offs] for _, offs, _ in self.gather_buckets]
        torch.cuda.synchronize()

    def _write(self, shards, off, values):
        n, pos, S = values.numel(), 0, self.S
        while pos < n:
            r, j = divmod(off + pos, S)
            k = min(n - pos, S - j)
            shards[r][j:j + k].copy_(values[pos:pos + k])
            pos += k

    def launches_per_step(self):
        n = 1 + (len(self.gather_buckets) if self.gather_buckets else len(self.plan.layers))
        if self.twopass:
            n += self.accum * len(self.rs_runs)
        else:
            n += (self.accum - 1) * len(self.rs_runs)
        if self.clip > 0:
            n += 1  # the norm pass
        return n

    def step_bytes(self):
        """Algorithmic HBM bytes of one step (and of its dominant kernel)."""
        R, T = self.R, self.T
        if self.twopass:
            # first micro-batch writes the accumulators, later ones read-modify-write
            main = (2 * R + 4) * T + (self.accum - 1) * (2 * R + 8) * T + 30 * T
            if self.clip > 0 and not self.rs_norm:
                main += 4 * T  # the norm pass over the accumulators
        elif self.accum > 1:
            # micro-batches 1..k-1 into the accumulators, the last fused with
            # the step (which reads the accumulators: 4 more bytes)
            main = (2 * R + 4) * T + (self.accum - 2) * (2 * R + 8) * T + (2 * R + 30) * T
        else:
            main = (2 * R + 26) * T
            if self.clip > 0:
                main += 2 * R * T  # the norm pass over the replicas
        return main + 4 * self.L, main

    def step_main(self, stream, grads=None):
        """The fused (or bucketed two-pass) step: the dominant kernel(s)."""
        Z = self.Z
        hp = self.wl["hp"]
        grads = self.grads if grads is None else grads
        if self.twopass:
            for mu in range(self.accum):
                flags = Z.ZERO_RS_ACCUMULATE if mu else 0
                if self.rs_norm and mu == self.accum - 1:
                    flags |= Z.ZERO_RS_NORM
                for first, count in self.rs_runs:
                    Z.zero_reduce_scatter_buckets(self.ctx, first, count, grads, self.state.acc, flags,
                                                  stream)
            Z.zero_step_ex(self.ctx, hp, self.state.handle, None, float(self.accum), self.clip,
                           stream, flags=Z.ZERO_STEP_NORM_FROM_RS if self.rs_norm else 0)
        elif self.accum > 1:
            for mu in range(self.accum - 1):
                flags = Z.ZERO_RS_ACCUMULATE if mu else 0
                for first, count in self.rs_runs:
                    Z.zero_reduce_scatter_buckets(self.ctx, first, count, grads, self.state.acc, flags,
                                                  stream)
            Z.zero_step_ex(self.ctx, hp, self.state.handle, grads, float(self.accum), 0.0, stream,
                           flags=Z.ZERO_STEP_ADD_ACC)
        elif self.clip > 0:
            Z.zero_step_ex(self.ctx, hp, self.state.handle, grads, 1.0, self.clip, stream)
        else:
            Z.zero_step(self.ctx, hp, self.state.handle, grads, stream)

    def gather(self, stream):
        Z = self.Z
        if self.gather_buckets:
            for (first, _, _), outs in zip(self.gather_buckets, self.gather_outs):
                Z.zero_gather_layers(self.ctx, first, outs, self.state.handle, stream)
        else:
            for l in range(len(self.plan.layers)):
                Z.zero_gather_layer(self.ctx, l, self.state.handle, self.layer_buf, stream)

    def capture(self, stream, steps):
        """Capture the step and the gathers into CUDA graphs (the event
        between them stays outside) after reserving `steps` bias corrections."""
        hp = self.wl["hp"]
        self.Z.zero_ctx_reserve_steps(self.ctx, steps, hp["beta1"], hp["beta2"], stream)
        self.step_graphs = {}
        self.capture_step(stream, self.grads)
        side = torch.cuda.Stream()
        side.wait_stream(stream)
        self.gather_graph = torch.cuda.CUDAGraph()
        with torch.cuda.graph(self.gather_graph, stream=side):
            self.gather(torch.cuda.current_stream())
        stream.wait_stream(side)
        self.graphs = True

    def capture_step(self, stream, grads):
        """One step graph per set of replica buffers (the e2e leg double-buffers)."""
        side = torch.cuda.Stream()
        side.wait_stream(stream)
        g = torch.cuda.CUDAGraph()
        with torch.cuda.graph(g, stream=side):
            self.step_main(torch.cuda.current_stream(), grads)
        stream.wait_stream(side)
        self.step_graphs[id(grads)] = (g, grads)

    def step(self, stream, ev=None, grads=None):
        graphs = getattr(self, "graphs", None)
        if ev is not None:
            ev[0].record(stream)
        if graphs:
            self.step_graphs[id(self.grads if grads is None else grads)][0].replay()
        else:
            self.step_main(stream, grads)
        if ev is not None:
            ev[1].record(stream)
        if graphs:
            self.gather_graph.replay()
        else:
            self.gather(stream)
        if ev is not None and len(ev) > 2:
            ev[2].record(stream)

    def loss_scale(self, stream):
        return self.Z.zero_loss_scale(self.ctx, stream=stream)

    def close(self):
        self.Z.zero_ctx_destroy(self.ctx)


def run_ours(args, world, rank, local):
    if not torch.cuda.is_available():
        print(json.dumps({"error": "no CUDA device: the benchmark has no CPU fallback"}))
        sys.exit(1)
    b = Bench(args.workload, args.path, args.tensor_range, args.gather_bucket, args.accum,
              args.clip, clip_norm=args.clip_norm, rs_group=args.rs_group)
    stream = torch.cuda.current_stream()
    if args.graph:
        b.capture(stream, args.warmup + args.steps + 16)  # + the e2e leg's steps
    for _ in range(args.warmup):
        b.step(stream)
    torch.cuda.synchronize()
    f0 = b.loss_scale(stream)
    assert f0["last_overflow"] == 0, "warm-up steps must be clean"

    K = args.steps
    evs = [tuple(torch.cuda.Event(enable_timing=True) for _ in range(3)) for _ in range(K)]
    start, end = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    clocks = ClockSampler(local)
    clocks.start()
    barrier(world)
    torch.cuda.synchronize()
    start.record(stream)
    for i in range(K):
        b.step(stream, evs[i])
    end.record(stream)
    torch.cuda.synchronize()
    barrier(world)
    clk = clocks.stop()
    ms_local = start.elapsed_time(end)
    kern_ms = [e0.elapsed_time(e1) for e0, e1, _ in evs]
    gather_ms = statistics.mean(e1.elapsed_time(e2) for _, e1, e2 in evs)
    f1 = b.loss_scale(stream)
    assert f1["last_overflow"] == 0 and f1["t"] == f0["t"] + K
    ms, units = aggregate(ms_local, float(b.P) * K, world)

    # one more step, untimed, through the library's per-call trace: the
    # device time of each call kind
    Z = b.Z
    Z.zero_trace_start(b.ctx, 4096)
    b.step_main(stream)
    b.gather(stream)
    recs, _ = Z.zero_trace_read(b.ctx)
    Z.zero_trace_stop(b.ctx)
    per_call = {}
    for name, _, t_ms in recs:
        e = per_call.setdefault(name, {"calls": 0, "ms": 0.0})
        e["calls"] += 1
        e["ms"] += t_ms

    step_bytes, main_bytes = b.step_bytes()
    peak, peak_src = hbm_peak()
    kavg = statistics.mean(kern_ms)
    achieved = main_bytes / (kavg * 1e-3) / 1e9
    # the library's dispatch: R <= 2 runs the fused step on the staged kernel
    # (the fused last micro-batch stays on the register kernel); the step from
    # the accumulators is the staged kernel at every R
    fused = "fused_step_tma_kernel" if b.R <= 2 else "fused_step_kernel"
    kernel_name = "reduce_scatter+step_from_acc_tma_kernel" if b.twopass else fused
    if b.twopass and (b.accum > 1 or b.clip > 0):
        kernel_name += f" (accum {b.accum}{', clip' if b.clip > 0 else ''})"
    elif b.clip > 0:
        kernel_name = f"grad_norm+{fused} (clip)"
    elif b.accum > 1:
        kernel_name = f"reduce_scatter+fused_step_kernel (accum {b.accum}, last micro-batch fused)"
    # the stored counters describe the full workload on the ping-pong fused
    # path; any other configuration reports no traffic
    same_config = args.tensor_range is None and b.path == "pingpong"
    traffic = profiled_traffic(kernel_name, args.workload) if same_config else None
    clip_label = ("" if b.clip <= 0 else
                  "global-norm clip from the reduce-scatters' norm shares, " if b.rs_norm else
                  "global-norm clip pass, ")
    out = {
        "metric": METRIC,
        "value": units / (ms * 1e-3),
        "unit": "params/s",
        "n_gpus": world,
        "steps": K,
        "warmup": args.warmup,
        "ms_per_step": ms / K,
        "higher_is_better": True,
        "scaling": "weak",
        "vs_baseline": None,
        "dtype": "f32",
        "data": "synthetic",
        "hbm_gbs": step_bytes * K * world / (ms * 1e-3) / 1e9,
        "hbm_frac_of_peak": step_bytes * K / (ms * 1e-3) / 1e9 / peak,
        "config": job_config(args, world, b.wl, b.R, b.T, b.S, len(b.plan.layers), False),
        "step": {
            "path": {"pingpong": f"{'global-norm clip pass, ' if b.clip > 0 else ''}"
                                 f"{f'{b.accum - 1} micro-batch(es) reduce-scattered, last ' if b.accum > 1 else ''}"
                                 "fused reduce-scatter+AdamW, ping-pong state",
                     "inplace": f"{'global-norm clip pass, ' if b.clip > 0 else ''}"
                                "fused reduce-scatter+AdamW, in place",
                     "twopass": f"bucketed reduce-scatter ({b.accum} micro-batch(es), "
                       f"{len(b.plan.buckets)} buckets in {len(b.rs_runs)} grouped launches each), "
                       f"{clip_label}"
                       "then AdamW from fp32 accumulators, in place",
                     "twopass_pingpong": f"bucketed reduce-scatter ({b.accum} micro-batch(es), "
                       f"{len(b.plan.buckets)} buckets in {len(b.rs_runs)} grouped launches each), "
                       f"{clip_label}"
                       "then AdamW from fp32 accumulators, ping-pong state"}[b.path]
                    + " + device loss-scale update + ZeRO-3 gather of every layer",
            "gather": (f"{len(b.gather_buckets)} bucketed launches of consecutive layers "
                       f"(<= {args.gather_bucket} elements each)" if b.gather_buckets
                       else f"{len(b.plan.layers)} per-layer launches"),
            "bytes_per_step": step_bytes,
            "launch": "CUDA graph replay (step graph, event, gather graph), captured through the C ABI"
                      if args.graph else "eager launches through the C ABI",
        },
        "roofline": {"bound": "hbm", "kernel": kernel_name, "achieved": achieved, "peak": peak,
                     "peak_source": f"{peak_src} hbm_gbs", "unit": "GB/s", "frac": achieved / peak,
                     "frac_of_nominal": achieved / NOMINAL_HBM_GBS,
                     "traffic": traffic, "algorithmic_bytes_per_launch": main_bytes,
                     "avg_launch_ms": kavg},
        "gather": {"avg_ms_per_step": gather_ms, "elements": b.L,
                   "gbs": 4.0 * b.L / (gather_ms * 1e-3) / 1e9,
                   "launches_per_step": len(b.gather_buckets) or len(b.plan.layers)},
        "clocks": clk,
        "gpu_launches": K * b.launches_per_step(),
        "trace_one_step": {"source": "zero_trace_read, one untimed step after the timed region",
                           "calls": per_call},
    }
    if not args.no_e2e:
        out["e2e"] = e2e(b, args, stream, world)
    b.graphs = None
    b.step_graphs, b.gather_graph = {}, None
    b.close()
    del b
    torch.cuda.empty_cache()
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        out["cpu_baseline"] = cpu_baseline(args.workload)
    if rank == 0:
        print(json.dumps(out), flush=True)


def e2e(b, args, stream, world):
    """The same metric through the C ABI with host buffers. Every step
    copies its R gradient replicas from pinned host memory, runs the step and
    the gathers, and reads the step's products back to pinned host memory:
    the updated half parameters of every shard (the model the next forward
    uses) and the loss-scale state (overflow, skip, scale, grad norm; this
    read synchronizes). The replicas are double-buffered where a second set
    fits: step s+1's upload runs on one copy stream while step s computes
    (with graphs, one step graph per buffer set), and step s's parameters go
    down on a second copy stream while step s+1 computes. Every copy is
    inside the timed region."""
    host = [g.cpu().pin_memory() for g in b.grads]
    half = b.grads[0].dtype
    host_param = [torch.empty(b.S, dtype=half).pin_memory() for _ in range(b.R)]
    K = max(3, min(args.steps, 10))
    nbytes = sum(h.numel() * h.element_size() for h in host)
    dbytes = sum(h.numel() * h.element_size() for h in host_param) + 40
    graphs = getattr(b, "graphs", None)
    room = torch.cuda.mem_get_info()[0] > 1.25 * nbytes
    bufs = [b.grads] if not room else [b.grads, [torch.empty_like(g) for g in b.grads]]
    if graphs and len(bufs) == 2:
        b.capture_step(stream, bufs[1])
    up, down = torch.cuda.Stream(), torch.cuda.Stream()
    copied = [torch.cuda.Event() for _ in bufs]
    consumed = [torch.cuda.Event() for _ in bufs]
    downloaded = [torch.cuda.Event() for _ in range(2)]
    # a step writes set 1-cur (two sets) or set cur (one): the download that
    # reads those parameters, step s-2's or step s-1's, must be done first
    lag = 2 if b.state.sets == 2 else 1

    def upload(i):
        k = i % len(bufs)
        up.wait_event(consumed[k])  # the step that last read this buffer is done
        with torch.cuda.stream(up):
            for r in range(b.R):
                bufs[k][r].copy_(host[r], non_blocking=True)
        copied[k].record(up)

    def run(n):
        for i in range(min(len(bufs), n)):
            upload(i)
        for i in range(n):
            k = i % len(bufs)
            stream.wait_event(copied[k])
            if i >= lag:
                stream.wait_event(downloaded[(i - lag) % 2])
            b.step(stream, grads=bufs[k])
            consumed[k].record(stream)
            cur = b.loss_scale(stream)["cur"]  # synchronizes: the state is on the host
            down.wait_stream(stream)
            with torch.cuda.stream(down):
                for r in range(b.R):
                    host_param[r].copy_(b.state.param[cur][r], non_blocking=True)
            downloaded[i % 2].record(down)
            if i + len(bufs) < n:
                upload(i + len(bufs))
        stream.wait_stream(down)  # the last parameters are on the host

    for e in consumed:
        e.record(stream)
    run(2)
    start, end = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    barrier(world)
    torch.cuda.synchronize()
    start.record(stream)
    run(K)
    end.record(stream)
    torch.cuda.synchronize()
    ms, units = aggregate(start.elapsed_time(end), float(b.P) * K, world)
    return {"value": units / (ms * 1e-3), "unit": "params/s", "h2d_bytes_per_step": nbytes * world,
            "d2h_bytes_per_step": dbytes * world, "steps": K,
            "d2h": "updated half parameters of every shard (2 B x T) + loss-scale state (40 B)",
            "pipelining": ("double-buffered replicas: step s+1 uploads during step s; step s's "
                           "parameters download during step s+1") if len(bufs) == 2
                          else "parameters download during the next step; one set of replicas"}


# ---- the CPU oracle as a baseline ----------------------------------------------

def oracle_inputs(name, n, R=None):
    """The oracle's state, replicas, hyper-parameters and loss-scale state
    for the first n params of the workload (R replicas: the workload's own
    count unless given)."""
    import oracle as O
    import synth
    wl = synth.workload(name)
    R, dtype = R or wl["R"], wl["dtype"]
    scale = wl["init_scale"] if wl["mode"] != synth.NONE else 1.0
    numels, left = [], n
    for k in wl["numels"]:
        if left <= 0:
            break
        numels.append(min(k, left))
        left -= numels[-1]
    x = torch.cat([synth.tensor_master(c, wl["index"], k, "cpu") for k, c in enumerate(numels)])
    g = np.stack([torch.cat([synth.tensor_grads(c, wl["dist"], wl["sigma"], scale, dtype,
                                                wl["index"], 1, r, k, "cpu")
                             for k, c in enumerate(numels)]).view(torch.int16).numpy()
                  .view(np.uint16) for r in range(R)])
    hp = O.AdamW(**{k: wl["hp"][k] for k in ("lr", "beta1", "beta2", "eps", "weight_decay")})
    fsm = O.make_fsm(wl["mode"], scale=scale, interval=wl["interval"])
    return O.State(x.numpy(), dtype), g, hp, fsm


def oracle_sample(name, target_s=10.0, max_elems=1 << 26):
    """Time the oracle's step on a prefix sample of the workload, sized for
    about target_s seconds. Returns (params/s, sample elements, seconds)."""
    import oracle as O
    n = 1 << 18
    st, g, hp, fsm = oracle_inputs(name, n)
    t = time.perf_counter()
    O.step(st, g, hp, fsm)
    rate = n / (time.perf_counter() - t)
    n = int(min(max_elems, max(n, rate * target_s)))
    st, g, hp, fsm = oracle_inputs(name, n)
    t = time.perf_counter()
    O.step(st, g, hp, fsm)
    dt = time.perf_counter() - t
    return n / dt, n, dt, (st, g, hp, fsm)


def _oracle_crew_worker(name, n, R, barrier, conn):
    """One single-threaded oracle process of OracleCrew: builds its sample,
    then on each request runs k steps between a common barrier and reports
    its start and end time (CLOCK_MONOTONIC, comparable across processes)."""
    import oracle as O
    torch.set_num_threads(1)
    st, g, hp, fsm = oracle_inputs(name, n, R)
    conn.send("ready")
    while True:
        k = conn.recv()
        if k is None:
            break
        barrier.wait()
        t0 = time.perf_counter()
        for _ in range(k):
            O.step(st, g, hp, fsm)
        conn.send((t0, time.perf_counter()))


class OracleCrew:
    """The oracle, as it stands, on every host core: one spawned process per
    hardware thread, each stepping its own copy of the same prefix sample.
    Throughput = processes x sample x steps / (last end - first start)."""

    def __init__(self, name, n, procs=None, R=None):
        import multiprocessing as mp
        ctx = mp.get_context("spawn")  # never fork a process that holds CUDA
        self.n, self.procs = n, procs or (os.cpu_count() or 1)
        self.barrier = ctx.Barrier(self.procs)
        self.conns, self.ps = [], []
        old = {k: os.environ.get(k) for k in ("OMP_NUM_THREADS", "MKL_NUM_THREADS")}
        os.environ.update(OMP_NUM_THREADS="1", MKL_NUM_THREADS="1")
        try:
            for _ in range(self.procs):
                a, b = ctx.Pipe()
                p = ctx.Process(target=_oracle_crew_worker, args=(name, n, R, self.barrier, b), daemon=True)
                p.start()
                self.conns.append(a)
                self.ps.append(p)
        finally:
            for k, v in old.items():
                if v is None:
                    os.environ.pop(k, None)
                else:
                    os.environ[k] = v
        for c in self.conns:
            assert c.recv() == "ready"

    def run(self, k):
        """k steps in every process; returns (params/s, seconds)."""
        for c in self.conns:
            c.send(k)
        spans = [c.recv() for c in self.conns]
        sec = max(t1 for _, t1 in spans) - min(t0 for t0, _ in spans)
        return self.procs * self.n * k / sec, sec

    def close(self):
        for c in self.conns:
            c.send(None)
        for p in self.ps:
            p.join(timeout=30)


def cpu_baseline(name):
    """The oracle on all host cores (one process per hardware thread), plus
    its single-threaded rate."""
    rate1, n1, dt1, _ = oracle_sample(name)
    n = 1 << 22
    crew = OracleCrew(name, n)
    try:
        crew.run(1)  # warm-up
        rate, sec = crew.run(2)
    finally:
        crew.close()
    return {"value": rate, "unit": "params/s", "cores": crew.procs, "kind": "oracle",
            "sample": f"{crew.procs} single-threaded processes, each 2 steps of the first {n} params of "
                      f"{name} (all R replicas), {sec:.1f} s",
            "single_thread": {"value": rate1, "cores": 1,
                              "sample": f"one step of the first {n1} params, {dt1:.1f} s"}}


def run_overlap(args, world, rank, local):
    """A synthetic ZeRO-3 training step on the workload's layers: forward
    (gather layer, one bf16 GEMM of 2 * tokens * n_layer flops on it), backward
    (gather again, two GEMMs, report the layer's gradients), then the two-pass
    optimizer step. Timed three ways: overlapped through the scheduler's
    communication stream and look-ahead ring, serialized on one stream, and
    compute only (no gathers, no reduce-scatters)."""
    if not torch.cuda.is_available():
        print(json.dumps({"error": "no CUDA device"}))
        sys.exit(1)
    b = Bench(args.workload, "twopass", args.tensor_range, 0, bucket_elems=args.bucket_elems)
    Z = b.Z
    stream = torch.cuda.current_stream()
    wl, plan = b.wl, b.plan
    d = 768 if args.workload == "gpt2s" else 2048
    nl = len(plan.layers)
    lids = wl["layer_ids"]
    first_t = [lids.index(l) for l in range(nl)]
    count_t = [lids.count(l) for l in range(nl)]
    biggest = b.max_layer
    nbufs, depth = 3, 1
    bufs = [torch.empty(biggest + 8, dtype=torch.bfloat16, device="cuda") for _ in range(nbufs)]
    by_addr = {t.data_ptr(): t for t in bufs}
    x = torch.randn(args.tokens, d, device="cuda", dtype=torch.bfloat16)

    def gemm(buf, l):
        # [tokens x d] @ [d x N] on the gathered layer; N a multiple of 64 keeps
        # the operand aligned for the tensor-core GEMM path
        lo, hi = plan.layers[l]
        n = ((hi - lo) // (d * 64)) * (d * 64)
        w = buf[:n].view(d, n // d)
        return x @ w

    def step_overlap():
        Z.zero_prefetch_begin(b.ctx, b.state.handle, bufs, depth, 1, stream)
        for l in range(nl):
            buf = by_addr[Z.zero_layer_acquire(b.ctx, l, stream)]
            gemm(buf, l)
            Z.zero_layer_release(b.ctx, l, stream)
        Z.zero_prefetch_begin(b.ctx, b.state.handle, bufs, depth, -1, stream)
        for l in reversed(range(nl)):
            buf = by_addr[Z.zero_layer_acquire(b.ctx, l, stream)]
            gemm(buf, l)
            gemm(buf, l)
            Z.zero_layer_release(b.ctx, l, stream)
            Z.zero_grads_ready(b.ctx, first_t[l], count_t[l], b.grads, b.state.acc, 0, stream)
        Z.zero_grads_join(b.ctx, stream)
        Z.zero_step(b.ctx, wl["hp"], b.state.handle, None, stream)

    def step_serial(comm=True):
        buf = bufs[0]
        for l in range(nl):
            if comm:
                Z.zero_gather_layer(b.ctx, l, b.state.handle, buf, stream)
            gemm(buf, l)
        done = 0
        for l in reversed(range(nl)):
            if comm:
                Z.zero_gather_layer(b.ctx, l, b.state.handle, buf, stream)
            gemm(buf, l)
            gemm(buf, l)
            # buckets complete once all their tensors (from the last one down) are done
            lowest = first_t[l]
            while comm and done < len(plan.buckets) and plan.buckets[done][0] >= plan.offsets[lowest]:
                Z.zero_reduce_scatter_bucket(b.ctx, done, b.grads, b.state.acc, stream)
                done += 1
        Z.zero_step(b.ctx, wl["hp"], b.state.handle, None, stream)

    def timed(fn, reps):
        for _ in range(args.warmup):
            fn()
        torch.cuda.synchronize()
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        e0.record(stream)
        for _ in range(reps):
            fn()
        e1.record(stream)
        torch.cuda.synchronize()
        return e0.elapsed_time(e1) / reps

    if args.carveout:
        torch._C._set_sm_carveout_experimental(args.carveout)
    Z.zero_sched_set_comm_sms(b.ctx, args.comm_sms)
    reps = max(3, min(args.steps, 50))
    # fill the accumulators once; the compute-only variant steps from them
    Z.zero_reduce_scatter_bucket(b.ctx, -1, b.grads, b.state.acc, stream)
    t_ovl = timed(step_overlap, reps)
    t_ser = timed(step_serial, reps)
    t_cmp = timed(lambda: step_serial(comm=False), reps)
    hidden = (t_ser - t_ovl) / (t_ser - t_cmp) if t_ser > t_cmp else None
    gemm_flops = 6.0 * args.tokens * sum(((hi - lo) // (d * 64)) * (d * 64) for lo, hi in plan.layers)
    out = {"mode": "overlap", "workload": args.workload, "tokens": args.tokens,
           "bucket_elems": wl["bucket_elems"],
           "gemm_carveout_sms": args.carveout, "comm_kernel_sms": args.comm_sms,
           "gemm_tflops_in_compute_only": gemm_flops / (t_cmp * 1e-3) / 1e12,
           "layers": nl, "buckets": len(plan.buckets), "ring": {"nbufs": nbufs, "depth": depth},
           "ms_overlapped": t_ovl, "ms_serialized": t_ser,
           "ms_compute_and_step_only": t_cmp,
           "comm_ms_serialized": t_ser - t_cmp, "comm_ms_exposed_overlapped": t_ovl - t_cmp,
           "fraction_of_comm_hidden": hidden, "steps": reps}
    b.close()
    if rank == 0:
        print(json.dumps(out), flush=True)


def run_rs_sweep(args, world, rank, local):
    """The bucketed reduce-scatter (one pass over every bucket of the plan)
    against bucket size, on the workload's tensors: for each size a plan is
    built (the flat layout does not depend on it), and the pass is timed
    issued launch by launch, replayed from a CUDA graph, and with consecutive
    buckets grouped into launches of about 25M elements. Reported as the
    kernel's algorithmic (2R + 4) bytes per padded element over the pass."""
    if not torch.cuda.is_available():
        print(json.dumps({"error": "no CUDA device"}))
        sys.exit(1)
    import zero_partitioned_mixed_reduce_b200 as Z
    import synth
    wl = synth.workload(args.workload)
    R, dtype = wl["R"], wl["dtype"]
    sizes = [int(x) for x in args.rs_sizes.split(",")]
    base = Z.Plan(wl["numels"], wl["layer_ids"], R, dtype, 8, 0)
    T, S = base.T, base.S
    scale = wl["init_scale"] if wl["mode"] != synth.NONE else 1.0
    grads = [base.pack(synth.flat_grads(wl, 1, r, scale, "cuda")) for r in range(R)]
    acc = [torch.empty(S, dtype=torch.float32, device="cuda") for _ in range(R)]
    stream = torch.cuda.current_stream()
    nbytes = (2 * R + 4) * T
    peak, peak_src = hbm_peak()
    reps = max(3, min(args.steps, 50))

    def timed(fn):
        for _ in range(args.warmup):
            fn()
        torch.cuda.synchronize()
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        e0.record(stream)
        for _ in range(reps):
            fn()
        e1.record(stream)
        torch.cuda.synchronize()
        return e0.elapsed_time(e1) / reps

    rows = []
    for size in sizes:
        plan = Z.Plan(wl["numels"], wl["layer_ids"], R, dtype, 8, size)
        assert plan.T == T
        ctx = Z.zero_ctx_create(plan.handle, wl["mode"], wl["init_scale"], wl["interval"])
        nb = len(plan.buckets)

        def one_pass(s=stream):
            for b in range(nb):
                Z.zero_reduce_scatter_bucket(ctx, b, grads, acc, s)

        # consecutive buckets grouped into launches of about 25M elements
        # (zero_reduce_scatter_buckets), as a caller reporting a layer at a
        # time would issue them
        group = max(1, (25 << 20) // size) if size > 0 else 1
        runs = [(b, min(group, nb - b)) for b in range(0, nb, group)]

        def grouped_pass(s=stream):
            for first, count in runs:
                Z.zero_reduce_scatter_buckets(ctx, first, count, grads, acc, 0, s)

        t_eager = timed(one_pass)
        t_grouped = timed(grouped_pass)
        side = torch.cuda.Stream()
        side.wait_stream(stream)
        g = torch.cuda.CUDAGraph()
        with torch.cuda.graph(g, stream=side):
            one_pass(torch.cuda.current_stream())
        stream.wait_stream(side)
        t_graph = timed(g.replay)
        del g
        fl = Z.zero_loss_scale(ctx)
        Z.zero_ctx_destroy(ctx)
        rows.append({"bucket_elems": size if size > 0 else "whole model", "buckets": nb,
                     "ms_eager": t_eager, "ms_graph": t_graph,
                     "grouped_launches": len(runs), "ms_grouped": t_grouped,
                     "gbs_grouped": nbytes / (t_grouped * 1e-3) / 1e9,
                     "gbs_eager": nbytes / (t_eager * 1e-3) / 1e9,
                     "gbs_graph": nbytes / (t_graph * 1e-3) / 1e9,
                     "frac_graph": nbytes / (t_graph * 1e-3) / 1e9 / peak,
                     "overflow_flag": fl["last_overflow"]})
    out = {"mode": "reduce_scatter_bucket_sweep", "workload": args.workload, "R": R, "T": T,
           "P": base.P, "tensors": len(wl["numels"]), "algorithmic_bytes_per_pass": nbytes,
           "peak": peak, "peak_source": f"{peak_src} hbm_gbs", "reps": reps,
           "l2": f"inputs larger than L2 ({nbytes / 1e9:.1f} GB per pass)", "rows": rows}
    if rank == 0:
        print(json.dumps(out), flush=True)


def dist_layer_buckets(layers, cap):
    """Consecutive layers gathered in one launch, up to `cap` elements (a
    larger layer alone) and 64 layers; each layer lands in its own
    16-byte-aligned slice of one bucket buffer. Returns [(first, offsets, size)]."""
    buckets, first, size, offs = [], 0, 0, []
    for l, (lo, hi) in enumerate(layers):
        n = hi - lo
        if offs and (size + n > cap or len(offs) == 64):
            buckets.append((first, offs, size))
            first, size, offs = l, 0, []
        offs.append(size)
        size += (n + 7) // 8 * 8
    buckets.append((first, offs, size))
    return buckets


def dist_step_bytes(T, S, N, push=False):
    """Algorithmic bytes of one rank's share of the sharded step.
    hbm: the fused launch reads the rank's own replica slice and serves its
    N - 1 peers theirs (2N S), reads and writes its state (26 S); the gathers
    read every rank's parameter slice (2T across all ranks, each rank
    serving its own 2S to N readers: 2N S) and write the whole model (2T).
    nvlink: the bytes the rank reads from its peers (per direction, the same
    amount it serves them): 2(N - 1) S in the step, 2(N - 1) S in the gathers.
    push (ZeRO-1/2): no gathers; the step also writes the whole model into the
    rank's full buffer (its own 2S, and 2(N - 1) S its peers push: 2T of HBM
    writes) and pushes its 2S to each of its N - 1 peers, the same 2(N - 1) S
    per direction that the gathers would have moved, now during the step."""
    step_hbm = (2 * N + 26) * S + (2 * T if push else 0)
    gather_hbm = 0 if push else 2 * N * S + 2 * T
    nvlink_step = 2 * (N - 1) * S + (2 * (N - 1) * S if push else 0)
    nvlink_gather = 0 if push else 2 * (N - 1) * S
    return {"step_hbm": step_hbm, "gather_hbm": gather_hbm, "nvlink_step": nvlink_step,
            "nvlink_gather": nvlink_gather}


NVLINK_PEER_GBS = 770.0  # measured peer copy per direction on this part (900 nominal)


def dist_roofline(nbytes, ms, peak_hbm):
    """The slower of the HBM stream and the NVLink reads bounds a sharded
    launch; achieved is that resource's bytes over the measured time."""
    t_hbm = nbytes["hbm"] / (peak_hbm * 1e9)
    t_nvl = nbytes["nvlink"] / (NVLINK_PEER_GBS * 1e9)
    if nbytes["nvlink"] > 0 and t_nvl > t_hbm:
        achieved = nbytes["nvlink"] / (ms * 1e-3) / 1e9
        return {"bound": "nvlink", "achieved": achieved, "peak": NVLINK_PEER_GBS,
                "peak_source": "measured peer copy per direction", "unit": "GB/s",
                "frac": achieved / NVLINK_PEER_GBS, "target_ms": 1e3 * t_nvl}
    achieved = nbytes["hbm"] / (ms * 1e-3) / 1e9
    return {"bound": "hbm", "achieved": achieved, "peak": peak_hbm, "unit": "GB/s",
            "frac": achieved / peak_hbm, "target_ms": 1e3 * t_hbm}


def run_dist(args, world, rank, local):
    """The real multi-GPU ZeRO step (DistributedZero): the workload's tensors
    sharded over the N GPUs of the job, each rank owning one shard and reading
    its peers' gradient replicas over NVLink inside the fused step, then the
    ZeRO-3 gathers of every layer from every rank's shard. Strong scaling:
    the model is fixed, N ranks share it. Each rank writes its own replica."""
    import socket
    import torch.distributed as dist
    import synth
    from zero_partitioned_mixed_reduce_b200.dist import DistributedZero
    if not torch.cuda.is_available():
        print(json.dumps({"error": "no CUDA device: the benchmark has no CPU fallback"}))
        sys.exit(1)
    if not dist.is_initialized():  # one process: a group of one
        with socket.socket() as sk:
            sk.bind(("127.0.0.1", 0))
            port = sk.getsockname()[1]
        os.environ.setdefault("MASTER_ADDR", "127.0.0.1")
        os.environ.setdefault("MASTER_PORT", str(port))
        dist.init_process_group("nccl", rank=0, world_size=1, timeout=datetime.timedelta(seconds=300))
    N = dist.get_world_size()
    wl = synth.workload(args.workload)
    restrict(wl, args.tensor_range)
    dz = DistributedZero(wl["numels"], wl["layer_ids"], wl["dtype"], wl["mode"], wl["init_scale"],
                         wl["interval"], 8, wl["bucket_elems"], push_params=args.zero2)
    plan = dz.plan
    T, S = plan.T, plan.S
    half = {0: torch.bfloat16, 1: torch.float16}[wl["dtype"]]
    x = torch.cat([synth.tensor_master(n, wl["index"], k, "cuda") for k, n in enumerate(wl["numels"])])
    dz.load(plan.pack(x), plan.pack(x.to(half)))
    del x
    scale = wl["init_scale"] if wl["mode"] != synth.NONE else 1.0
    for k, (n, off) in enumerate(zip(wl["numels"], plan.offsets)):
        dz.grads[off:off + n] = synth.tensor_grads(n, wl["dist"], wl["sigma"], scale, wl["dtype"], wl["index"],
                                                   1, dz.rank, k, "cuda")
    torch.cuda.synchronize()
    # ZeRO-3 gathers of every layer, bucketed as in the single-GPU step
    buckets = dist_layer_buckets(plan.layers, args.gather_bucket if args.gather_bucket > 0 else 1)
    layer_buf = torch.empty(max(b[2] for b in buckets), dtype=half, device="cuda")
    outs = [[layer_buf.data_ptr() + 2 * o for o in offs] for _, offs, _ in buckets]
    hp = wl["hp"]
    stream = torch.cuda.current_stream()

    def step(ev=None):
        if ev is not None:
            ev[0].record(stream)
        dz.step(hp)
        if ev is not None:
            ev[1].record(stream)
        if not args.zero2:  # ZeRO-2 pushed the parameters within the step
            for (f, _, _), o in zip(buckets, outs):
                dz.gather_layers(f, o)
        if ev is not None:
            ev[2].record(stream)

    for _ in range(args.warmup):
        step()
    torch.cuda.synchronize()
    f0 = dz.loss_scale()
    K = args.steps
    evs = [tuple(torch.cuda.Event(enable_timing=True) for _ in range(3)) for _ in range(K)]
    start, end = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    clocks = ClockSampler(local)
    clocks.start()
    dist.barrier()
    torch.cuda.synchronize()
    start.record(stream)
    for i in range(K):
        step(evs[i])
    end.record(stream)
    torch.cuda.synchronize()
    dist.barrier()
    clk = clocks.stop()
    f1 = dz.loss_scale()
    ok = f1["last_overflow"] == 0 and f1["t"] == f0["t"] + K
    ms, units = aggregate(start.elapsed_time(end), float(plan.P) * K / N, N)
    step_ms, _ = aggregate(statistics.mean(e0.elapsed_time(e1) for e0, e1, _ in evs), 0.0, N)
    gather_ms, _ = aggregate(statistics.mean(e1.elapsed_time(e2) for _, e1, e2 in evs), 0.0, N)
    nb = dist_step_bytes(T, S, N, push=args.zero2)
    peak, peak_src = hbm_peak()
    roof = dist_roofline({"hbm": nb["step_hbm"], "nvlink": nb["nvlink_step"]}, step_ms, peak)
    roof.update({"kernel": "fused_step_kernel (sharded: one owner per rank) + loss-scale commit",
                 "traffic": None, "algorithmic_bytes_per_launch": nb["step_hbm"], "avg_launch_ms": step_ms})
    roof.setdefault("peak_source", f"{peak_src} hbm_gbs")
    e2e_out = None if args.no_e2e else dist_e2e(dz, step, args, stream, N)
    out = {
        "metric": METRIC, "value": units / (ms * 1e-3), "unit": "params/s",
        "n_gpus": N, "steps": K, "warmup": args.warmup, "ms_per_step": ms / K, "higher_is_better": True,
        "scaling": "strong", "vs_baseline": None, "dtype": "f32", "data": "synthetic",
        "config": job_config(args, N, wl, N, T, S, len(plan.layers), True),
        "step": {"path": "DistributedZero: 4-byte NCCL all-reduce (every replica written), fused "
                           "reduce-scatter+AdamW over the rank's shard reading the peers' replicas over "
                           "NVLink (plain or 1-D bulk loads, no multicast)"
                           + (", the updated parameters pushed into every rank's full-model buffer by the "
                              "same kernel (ZeRO-1/2)" if args.zero2 else "")
                           + ", 16-byte NCCL all-reduce of {norm, overflow}, loss-scale commit"
                           + ("" if args.zero2 else ", ZeRO-3 gather of every layer from every rank's shard"),
                 "bytes_per_rank_per_step": nb["step_hbm"] + nb["gather_hbm"],
                 "gather": ("none: the step pushes the parameters (ZeRO-1/2)" if args.zero2 else
                              f"{len(buckets)} bucketed launches per step over every rank's shard"),
                 "launch": "eager (the step issues NCCL all-reduces between its launches)"},
        "roofline": roof,
        "gather": None if args.zero2 else {
            "avg_ms_per_step": gather_ms, "elements": plan.L, "launches_per_step": len(buckets),
            "roofline": dist_roofline({"hbm": nb["gather_hbm"], "nvlink": nb["nvlink_gather"]}, gather_ms, peak)},
        "per_rank_bytes": nb,
        "nccl": {"backend": dist.get_backend(), "world_size": N,
                 "version": ".".join(str(v) for v in torch.cuda.nccl.version())},
        "clocks": clk,
        "gpu_launches": K * (2 + (0 if args.zero2 else len(buckets))),
        "state_check": "ok" if ok else f"t {f0['t']} -> {f1['t']}, overflow {f1['last_overflow']}",
    }
    if e2e_out is not None:
        out["e2e"] = e2e_out
    dz.close()
    if rank == 0:
        print(json.dumps(out), flush=True)


def dist_e2e(dz, step, args, stream, N):
    """The sharded step through the public API with host buffers: every rank
    uploads its gradient replica from pinned host memory, runs the step and
    the gathers, and reads back its updated parameter shard and the loss-scale
    state (which synchronizes). Time: max over ranks."""
    import torch.distributed as dist
    host_g = dz.grads.cpu().pin_memory()
    host_p = torch.empty(dz.plan.S, dtype=dz.grads.dtype).pin_memory()
    K = max(3, min(args.steps, 10))

    def one():
        dz.grads.copy_(host_g, non_blocking=True)
        step()
        host_p.copy_(dz.current("param"), non_blocking=True)
        dz.loss_scale()

    one()
    start, end = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    dist.barrier()
    torch.cuda.synchronize()
    start.record(stream)
    for _ in range(K):
        one()
    end.record(stream)
    torch.cuda.synchronize()
    ms, units = aggregate(start.elapsed_time(end), float(dz.plan.P) * K / N, N)
    return {"value": units / (ms * 1e-3), "unit": "params/s",
            "h2d_bytes_per_step": host_g.numel() * host_g.element_size() * N,
            "d2h_bytes_per_step": (host_p.numel() * host_p.element_size() + 40) * N, "steps": K,
            "pipelining": "none: each rank uploads, steps, gathers and reads back in turn"}


def run_offload(args, world, rank, local):
    """ZeRO-Offload on the workload: per step the GPU runs a synthetic
    forward/backward (bf16 GEMMs of 6 * tokens * P flops) and reduce-scatters
    the gradients; the fp32 accumulators go to pinned host memory, the AdamW
    step runs on CPU threads (zero_cpu_step) and the half parameters come back.
    Timed serialized and with the one-step delayed parameter update (the CPU
    step of step s overlapping the GPU work of step s+1)."""
    import threading
    if not torch.cuda.is_available():
        print(json.dumps({"error": "no CUDA device"}))
        sys.exit(1)
    import zero_partitioned_mixed_reduce_b200 as Z
    import synth
    wl = synth.workload(args.workload)
    restrict(wl, args.tensor_range)
    plan = Z.Plan(wl["numels"], wl["layer_ids"], wl["R"], wl["dtype"], 8, wl["bucket_elems"])
    R, S, T, P = plan.R, plan.S, plan.T, plan.P
    half = Z.state.HALF[wl["dtype"]]
    ctx = Z.zero_ctx_create(plan.handle, wl["mode"], wl["init_scale"], wl["interval"])
    scale = wl["init_scale"] if wl["mode"] != synth.NONE else 1.0
    grads = []
    for r in range(R):
        g = torch.zeros(T, dtype=half, device="cuda")
        for k, (n, off) in enumerate(zip(wl["numels"], plan.offsets)):
            g[off:off + n] = synth.tensor_grads(n, wl["dist"], wl["sigma"], scale, wl["dtype"],
                                                wl["index"], 1, r, k, "cuda")
        grads.append(g)
    acc_gpu = [torch.zeros(S, device="cuda") for _ in range(R)]
    pin = lambda t: t.pin_memory()
    master = [pin(torch.randn(S) * 0.02) for _ in range(R)]
    m = [pin(torch.zeros(S)) for _ in range(R)]
    v = [pin(torch.zeros(S)) for _ in range(R)]
    param_host = [pin(torch.zeros(S, dtype=half)) for _ in range(R)]
    acc_host = [[pin(torch.zeros(S)) for _ in range(R)] for _ in range(2)]
    # the reduce-scatters' overflow flag, taken on the GPU and copied down with
    # the accumulators: a clean DYNAMIC step then runs in one pass on the CPU
    flag_gpu = torch.zeros(1, dtype=torch.int32, device="cuda")
    flag_host = [pin(torch.zeros(1, dtype=torch.int32)) for _ in range(2)]
    # the reduce-scatters also take the squared norm (ZERO_RS_NORM, with the
    # host's loss scale on the device), copied down with the flag: the split
    # CPU step (and the clipped one under --clip) decides from the two without
    # scanning the host accumulators
    clip_on = args.clip > 0
    norm_gpu = torch.zeros(2, dtype=torch.float64, device="cuda")
    norm_host = [pin(torch.zeros(2, dtype=torch.float64)) for _ in range(2)]
    param_gpu = [torch.zeros(S, dtype=half, device="cuda") for _ in range(R)]
    copy = torch.cuda.Stream()
    d = 768 if args.workload == "gpt2s" else 2048
    x = torch.randn(args.tokens, d, device="cuda", dtype=torch.bfloat16)
    w = torch.randn(d, 8192, device="cuda", dtype=torch.bfloat16)
    n_gemm = max(1, int(round(6.0 * args.tokens * P / (2.0 * args.tokens * d * 8192))))
    cfg = dict(mode=wl["mode"], growth_interval=wl["interval"])
    ls = {"state": dict(scale=scale, cur=0, good=0, t=0), "up": None}
    hp = wl["hp"]

    def gpu_half(slot):
        for _ in range(n_gemm):
            x @ w
        if ls.get("scale_on_device") != ls["state"]["scale"]:  # the host's loss scale moved
            Z.zero_loss_scale(ctx, Z.ZERO_LOSS_SCALE_SET, ls["state"])
            ls["scale_on_device"] = ls["state"]["scale"]
        Z.zero_reduce_scatter_shard(ctx, -1, grads, acc_gpu, 0, R, Z.ZERO_RS_NORM)
        Z.zero_grad_norm_shard(ctx, None, None, 0, R, norm_gpu, 1.0)
        Z.zero_take_overflow(ctx, flag_gpu)
        ev = torch.cuda.Event()
        ev.record()
        copy.wait_event(ev)
        with torch.cuda.stream(copy):
            for r in range(R):
                acc_host[slot][r].copy_(acc_gpu[r], non_blocking=True)
            flag_host[slot].copy_(flag_gpu, non_blocking=True)
            norm_host[slot].copy_(norm_gpu, non_blocking=True)
        done = torch.cuda.Event()
        done.record(copy)
        torch.cuda.current_stream().wait_event(done)
        return done

    # while the CPU step overlaps the GPU work, one hardware thread stays free
    # for the thread that launches it
    ncpu = os.cpu_count() or 1
    nt = {"n": 0}

    def cpu_half(slot, done):
        done.synchronize()
        if ls["up"] is not None:
            ls["up"].synchronize()  # the last upload has finished reading param_host
        if clip_on:
            st = ls["state"]
            dec = decide(slot, st)
            Z.zero_cpu_update(plan.handle, st, hp, dec, acc_host[slot], master, m, v, param_host, 0, S,
                              nthreads=nt["n"])
            ls["state"] = Z.zero_cpu_commit(cfg, st, dec)
            return
        clean = Z.ZERO_STEP_CLEAN if int(flag_host[slot][0]) == 0 else 0
        ls["state"] = Z.zero_cpu_step(plan.handle, cfg, ls["state"], hp, acc_host[slot], master, m, v,
                                      param_host, nthreads=nt["n"], flags=clean)

    def decide(slot, st):
        """The step's decision from the device's norm and flag."""
        reduced = (float(norm_host[slot][0]), float(flag_host[slot][0]))
        return Z.zero_cpu_decide(plan.handle, cfg, st, reduced, 1.0, args.clip if clip_on else 0.0)

    chunks = [(S * i // 8, S * (i + 1) // 8) for i in range(8)]

    def cpu_half_pipelined(slot, done):
        # the update in 8 ranges; each range's half parameters go to the GPU
        # on the copy stream while the next range updates
        done.synchronize()
        if ls["up"] is not None:
            ls["up"].synchronize()
        st = ls["state"]
        dec = decide(slot, st)
        for lo, hi in chunks:
            Z.zero_cpu_update(plan.handle, st, hp, dec, acc_host[slot], master, m, v, param_host, lo, hi,
                              nthreads=nt["n"])
            with torch.cuda.stream(copy):
                for r in range(R):
                    param_gpu[r][lo:hi].copy_(param_host[r][lo:hi], non_blocking=True)
        ls["state"] = Z.zero_cpu_commit(cfg, st, dec)
        ev = torch.cuda.Event()
        ev.record(copy)
        ls["up_pipelined"] = ev

    def upload(pipelined=False):
        if pipelined:  # the ranges were queued by the CPU step itself
            ev = ls["up_pipelined"]
        else:
            with torch.cuda.stream(copy):
                for r in range(R):
                    param_gpu[r].copy_(param_host[r], non_blocking=True)
            ev = torch.cuda.Event()
            ev.record(copy)
        ls["up"] = ev
        torch.cuda.current_stream().wait_event(ev)  # the next forward reads the new parameters

    def run(steps, delayed, pipelined=False):
        nt["n"] = max(1, ncpu - 1) if delayed else 0
        pending = None
        work = cpu_half_pipelined if pipelined else cpu_half
        for s in range(steps):
            done = gpu_half(s % 2)
            if pending is not None:
                pending.join()
                upload(pipelined)
            th = threading.Thread(target=work, args=(s % 2, done))
            th.start()
            if delayed:
                pending = th
            else:
                th.join()
                upload(pipelined)
        if pending is not None:
            pending.join()
            upload(pipelined)
        torch.cuda.synchronize()

    def wall(fn):
        torch.cuda.synchronize()
        t = time.perf_counter()
        fn()
        torch.cuda.synchronize()
        return time.perf_counter() - t

    def med(fn, reps=3):
        # the host is shared: the median of three timed loops
        return sorted(wall(fn) for _ in range(reps))[reps // 2] / K

    K = max(3, min(args.steps, 20))
    run(args.warmup, False)
    t_ser = med(lambda: run(K, False))
    t_dpu = med(lambda: run(K, True))
    t_ser_pipe = med(lambda: run(K, False, True))
    t_dpu_pipe = med(lambda: run(K, True, True))
    # the parts alone
    t_gpu = med(lambda: [gpu_half(0) for _ in range(K)])
    done = gpu_half(0)
    done.synchronize()
    nt["n"] = 0
    t_cpu = med(lambda: [cpu_half(0, done) for _ in range(K)])
    t_up = med(lambda: [upload() for _ in range(K)])
    # the clipped CPU step alone: the host scans every accumulator for the
    # norm first (zero_cpu_step with clipping), against the decision from the
    # norm and flag the GPU took while reducing (ZERO_RS_NORM shares with the
    # host's loss scale on the device, zero_take_overflow), after which the
    # update reads each host accumulator once
    clip = args.clip if clip_on else 1.0
    Z.zero_loss_scale(ctx, Z.ZERO_LOSS_SCALE_SET, ls["state"])
    Z.zero_reduce_scatter_shard(ctx, -1, grads, acc_gpu, 0, R, Z.ZERO_RS_NORM)
    norm_dev = torch.zeros(2, dtype=torch.float64, device="cuda")
    Z.zero_grad_norm_shard(ctx, None, None, 0, R, norm_dev, 1.0)
    Z.zero_take_overflow(ctx, flag_gpu)
    for r in range(R):
        acc_host[0][r].copy_(acc_gpu[r])
    reduced = (float(norm_dev[0].item()), float(flag_gpu.item()))

    def clip_scan():
        ls["state"] = Z.zero_cpu_step(plan.handle, cfg, ls["state"], hp, acc_host[0], master, m, v, param_host,
                                      max_grad_norm=clip)

    def clip_device_norm():
        st = ls["state"]
        dec = Z.zero_cpu_decide(plan.handle, cfg, st, reduced, 1.0, clip)
        Z.zero_cpu_update(plan.handle, st, hp, dec, acc_host[0], master, m, v, param_host, 0, S)
        ls["state"] = Z.zero_cpu_commit(cfg, st, dec)

    t_clip_scan = med(lambda: [clip_scan() for _ in range(K)])
    t_clip_dev = med(lambda: [clip_device_norm() for _ in range(K)])
    # the host's streaming rates, measured now on all hardware threads: a copy
    # (1 read + 1 write) and a triad (2 reads + 1 write) over 1 GiB fp32 buffers
    nthr = torch.get_num_threads()
    torch.set_num_threads(ncpu)
    a, b, c = torch.ones(1 << 28), torch.ones(1 << 28), torch.empty(1 << 28)

    def best_rate(fn, nbytes):
        fn()
        ts = []
        for _ in range(5):
            t = time.perf_counter()
            fn()
            ts.append(time.perf_counter() - t)
        return nbytes / min(ts) / 1e9

    host_copy = best_rate(lambda: c.copy_(a), 2 * 4 * a.numel())
    host_triad = best_rate(lambda: torch.add(a, b, alpha=2.0, out=c), 3 * 4 * a.numel())
    torch.set_num_threads(nthr)
    del a, b, c
    # host bytes per element: acc, master, m, v read and master, m, v, param
    # written (30); a DYNAMIC step runs in one pass when the GPU's overflow flag
    # said clean (the serialized zero_cpu_step here), else it scans the
    # accumulators first (+4); the split steps (pipelined upload, --clip)
    # decide from the device's norm and flag and read them once
    cpu_bpp = 30.0
    out = {"mode": "offload", "workload": args.workload, "P": P, "R": R, "tokens": args.tokens,
           "clip": args.clip if clip_on else None,
           "host_threads": os.cpu_count(), "gemm_flops_per_step": 2.0 * args.tokens * d * 8192 * n_gemm,
           "ms_serialized": t_ser * 1e3, "ms_delayed_update": t_dpu * 1e3,
           "ms_serialized_pipelined_upload": t_ser_pipe * 1e3,
           "ms_delayed_update_pipelined_upload": t_dpu_pipe * 1e3,
           "ms_gpu_part": t_gpu * 1e3, "ms_cpu_adamw": t_cpu * 1e3, "ms_param_upload": t_up * 1e3,
           "cpu_adamw_params_per_s": T / t_cpu, "cpu_adamw_bytes_per_param": cpu_bpp,
           "cpu_adamw_host_GBps": cpu_bpp * T / t_cpu / 1e9,
           "host_copy_GBps": host_copy, "host_triad_GBps": host_triad,
           "cpu_adamw_frac_of_host_stream": cpu_bpp * T / t_cpu / 1e9 / max(host_copy, host_triad),
           "cpu_threads_overlapped": max(1, ncpu - 1),
           "speedup_from_delayed_update": t_ser / t_dpu,
           "clipped_cpu_step": {"max_grad_norm": clip, "ms_host_scan_first": t_clip_scan * 1e3,
                                "ms_norm_from_device": t_clip_dev * 1e3,
                                "speedup": t_clip_scan / t_clip_dev,
                                "host_bytes_per_param": {"host_scan_first": cpu_bpp + 4.0,
                                                         "norm_from_device": cpu_bpp}},
           "steps": K,
           "timing": "host wall clock around synchronized loops (the CPU step is host work), "
                     "median of 3 loops"}
    Z.zero_ctx_destroy(ctx)
    if rank == 0:
        print(json.dumps(out), flush=True)


def run_reference(args, world, rank):
    """The oracle on host cores: each step a bounded prefix sample."""
    if rank != 0:
        return
    import oracle as O
    import synth
    # the same `config` as the GPU arm of this command line: the sharded job
    # over the ranks, else the workload's own simulated ranks
    sharded = args.dist or (world > 1 and not args.replicas)
    wl = synth.workload(args.workload)
    restrict(wl, args.tensor_range)
    R = world if sharded else wl["R"]
    lay = O.Layout(wl["numels"], R, 8, 0, wl["layer_ids"])
    config = job_config(args, world, wl, R, lay.T, lay.S, len(lay.layers), sharded)
    # every host core runs the oracle on its own copy of a 1M-param prefix
    # (all R replicas)
    n = 1 << 20
    crew = OracleCrew(args.workload, n, R=R)
    try:
        crew.run(args.warmup)
        value, sec = crew.run(args.steps)
    finally:
        crew.close()
    out = {
        "impl": "reference", "metric": METRIC, "value": value, "unit": "params/s",
        "n_gpus": world, "steps": args.steps, "warmup": args.warmup,
        "ms_per_step": sec * 1e3 / args.steps, "higher_is_better": True,
        "scaling": "strong" if sharded else "weak",
        "vs_baseline": None, "dtype": "f32", "data": "synthetic",
        "config": config,
        "cpu_baseline": {"value": value, "unit": "params/s", "cores": crew.procs, "kind": "oracle",
                         "sample": f"each step, in each of {crew.procs} single-threaded processes, "
                                   f"the first {n} params of {args.workload} ({R} replicas); "
                                   f"{n * crew.procs} params per step"},
        "e2e": {"value": value, "unit": "params/s", "h2d_bytes_per_step": 0,
                "d2h_bytes_per_step": 0},
    }
    print(json.dumps(out), flush=True)


def choose_mode(args, world):
    """The measurement a command line asks for. With N > 1 GPUs the default
    is the real sharded step over the job (DistributedZero); `--replicas`
    keeps N independent single-GPU copies instead."""
    if args.impl == "reference":
        return "reference"
    if args.overlap:
        return "overlap"
    if args.offload:
        return "offload"
    if args.rs_sweep:
        return "rs_sweep"
    if args.dist or (world > 1 and not args.replicas):
        return "dist"
    return "single"


def main(argv=None):
    args = parse_args(argv)
    world = int(os.environ.get("WORLD_SIZE", "1"))
    mode = choose_mode(args, world)
    if mode == "dist" and world > 1 and "NCCL_DEBUG" not in os.environ:
        # the communicators' set-up lines (ranks, devices, transports) on stderr,
        # so that a log shows how many ranks the step ran over
        os.environ.update(NCCL_DEBUG="INFO", NCCL_DEBUG_SUBSYS="INIT", NCCL_DEBUG_FILE="/dev/stderr")
    world, rank, local = dist_init()
    try:
        if mode == "reference":
            run_reference(args, world, rank)
        elif mode == "overlap":
            run_overlap(args, world, rank, local)
        elif mode == "offload":
            run_offload(args, world, rank, local)
        elif mode == "rs_sweep":
            run_rs_sweep(args, world, rank, local)
        elif mode == "dist":
            run_dist(args, world, rank, local)
        else:
            run_ours(args, world, rank, local)
    finally:
        import torch.distributed as dist
        if dist.is_available() and dist.is_initialized():
            dist.destroy_process_group()


if __name__ == "__main__":
    main()
