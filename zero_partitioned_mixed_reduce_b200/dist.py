"""ZeRO across GPUs: one process per GPU, rank o owns shard o.

Each rank's full gradient buffer and half parameter shards are shared with
its peers through CUDA IPC (zero_ipc_export / zero_ipc_open: the handles
travel in one all_gather_object), so every rank reads every other rank's
buffers with plain loads over NVLink: a plain peer mapping, with no NVLink
multicast object and no allocator of its own. A step is:

  1. a one-element all-reduce on the compute stream, so that every rank's
     gradients are written before any rank reads them;
  2. zero_step_shard_ex on the rank's own shard, reading the R gradient
     buffers through the peer pointers -- the reduce-scatter is the fused
     kernel's own loads, summed in fp32 in rank order, so no half-precision
     partial sum ever leaves a GPU;
  3. an all-reduce (sum) of the two totals {sum g^2, overflow}, which also
     orders every rank's kernel before anyone overwrites its gradients;
  4. zero_step_commit, the same skip / loss-scale decision on every rank.

With global-norm clipping, a norm pass over the rank's shard (again through
the peer pointers) and a one-double all-reduce come before step 2. Built
with norm_divisor=k, the reduce-scatters of the two-pass form also take the
rank's share of that norm (unscaled by the divisor k), and a clipped
step_accumulated with divisor k sums the shares instead of reading the
accumulator again.

Gradient accumulation uses the two-pass form: after each micro-batch,
reduce_scatter() sums the rank's shard of every replica into its local fp32
accumulator (zero_reduce_scatter_shard, between two one-element
all-reduces that order the peers' writes and reads), and
step_accumulated() steps from it.

Overlap with backward: grads_ready(first, count) reports tensors whose
gradients the compute stream has written. When a bucket is complete, a
one-element all-reduce (which every rank reaches only after writing that
bucket) and the bucket's sharded reduce-scatter are queued on a
high-priority communication stream, so the reduction runs while backward
continues; join() ends the micro-batch with one more all-reduce, after which
no peer still reads this rank's gradients, and makes the compute stream wait
for the communication stream. Every rank reports the same tensors in the
same order, so the ranks issue the same collectives in the same order.

ZeRO-3 layer gathers read the peers' parameter shards the same way. Built
with push_params=True (ZeRO-1/2: every rank keeps the whole model), each
rank's step also stores its updated parameters into every rank's full-model
buffer over the same peer mappings (ZERO_STEP_PUSH_PARAMS): the all-gather
of the parameters leaves with the step's own stores, and after the commit
full_params() holds the whole updated model on every rank.
Every method takes an optional stream (a torch.cuda.Stream or a raw
handle; default the current stream). Its kernels and its collectives run in
that stream's order: the collectives are issued with it as the current
stream, so a launch never overtakes the all-reduce that orders it.
Argument marshalling only; the arithmetic runs in libzero_b200.so. The
loads from peer memory are plain loads or bulk copies without multicast.
"""
import torch
import torch.distributed as dist

from . import _capi as Z
from .state import HALF, Plan


def _resolve(stream):
    """The torch stream a call runs on: the given one (a raw handle is
    wrapped), else the current stream."""
    if stream is None:
        return torch.cuda.current_stream()
    if isinstance(stream, int):
        return torch.cuda.ExternalStream(stream)
    return stream


class DistributedZero:
    def __init__(self, numels, layer_ids=None, dtype=Z.ZERO_BF16, mode=Z.ZERO_SCALE_NONE,
                 init_scale=1.0, growth_interval=1000, tensor_align=8, bucket_elems=0, group=None,
                 accumulate=False, norm_divisor=None, push_params=False):
        self.group = group or dist.group.WORLD
        self._opened = []  # peers' IPC handles this rank has mapped
        self.world = dist.get_world_size(self.group)
        self.rank = dist.get_rank(self.group)
        self.plan = Plan(numels, layer_ids, self.world, dtype, tensor_align, bucket_elems)
        dev = torch.device("cuda", torch.cuda.current_device())
        T, S, R = self.plan.T, self.plan.S, self.world
        half = HALF[dtype]
        self.dtype, self.mode = dtype, mode
        # this rank's full gradient buffer, readable by every rank
        self.grads = torch.zeros(T, dtype=half, device=dev)
        self.grad_ptrs = self._share(self.grads)
        sets = 2 if mode == Z.ZERO_SCALE_DYNAMIC else 1
        self.sets = sets
        self.master = [torch.zeros(S, dtype=torch.float32, device=dev) for _ in range(sets)]
        self.m = [torch.zeros(S, dtype=torch.float32, device=dev) for _ in range(sets)]
        self.v = [torch.zeros(S, dtype=torch.float32, device=dev) for _ in range(sets)]
        self.param = [torch.zeros(S, dtype=half, device=dev) for _ in range(sets)]
        self.param_ptrs = [self._share(p) for p in self.param]

        def own(x):  # pointer list with only this rank's shard filled in
            return [x.data_ptr() if r == self.rank else None for r in range(R)]
        # the two-pass form keeps this rank's fp32 accumulator
        self.acc = torch.zeros(S, dtype=torch.float32, device=dev) if accumulate else None
        self.acc_list = [self.acc if r == self.rank else None for r in range(R)] if accumulate else None
        self.handle = Z.StateHandle([dict(master=own(self.master[k]), m=own(self.m[k]),
                                          v=own(self.v[k]), param=own(self.param[k]))
                                     for k in range(sets)], self.acc_list)
        self.micro = 0
        self.comm = None
        self.gather_handle = Z.StateHandle([dict(master=[None] * R, m=[None] * R, v=[None] * R,
                                                 param=self.param_ptrs[k]) for k in range(sets)])
        self.ctx = Z.zero_ctx_create(self.plan.handle, mode, init_scale, growth_interval)
        # norm_divisor: the reduce-scatters also take this rank's share of the
        # clipping norm, unscaled by this gradient divisor, so that a clipped
        # step_accumulated with the same divisor reads no accumulator first
        self.norm_divisor = norm_divisor
        if norm_divisor is not None:
            Z.zero_ctx_set_grad_divisor(self.ctx, float(norm_divisor))
        # push_params: every rank's full-model parameter buffer, one per state
        # set, written by every rank's step
        self.push = bool(push_params)
        if self.push:
            self.full = [torch.zeros(T, dtype=half, device=dev) for _ in range(sets)]
            self.full_ptrs = [self._share(f) for f in self.full]
            Z.zero_ctx_set_param_push(self.ctx, self.full_ptrs[0], self.full_ptrs[1] if sets == 2 else None)
        self.partial = torch.zeros(2, dtype=torch.float64, device=dev)
        self.norm = torch.zeros(2, dtype=torch.float64, device=dev)
        self.token = torch.zeros(1, dtype=torch.float32, device=dev)

    def _share(self, t):
        """Every rank's device address of its own tensor `t` (one per rank, the
        same shape everywhere): this rank's pointer, and the peers' buffers
        mapped through CUDA IPC. The tensors stay alive until close()."""
        torch.cuda.synchronize()  # t is allocated and initialized before a peer maps it
        if self.world == 1:
            return [t.data_ptr()]
        blobs = [None] * self.world
        dist.all_gather_object(blobs, Z.zero_ipc_export(t), group=self.group)
        ptrs = []
        for r in range(self.world):
            if r == self.rank:
                ptrs.append(t.data_ptr())
            else:
                ptrs.append(Z.zero_ipc_open(blobs[r]))
                self._opened.append(blobs[r])
        return ptrs

    def load(self, master_padded, param_padded):
        """Initialize this rank's shard from padded flat master (fp32) and param
        (half) buffers of length T; m = v = 0."""
        S, o = self.plan.S, self.rank
        for k in range(self.sets):
            self.master[k].copy_(master_padded[o * S:(o + 1) * S])
            self.param[k].copy_(param_padded[o * S:(o + 1) * S])
            self.m[k].zero_()
            self.v[k].zero_()
        torch.cuda.synchronize()
        dist.barrier(self.group)

    def _global_norm(self, grads, acc, divisor, stream):
        # stream is the current stream here (the callers' context)
        Z.zero_grad_norm_shard(self.ctx, grads, acc, self.rank, self.rank + 1, self.norm, divisor,
                               stream)
        dist.all_reduce(self.norm, group=self.group)

    def step(self, hp, max_grad_norm=0.0, grad_divisor=None, stream=None):
        """One fused ZeRO step; the gradients of every rank must be in
        self.grads. max_grad_norm > 0 clips to that global norm. After
        reduce_scatter() of earlier micro-batches, self.grads holds the last
        one: it is added to the accumulator inside the fused step
        (ZERO_STEP_ADD_ACC), or, with clipping, reduce-scattered first.
        grad_divisor defaults to the number of micro-batches."""
        stream = _resolve(stream)
        if self.micro > 0 and max_grad_norm > 0:
            self.reduce_scatter(stream)
            self.step_accumulated(hp, grad_divisor, max_grad_norm, stream)
            return
        k = float(self.micro + 1) if grad_divisor is None else grad_divisor
        flags = (Z.ZERO_STEP_ADD_ACC if self.micro > 0 else 0) | self._push_flag()
        with torch.cuda.stream(stream):
            dist.all_reduce(self.token, group=self.group)
            if max_grad_norm > 0:
                self._global_norm(self.grad_ptrs, None, k, stream)
            Z.zero_step_shard_ex(self.ctx, hp, self.handle, self.grad_ptrs, self.rank, self.rank + 1,
                                 self.partial, k, max_grad_norm, self.norm, stream, flags=flags)
            dist.all_reduce(self.partial, group=self.group)
            Z.zero_step_commit(self.ctx, self.partial, stream)
        self.micro = 0

    def _push_flag(self):
        return Z.ZERO_STEP_PUSH_PARAMS if self.push else 0

    def full_params(self):
        """With push_params: this rank's copy of the whole updated model (the
        current set), in the plan's flat layout."""
        assert self.push, "construct with push_params=True"
        k = self.loss_scale()["cur"] if self.sets == 2 else 0
        return self.full[k]

    def _rs_flags(self):
        # every micro-batch takes its norm share: the last one leaves the share
        # of the final accumulator
        return ((Z.ZERO_RS_ACCUMULATE if self.micro else 0) |
                (Z.ZERO_RS_NORM if self.norm_divisor is not None else 0))

    def reduce_scatter(self, stream=None):
        """After a micro-batch's backward wrote self.grads on every rank: add
        this rank's shard of the reduced gradients to its accumulator (the
        first micro-batch of a step overwrites it)."""
        assert self.acc is not None, "construct with accumulate=True"
        stream = _resolve(stream)
        with torch.cuda.stream(stream):
            dist.all_reduce(self.token, group=self.group)  # every replica is written
            Z.zero_reduce_scatter_shard(self.ctx, -1, self.grad_ptrs, self.acc_list, self.rank, self.rank + 1,
                                        self._rs_flags(), stream)
            dist.all_reduce(self.token, group=self.group)  # every peer has read this rank's replica
        self.micro += 1

    def grads_ready(self, first, count=1):
        """Tensors first .. first+count-1 of this micro-batch have their
        gradients written in self.grads (by work on the current stream)."""
        assert self.acc is not None, "construct with accumulate=True"
        if self.comm is None:
            self.comm = torch.cuda.Stream(priority=-1)
            self.bucket_size = [0] * len(self.plan.buckets)
            for b in self.plan.tensor_bucket:
                self.bucket_size[b] += 1
            self.bucket_seen = [0] * len(self.plan.buckets)
            self.comm_token = torch.zeros(1, dtype=torch.float32, device=self.token.device)
        compute = torch.cuda.current_stream()
        done = []
        for k in range(first, first + count):
            b = self.plan.tensor_bucket[k]
            self.bucket_seen[b] += 1
            if self.bucket_seen[b] == self.bucket_size[b]:
                done.append(b)
        if not done:
            return
        ready = torch.cuda.Event()
        ready.record(compute)
        # one token all-reduce per run of consecutive buckets this call
        # completes (every rank reports alike, so the runs match across ranks)
        done.sort()
        runs, i = [], 0
        while i < len(done):
            j = i + 1
            while j < len(done) and done[j] == done[j - 1] + 1:
                j += 1
            runs.append(done[i:j])
            i = j
        with torch.cuda.stream(self.comm):
            self.comm.wait_event(ready)
            for run in runs:
                dist.all_reduce(self.comm_token, group=self.group)  # every rank wrote these buckets
                for b in run:
                    Z.zero_reduce_scatter_shard(self.ctx, b, self.grad_ptrs, self.acc_list, self.rank,
                                                self.rank + 1, self._rs_flags(), self.comm)

    def join(self):
        """End of a micro-batch's backward: every bucket must have been
        reported. The compute stream then waits for the reductions."""
        assert self.comm is not None and all(a == n for a, n in zip(self.bucket_seen, self.bucket_size)), \
            "every tensor must be reported before join()"
        with torch.cuda.stream(self.comm):
            dist.all_reduce(self.comm_token, group=self.group)  # no peer reads this rank's grads any more
        torch.cuda.current_stream().wait_stream(self.comm)
        self.bucket_seen = [0] * len(self.bucket_seen)
        self.micro += 1

    def step_accumulated(self, hp, grad_divisor=None, max_grad_norm=0.0, stream=None):
        """The step from the accumulated micro-batches; grad_divisor defaults
        to their count (the mean)."""
        assert self.micro > 0, "no micro-batch was reduce-scattered"
        k = float(self.micro) if grad_divisor is None else grad_divisor
        stream = _resolve(stream)
        with torch.cuda.stream(stream):
            if max_grad_norm > 0 and self.norm_divisor is not None and float(self.norm_divisor) == k:
                # the reduce-scatters' shares: nothing to read again
                Z.zero_grad_norm_shard(self.ctx, None, None, self.rank, self.rank + 1, self.norm, k, stream)
                dist.all_reduce(self.norm, group=self.group)
            elif max_grad_norm > 0:
                self._global_norm(None, self.acc_list, k, stream)
            Z.zero_step_shard_ex(self.ctx, hp, self.handle, None, self.rank, self.rank + 1, self.partial, k,
                                 max_grad_norm, self.norm, stream, flags=self._push_flag())
            dist.all_reduce(self.partial, group=self.group)
            Z.zero_step_commit(self.ctx, self.partial, stream)
        self.micro = 0

    def gather_layer(self, layer, out, stream=None):
        """ZeRO-3 all-gather of one layer from every rank's parameter shard."""
        Z.zero_gather_layer(self.ctx, layer, self.gather_handle, out, _resolve(stream))

    def gather_layers(self, first, outs, stream=None):
        """ZeRO-3 all-gather of consecutive layers first, first+1, ... in one launch."""
        Z.zero_gather_layers(self.ctx, first, outs, self.gather_handle, _resolve(stream))

    def prefetch_begin(self, bufs, depth, direction=1, stream=None):
        """Start a pass of look-ahead ZeRO-3 gathers into the ring `bufs`
        (the scheduler's communication stream reads every rank's shard);
        then acquire / release each layer in order. The step that produced
        the parameters has been committed on every rank, so their shards
        are final."""
        Z.zero_prefetch_begin(self.ctx, self.gather_handle, bufs, depth, direction, _resolve(stream))

    def layer_acquire(self, layer, stream=None):
        return Z.zero_layer_acquire(self.ctx, layer, _resolve(stream))

    def layer_release(self, layer, stream=None):
        Z.zero_layer_release(self.ctx, layer, _resolve(stream))

    def loss_scale(self):
        return Z.zero_loss_scale(self.ctx)

    def current(self, field):
        """This rank's shard of master / m / v / param in the current set."""
        k = self.loss_scale()["cur"] if self.sets == 2 else 0
        return getattr(self, field)[k]

    def close(self):
        """Release the context and unmap the peers' buffers. Every rank calls
        it; no rank frees its own shared buffers before all have unmapped them
        (the barrier at the end)."""
        if self.ctx:
            torch.cuda.synchronize()
            Z.zero_ctx_destroy(self.ctx)
            self.ctx = None
        if self._opened:
            for blob in self._opened:
                Z.zero_ipc_close(blob)
            self._opened = []
        if self.world > 1:
            dist.barrier(self.group)
