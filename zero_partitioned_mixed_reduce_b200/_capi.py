"""ctypes binding of libzero_b200.so (include/zero_b200.h).

Argument marshalling only: every step of the hot path runs in the library's
CUDA kernels. The functions carry the C names; on a non-OK status they raise
ZeroError with the library's message. Device buffers can be passed as
integers or as any object with a ``data_ptr()`` method (torch tensors).
If the shared library is missing this module raises ImportError: there is
no fallback.
"""
import ctypes as C
import os

_HERE = os.path.dirname(os.path.abspath(__file__))
# ZERO_B200_LIB selects another build of the library (the bounds-checking
# debug build in the tests); by default the in-tree release build
LIB_PATH = os.environ.get("ZERO_B200_LIB") or os.path.join(_HERE, "libzero_b200.so")

ZERO_MAX_RANKS = 64
ZERO_OK, ZERO_ERR_INVALID_ARG, ZERO_ERR_ALIGN, ZERO_ERR_CUDA = 0, 1, 2, 3
ZERO_ERR_OOM, ZERO_ERR_RANGE, ZERO_ERR_TIMEOUT, ZERO_ERR_STATE = 4, 5, 6, 7
ZERO_BF16, ZERO_FP16 = 0, 1
ZERO_SCALE_NONE, ZERO_SCALE_STATIC, ZERO_SCALE_DYNAMIC = 0, 1, 2
ZERO_LOSS_SCALE_GET, ZERO_LOSS_SCALE_SET = 0, 1
ZERO_RS_ACCUMULATE = 1
ZERO_RS_NORM = 2
ZERO_STEP_ADD_ACC = 1
ZERO_STEP_NORM_FROM_RS = 2
ZERO_STEP_PUSH_PARAMS = 4
ZERO_STEP_CLEAN = 8
ZERO_TRACE_REDUCE_SCATTER, ZERO_TRACE_STEP, ZERO_TRACE_GATHER, ZERO_TRACE_NORM, ZERO_TRACE_COMMIT = 1, 2, 3, 4, 5
TRACE_NAMES = {0: "untimed", 1: "reduce_scatter", 2: "step", 3: "gather", 4: "norm", 5: "commit"}


class zero_trace_record(C.Structure):
    _fields_ = [("call", C.c_int32), ("reserved", C.c_int32), ("arg", C.c_int64), ("ms", C.c_float),
                ("reserved2", C.c_float)]

STATUS_NAMES = {0: "ZERO_OK", 1: "ZERO_ERR_INVALID_ARG", 2: "ZERO_ERR_ALIGN", 3: "ZERO_ERR_CUDA",
                4: "ZERO_ERR_OOM", 5: "ZERO_ERR_RANGE", 6: "ZERO_ERR_TIMEOUT", 7: "ZERO_ERR_STATE"}

if not os.path.exists(LIB_PATH):
    raise ImportError(
        f"{LIB_PATH} is missing: build it with `python zero_partitioned_mixed_reduce_b200/build.py` "
        "(nvcc, sm_100a). There is no CPU fallback.")


class ZeroError(RuntimeError):
    def __init__(self, status, message):
        super().__init__(f"{STATUS_NAMES.get(status, status)}: {message}")
        self.status = status


class zero_plan_config(C.Structure):
    _fields_ = [("R", C.c_int32), ("dtype", C.c_int32), ("tensor_align", C.c_int32),
                ("reserved", C.c_int32), ("bucket_elems", C.c_int64)]


class zero_plan_info(C.Structure):
    _fields_ = [("P", C.c_int64), ("L", C.c_int64), ("S", C.c_int64), ("T", C.c_int64),
                ("n_tensors", C.c_int64), ("n_buckets", C.c_int64), ("n_layers", C.c_int64),
                ("R", C.c_int32), ("dtype", C.c_int32), ("tensor_align", C.c_int32),
                ("reserved", C.c_int32)]


class zero_loss_scale_config(C.Structure):
    _fields_ = [("mode", C.c_int32), ("init_scale", C.c_float), ("growth_interval", C.c_int64),
                ("growth_factor", C.c_float), ("backoff_factor", C.c_float),
                ("min_scale", C.c_float), ("reserved", C.c_int32)]


class zero_adamw(C.Structure):
    _fields_ = [("lr", C.c_double), ("beta1", C.c_double), ("beta2", C.c_double),
                ("eps", C.c_double), ("weight_decay", C.c_double)]


_PP = C.POINTER(C.c_void_p)


class zero_state(C.Structure):
    _fields_ = [("master", _PP * 2), ("m", _PP * 2), ("v", _PP * 2), ("param", _PP * 2),
                ("acc", _PP)]


class zero_step_opts(C.Structure):
    _fields_ = [("grad_divisor", C.c_double), ("max_grad_norm", C.c_double), ("flags", C.c_int64),
                ("reserved", C.c_int64)]


class zero_loss_scale_state(C.Structure):
    _fields_ = [("scale", C.c_float), ("cur", C.c_int32), ("good", C.c_int64), ("t", C.c_int64),
                ("last_overflow", C.c_int32), ("last_skipped", C.c_int32),
                ("grad_norm_sq", C.c_double)]


class zero_cpu_decision(C.Structure):
    _fields_ = [("grad_norm_sq", C.c_double), ("inv", C.c_float), ("clip", C.c_float),
                ("overflow", C.c_int32), ("skip", C.c_int32), ("clipping", C.c_int32),
                ("reserved", C.c_int32)]


_lib = C.CDLL(LIB_PATH)
_P = C.c_void_p
_S = C.c_int32  # zero_status


def _sig(name, restype, argtypes):
    f = getattr(_lib, name)
    f.restype = restype
    f.argtypes = argtypes
    return f


_sig("zero_plan", _S, [_P, _P, C.c_int64, C.POINTER(zero_plan_config), C.POINTER(_P)])
_sig("zero_plan_destroy", None, [_P])
_sig("zero_plan_get_info", _S, [_P, C.POINTER(zero_plan_info)])
_sig("zero_plan_tensor", _S, [_P, C.c_int64, C.POINTER(C.c_int64), C.POINTER(C.c_int64),
                              C.POINTER(C.c_int64), C.POINTER(C.c_int64)])
_sig("zero_plan_bucket", _S, [_P, C.c_int64, C.POINTER(C.c_int64), C.POINTER(C.c_int64)])
_sig("zero_plan_layer", _S, [_P, C.c_int64, C.POINTER(C.c_int64), C.POINTER(C.c_int64)])
_sig("zero_plan_memory", _S, [_P, C.c_int32, C.POINTER(C.c_int64)])
_sig("zero_plan_step_tiles", _S, [_P, C.POINTER(C.c_int64), C.POINTER(C.c_int64), C.POINTER(C.c_int64)])


class zero_ipc_handle(C.Structure):
    _fields_ = [("handle", C.c_uint8 * 64), ("offset", C.c_int64), ("alloc_bytes", C.c_int64)]


_sig("zero_ipc_export", _S, [_P, C.POINTER(zero_ipc_handle)])
_sig("zero_ipc_open", _S, [C.POINTER(zero_ipc_handle), C.POINTER(C.c_void_p)])
_sig("zero_ipc_close", _S, [C.POINTER(zero_ipc_handle)])
_sig("zero_ctx_create", _S, [_P, C.POINTER(zero_loss_scale_config), C.POINTER(_P)])
_sig("zero_ctx_destroy", _S, [_P])
_sig("zero_ctx_reserve_steps", _S, [_P, C.c_int64, C.c_double, C.c_double, _P])
_sig("zero_ctx_set_grad_divisor", _S, [_P, C.c_double])
_sig("zero_ctx_set_param_push", _S, [_P, _PP, _PP])
_sig("zero_take_overflow", _S, [_P, _P, _P])
_sig("zero_test_drop_tile", _S, [_P, C.c_int64])
_sig("zero_reduce_scatter_bucket", _S, [_P, C.c_int64, _PP, _PP, _P])
_sig("zero_step", _S, [_P, C.POINTER(zero_adamw), C.POINTER(zero_state), _PP, _P])
_sig("zero_reduce_scatter_bucket_ex", _S, [_P, C.c_int64, _PP, _PP, C.c_int32, _P])
_sig("zero_reduce_scatter_buckets", _S, [_P, C.c_int64, C.c_int64, _PP, _PP, C.c_int32, _P])
_sig("zero_trace_start", _S, [_P, C.c_int32])
_sig("zero_trace_read", _S, [_P, C.POINTER(zero_trace_record), C.c_int32, C.POINTER(C.c_int32),
                             C.POINTER(C.c_int64)])
_sig("zero_trace_stop", _S, [_P])
_sig("zero_step_ex", _S, [_P, C.POINTER(zero_adamw), C.POINTER(zero_state), _PP,
                          C.POINTER(zero_step_opts), _P])
_sig("zero_gather_layer", _S, [_P, C.c_int64, C.POINTER(zero_state), _P, _P])
_sig("zero_gather_layers", _S, [_P, C.c_int64, C.c_int64, C.POINTER(zero_state), _PP, _P])
_sig("zero_loss_scale", _S, [_P, C.POINTER(zero_loss_scale_state), C.c_int32, _P])
_sig("zero_step_noalloc", _S, [_P, C.POINTER(zero_loss_scale_config),
                               C.POINTER(zero_loss_scale_state), C.POINTER(zero_adamw), _PP, _PP,
                               _PP, _PP, _PP, _P])
_sig("zero_grads_ready", _S, [_P, C.c_int64, C.c_int64, _PP, _PP, C.c_int32, _P])
_sig("zero_grads_join", _S, [_P, _P])
_sig("zero_sched_set_comm_sms", _S, [_P, C.c_int32])
_sig("zero_prefetch_begin", _S, [_P, C.POINTER(zero_state), _PP, C.c_int32, C.c_int32, C.c_int32, _P])
_sig("zero_layer_acquire", _S, [_P, C.c_int64, C.POINTER(C.c_void_p), _P])
_sig("zero_layer_release", _S, [_P, C.c_int64, _P])
_sig("zero_cpu_step", _S, [_P, C.POINTER(zero_loss_scale_config), C.POINTER(zero_loss_scale_state),
                           C.POINTER(zero_adamw), C.POINTER(zero_step_opts), _PP, _PP, _PP, _PP, _PP,
                           C.c_int32])
_sig("zero_cpu_scan", _S, [_P, C.POINTER(zero_loss_scale_config), C.POINTER(zero_loss_scale_state),
                           C.POINTER(zero_step_opts), _PP, C.c_int32, C.POINTER(zero_cpu_decision)])
_sig("zero_cpu_update", _S, [_P, C.POINTER(zero_loss_scale_state), C.POINTER(zero_adamw),
                             C.POINTER(zero_cpu_decision), _PP, _PP, _PP, _PP, _PP, C.c_int64, C.c_int64,
                             C.c_int32])
_sig("zero_cpu_scan_shard", _S, [_P, C.POINTER(zero_loss_scale_config), C.POINTER(zero_loss_scale_state),
                                 C.POINTER(zero_step_opts), _PP, C.c_int32, C.c_int32, C.c_int32,
                                 C.POINTER(C.c_double)])
_sig("zero_cpu_decide", _S, [_P, C.POINTER(zero_loss_scale_config), C.POINTER(zero_loss_scale_state),
                             C.POINTER(zero_step_opts), C.POINTER(C.c_double), C.POINTER(zero_cpu_decision)])
_sig("zero_cpu_update_shard", _S, [_P, C.POINTER(zero_loss_scale_state), C.POINTER(zero_adamw),
                                   C.POINTER(zero_cpu_decision), _PP, _PP, _PP, _PP, _PP, C.c_int32, C.c_int32,
                                   C.c_int32])
_sig("zero_cpu_commit", _S, [C.POINTER(zero_loss_scale_config), C.POINTER(zero_loss_scale_state),
                             C.POINTER(zero_cpu_decision)])
_sig("zero_step_shard", _S, [_P, C.POINTER(zero_adamw), C.POINTER(zero_state), _PP, C.c_int32,
                             C.c_int32, _P, _P])
_sig("zero_step_commit", _S, [_P, _P, _P])
_sig("zero_step_shard_ex", _S, [_P, C.POINTER(zero_adamw), C.POINTER(zero_state), _PP, C.c_int32,
                                C.c_int32, C.POINTER(zero_step_opts), _P, _P, _P])
_sig("zero_reduce_scatter_shard", _S, [_P, C.c_int64, _PP, _PP, C.c_int32, C.c_int32, C.c_int32, _P])
_sig("zero_grad_norm_shard", _S, [_P, _PP, _PP, C.c_double, C.c_int32, C.c_int32, _P, _P])
_sig("zero_sync", _S, [_P, _P])
_sig("zero_debug_bounds", _S, [C.POINTER(C.c_int64), C.POINTER(C.c_int64), C.POINTER(C.c_int64),
                               C.c_int32])
_sig("zero_last_error", C.c_size_t, [C.c_char_p, C.c_size_t])
_sig("zero_version", C.c_char_p, [])


def _check(status):
    if status != ZERO_OK:
        buf = C.create_string_buffer(1024)
        _lib.zero_last_error(buf, 1024)
        raise ZeroError(status, buf.value.decode(errors="replace"))


def _addr(x):
    if x is None:
        return None
    if isinstance(x, int):
        return x
    return int(x.data_ptr())


def _ptr_array(xs):
    """R device pointers -> C array (kept alive by the caller)."""
    if xs is None:
        return None
    arr = (C.c_void_p * len(xs))(*[_addr(x) for x in xs])
    return C.cast(arr, _PP), arr


def _stream(s):
    if s is None:
        return None
    if isinstance(s, int):
        return s
    return int(s.cuda_stream)  # torch.cuda.Stream


# ---- plan ------------------------------------------------------------------

def zero_plan(numels, layer_ids=None, R=1, dtype=ZERO_BF16, tensor_align=8, bucket_elems=0):
    """Returns an opaque plan handle (int). Free with zero_plan_destroy."""
    import numpy as np
    n = len(numels)
    nb = np.ascontiguousarray(numels if n else [0], dtype=np.int64)
    lid = None if layer_ids is None else np.ascontiguousarray(layer_ids if n else [0], dtype=np.int32)
    cfg = zero_plan_config(R, dtype, tensor_align, 0, bucket_elems)
    out = C.c_void_p()
    _check(_lib.zero_plan(nb.ctypes.data, None if lid is None else lid.ctypes.data, n, C.byref(cfg),
                          C.byref(out)))
    return out.value


def zero_plan_destroy(plan):
    _lib.zero_plan_destroy(plan)


def zero_plan_get_info(plan):
    info = zero_plan_info()
    _check(_lib.zero_plan_get_info(plan, C.byref(info)))
    return {k: getattr(info, k) for k, _ in zero_plan_info._fields_ if k != "reserved"}


def zero_plan_tensor(plan, k):
    off, num, b, l = C.c_int64(), C.c_int64(), C.c_int64(), C.c_int64()
    _check(_lib.zero_plan_tensor(plan, k, C.byref(off), C.byref(num), C.byref(b), C.byref(l)))
    return off.value, num.value, b.value, l.value


def zero_plan_bucket(plan, b):
    lo, hi = C.c_int64(), C.c_int64()
    _check(_lib.zero_plan_bucket(plan, b, C.byref(lo), C.byref(hi)))
    return lo.value, hi.value


def zero_plan_layer(plan, l):
    lo, hi = C.c_int64(), C.c_int64()
    _check(_lib.zero_plan_layer(plan, l, C.byref(lo), C.byref(hi)))
    return lo.value, hi.value


def zero_plan_memory(plan, stage):
    b = C.c_int64()
    _check(_lib.zero_plan_memory(plan, stage, C.byref(b)))
    return b.value


def zero_ipc_export(ptr):
    """The IPC description (bytes) of the device buffer at ptr, for the job's
    other processes."""
    h = zero_ipc_handle()
    _check(_lib.zero_ipc_export(_addr(ptr), C.byref(h)))
    return C.string_at(C.addressof(h), C.sizeof(h))


def zero_ipc_open(blob):
    """Map a buffer another process exported; returns its device address here."""
    h = zero_ipc_handle.from_buffer_copy(blob)
    p = C.c_void_p()
    _check(_lib.zero_ipc_open(C.byref(h), C.byref(p)))
    return p.value


def zero_ipc_close(blob):
    h = zero_ipc_handle.from_buffer_copy(blob)
    _check(_lib.zero_ipc_close(C.byref(h)))


def zero_plan_step_tiles(plan):
    """(tile_elems, tiles_per_shard, tiles_total) of the staged fused step."""
    e, t, n = C.c_int64(), C.c_int64(), C.c_int64()
    _check(_lib.zero_plan_step_tiles(plan, C.byref(e), C.byref(t), C.byref(n)))
    return e.value, t.value, n.value


# ---- context ---------------------------------------------------------------

def zero_ctx_create(plan, mode=ZERO_SCALE_NONE, init_scale=1.0, growth_interval=1000,
                    growth_factor=2.0, backoff_factor=0.5, min_scale=1.0):
    cfg = zero_loss_scale_config(mode, init_scale, growth_interval, growth_factor,
                                 backoff_factor, min_scale, 0)
    out = C.c_void_p()
    _check(_lib.zero_ctx_create(plan, C.byref(cfg), C.byref(out)))
    return out.value


def zero_ctx_destroy(ctx):
    _check(_lib.zero_ctx_destroy(ctx))


def zero_ctx_reserve_steps(ctx, steps, beta1=0.9, beta2=0.999, stream=None):
    _check(_lib.zero_ctx_reserve_steps(ctx, steps, beta1, beta2, _stream(stream)))


def zero_sched_set_comm_sms(ctx, sms):
    _check(_lib.zero_sched_set_comm_sms(ctx, sms))


def zero_test_drop_tile(ctx, tile):
    _check(_lib.zero_test_drop_tile(ctx, tile))


class StateHandle:
    """A zero_state built from R-long lists of device buffers per field.

    sets: list of one or two dicts with keys master, m, v, param; acc: list or
    None. Keeps the pointer arrays alive as long as the handle lives."""

    def __init__(self, sets, acc=None):
        self._keep = []
        self.c = zero_state()
        for k, d in enumerate(sets):
            for field in ("master", "m", "v", "param"):
                p, arr = _ptr_array(d[field])
                self._keep.append(arr)
                getattr(self.c, field)[k] = p
        if acc is not None:
            p, arr = _ptr_array(acc)
            self._keep.append(arr)
            self.c.acc = p


def zero_reduce_scatter_bucket(ctx, bucket, grads, acc, stream=None):
    g, ga = _ptr_array(grads)
    a, aa = _ptr_array(acc)
    _check(_lib.zero_reduce_scatter_bucket(ctx, bucket, g, a, _stream(stream)))


def zero_reduce_scatter_buckets(ctx, first, count, grads, acc, flags=0, stream=None):
    """Buckets first .. first+count-1 (a contiguous flat range) in one launch."""
    g, ga = _ptr_array(grads)
    a, aa = _ptr_array(acc)
    _check(_lib.zero_reduce_scatter_buckets(ctx, first, count, g, a, flags, _stream(stream)))


def zero_trace_start(ctx, capacity=4096):
    _check(_lib.zero_trace_start(ctx, capacity))


def zero_trace_read(ctx, max_records=4096):
    """The traced calls since the last read: (list of (name, arg, ms), dropped)."""
    buf = (zero_trace_record * max_records)()
    n, dropped = C.c_int32(0), C.c_int64(0)
    _check(_lib.zero_trace_read(ctx, buf, max_records, C.byref(n), C.byref(dropped)))
    return [(TRACE_NAMES.get(buf[i].call, str(buf[i].call)), int(buf[i].arg), float(buf[i].ms))
            for i in range(n.value)], int(dropped.value)


def zero_trace_stop(ctx):
    _check(_lib.zero_trace_stop(ctx))


def zero_ctx_set_grad_divisor(ctx, grad_divisor):
    """The divisor that ZERO_RS_NORM reduce-scatters unscale by."""
    _check(_lib.zero_ctx_set_grad_divisor(ctx, float(grad_divisor)))


def zero_take_overflow(ctx, flag, stream=None):
    """The reduce-scatters' overflow flag (0/1) into the device int32 `flag`,
    and the flag cleared (asynchronous on the stream)."""
    _check(_lib.zero_take_overflow(ctx, _addr(flag), _stream(stream)))


def zero_ctx_set_param_push(ctx, full0, full1=None):
    """Register every rank's full-model parameter buffer of state set 0
    (full0) and set 1 (full1) for steps with ZERO_STEP_PUSH_PARAMS; full0 None
    clears the registration."""
    a = _ptr_array(full0)
    b = _ptr_array(full1)
    _check(_lib.zero_ctx_set_param_push(ctx, a[0] if a else None, b[0] if b else None))


def zero_reduce_scatter_bucket_ex(ctx, bucket, grads, acc, flags=0, stream=None):
    """flags: ZERO_RS_ACCUMULATE adds to the accumulators; ZERO_RS_NORM also
    records the bucket's share of the clipping norm."""
    g, ga = _ptr_array(grads)
    a, aa = _ptr_array(acc)
    _check(_lib.zero_reduce_scatter_bucket_ex(ctx, bucket, g, a, flags, _stream(stream)))


def zero_step(ctx, hp, state: StateHandle, grads=None, stream=None):
    """hp: zero_adamw or a dict with lr, beta1, beta2, eps, weight_decay."""
    if isinstance(hp, dict):
        hp = zero_adamw(hp["lr"], hp["beta1"], hp["beta2"], hp["eps"], hp["weight_decay"])
    g = None
    if grads is not None:
        g, ga = _ptr_array(grads)
    _check(_lib.zero_step(ctx, C.byref(hp), C.byref(state.c), g, _stream(stream)))


def zero_step_ex(ctx, hp, state: StateHandle, grads=None, grad_divisor=1.0, max_grad_norm=0.0,
                 stream=None, flags=0):
    """zero_step with a grad divisor, global-norm clipping and flags
    (ZERO_STEP_ADD_ACC: the fused step adds state's accumulators;
    ZERO_STEP_NORM_FROM_RS: the clipping norm from the reduce-scatters' shares;
    ZERO_STEP_PUSH_PARAMS: the step also writes every rank's registered
    full-model parameter buffer)."""
    if isinstance(hp, dict):
        hp = zero_adamw(hp["lr"], hp["beta1"], hp["beta2"], hp["eps"], hp["weight_decay"])
    g = None
    if grads is not None:
        g, ga = _ptr_array(grads)
    opts = zero_step_opts(grad_divisor, max_grad_norm, flags)
    _check(_lib.zero_step_ex(ctx, C.byref(hp), C.byref(state.c), g, C.byref(opts),
                             _stream(stream)))


def zero_gather_layer(ctx, layer, state: StateHandle, out, stream=None):
    _check(_lib.zero_gather_layer(ctx, layer, C.byref(state.c), _addr(out), _stream(stream)))


ZERO_GATHER_MAX_LAYERS = 64


def zero_gather_layers(ctx, first, outs, state: StateHandle, stream=None):
    """Gather layers first .. first+len(outs)-1, layer first+i into outs[i]."""
    o, oa = _ptr_array(outs)
    _check(_lib.zero_gather_layers(ctx, first, len(outs), C.byref(state.c), o, _stream(stream)))


def zero_loss_scale(ctx, op=ZERO_LOSS_SCALE_GET, state=None, stream=None):
    """GET returns a dict; SET takes a dict (or zero_loss_scale_state)."""
    st = zero_loss_scale_state()
    if op == ZERO_LOSS_SCALE_SET:
        if isinstance(state, dict):
            for k, _ in zero_loss_scale_state._fields_:
                if k in state:
                    setattr(st, k, state[k])
        else:
            st = state
    _check(_lib.zero_loss_scale(ctx, C.byref(st), op, _stream(stream)))
    return {k: getattr(st, k) for k, _ in zero_loss_scale_state._fields_}


ZERO_NOALLOC_MAX_ELEMS = 4194304


def zero_step_noalloc(plan, cfg, state, hp, grads, master, m, v, param, stream=None):
    """The two-pass step without any device allocation (see the header).

    cfg: dict with mode, growth_interval, growth_factor, backoff_factor,
    min_scale (init_scale is ignored: the scale comes from `state`). state:
    dict with scale, cur (0), good, t (and optionally the last_* fields).
    Returns the loss-scale state after the step. Synchronizes `stream`."""
    c = zero_loss_scale_config(cfg.get("mode", ZERO_SCALE_NONE), 1.0,
                               cfg.get("growth_interval", 1000), cfg.get("growth_factor", 2.0),
                               cfg.get("backoff_factor", 0.5), cfg.get("min_scale", 1.0), 0)
    st = zero_loss_scale_state()
    for k, _ in zero_loss_scale_state._fields_:
        if k in state:
            setattr(st, k, state[k])
    if isinstance(hp, dict):
        hp = zero_adamw(hp["lr"], hp["beta1"], hp["beta2"], hp["eps"], hp["weight_decay"])
    arrays = [_ptr_array(x) for x in (grads, master, m, v, param)]
    _check(_lib.zero_step_noalloc(plan, C.byref(c), C.byref(st), C.byref(hp),
                                  *[a[0] for a in arrays], _stream(stream)))
    return {k: getattr(st, k) for k, _ in zero_loss_scale_state._fields_}


def zero_grads_ready(ctx, first, count, grads, acc, flags=0, stream=None):
    g, ga = _ptr_array(grads)
    a, aa = _ptr_array(acc)
    _check(_lib.zero_grads_ready(ctx, first, count, g, a, flags, _stream(stream)))


def zero_grads_join(ctx, stream=None):
    _check(_lib.zero_grads_join(ctx, _stream(stream)))


def zero_prefetch_begin(ctx, state: StateHandle, bufs, depth, direction=1, stream=None):
    b, ba = _ptr_array(bufs)
    _check(_lib.zero_prefetch_begin(ctx, C.byref(state.c), b, len(bufs), depth, direction,
                                    _stream(stream)))


def zero_layer_acquire(ctx, layer, stream=None):
    """Returns the device address of the buffer holding `layer`."""
    out = C.c_void_p()
    _check(_lib.zero_layer_acquire(ctx, layer, C.byref(out), _stream(stream)))
    return out.value


def zero_layer_release(ctx, layer, stream=None):
    _check(_lib.zero_layer_release(ctx, layer, _stream(stream)))


def _cpu_cfg(cfg):
    return zero_loss_scale_config(cfg.get("mode", ZERO_SCALE_NONE), 1.0,
                                  cfg.get("growth_interval", 1000), cfg.get("growth_factor", 2.0),
                                  cfg.get("backoff_factor", 0.5), cfg.get("min_scale", 1.0), 0)


def _cpu_state(state):
    st = zero_loss_scale_state()
    for k, _ in zero_loss_scale_state._fields_:
        if k in state:
            setattr(st, k, state[k])
    return st


def _cpu_hp(hp):
    if isinstance(hp, dict):
        return zero_adamw(hp["lr"], hp["beta1"], hp["beta2"], hp["eps"], hp["weight_decay"])
    return hp


def zero_cpu_step(plan, cfg, state, hp, acc, master, m, v, param, grad_divisor=1.0,
                  max_grad_norm=0.0, nthreads=0, flags=0):
    """The optimizer step on host memory (all buffers host pointers, numpy
    arrays or CPU tensors). cfg / state as for zero_step_noalloc; returns the
    loss-scale state after the step. flags: ZERO_STEP_CLEAN (no accumulator is
    inf or NaN, as zero_take_overflow reported) lets a DYNAMIC step run in one pass."""
    c, st, hp = _cpu_cfg(cfg), _cpu_state(state), _cpu_hp(hp)
    opts = zero_step_opts(grad_divisor, max_grad_norm, flags)
    arrays = [_ptr_array([_host_addr(x) for x in xs]) for xs in (acc, master, m, v, param)]
    _check(_lib.zero_cpu_step(plan, C.byref(c), C.byref(st), C.byref(hp), C.byref(opts),
                              *[a[0] for a in arrays], nthreads))
    return {k: getattr(st, k) for k, _ in zero_loss_scale_state._fields_}


def zero_cpu_scan(plan, cfg, state, acc, grad_divisor=1.0, max_grad_norm=0.0, nthreads=0):
    """The global part of the CPU step; returns a zero_cpu_decision."""
    c, st = _cpu_cfg(cfg), _cpu_state(state)
    opts = zero_step_opts(grad_divisor, max_grad_norm)
    a = _ptr_array([_host_addr(x) for x in acc])
    d = zero_cpu_decision()
    _check(_lib.zero_cpu_scan(plan, C.byref(c), C.byref(st), C.byref(opts), a[0], nthreads, C.byref(d)))
    return d


def zero_cpu_update(plan, state, hp, decision, acc, master, m, v, param, lo, hi, nthreads=0):
    """Update elements [lo, hi) of every shard from a zero_cpu_scan decision."""
    st, hp = _cpu_state(state), _cpu_hp(hp)
    arrays = [_ptr_array([_host_addr(x) for x in xs]) for xs in (acc, master, m, v, param)]
    _check(_lib.zero_cpu_update(plan, C.byref(st), C.byref(hp), C.byref(decision),
                                *[a[0] for a in arrays], lo, hi, nthreads))


def zero_cpu_scan_shard(plan, cfg, state, acc, owner_lo, owner_hi, grad_divisor=1.0, max_grad_norm=0.0,
                        nthreads=0):
    """Owners [lo, hi)'s part of the CPU scan: (sum of unscaled g^2, overflow 0/1)."""
    c, st = _cpu_cfg(cfg), _cpu_state(state)
    opts = zero_step_opts(grad_divisor, max_grad_norm)
    a = _ptr_array([_host_addr(x) for x in acc])
    part = (C.c_double * 2)()
    _check(_lib.zero_cpu_scan_shard(plan, C.byref(c), C.byref(st), C.byref(opts), a[0], owner_lo, owner_hi,
                                    nthreads, part))
    return float(part[0]), float(part[1])


def zero_cpu_decide(plan, cfg, state, reduced, grad_divisor=1.0, max_grad_norm=0.0):
    """The decision from all-reduced (norm sum, overflow count)."""
    c, st = _cpu_cfg(cfg), _cpu_state(state)
    opts = zero_step_opts(grad_divisor, max_grad_norm)
    red = (C.c_double * 2)(float(reduced[0]), float(reduced[1]))
    d = zero_cpu_decision()
    _check(_lib.zero_cpu_decide(plan, C.byref(c), C.byref(st), C.byref(opts), red, C.byref(d)))
    return d


def zero_cpu_update_shard(plan, state, hp, decision, acc, master, m, v, param, owner_lo, owner_hi, nthreads=0):
    """Update every element of shards [owner_lo, owner_hi) (the others' pointers may be None)."""
    st, hp = _cpu_state(state), _cpu_hp(hp)
    arrays = [_ptr_array([_host_addr(x) for x in xs]) for xs in (acc, master, m, v, param)]
    _check(_lib.zero_cpu_update_shard(plan, C.byref(st), C.byref(hp), C.byref(decision),
                                      *[a[0] for a in arrays], owner_lo, owner_hi, nthreads))


def zero_cpu_commit(cfg, state, decision):
    """The loss-scale state after the step (a dict)."""
    c, st = _cpu_cfg(cfg), _cpu_state(state)
    _check(_lib.zero_cpu_commit(C.byref(c), C.byref(st), C.byref(decision)))
    return {k: getattr(st, k) for k, _ in zero_loss_scale_state._fields_}


def _host_addr(x):
    if x is None:
        return 0
    if isinstance(x, int):
        return x
    if hasattr(x, "ctypes"):  # numpy
        assert x.flags["C_CONTIGUOUS"]
        return x.ctypes.data
    return int(x.data_ptr())


def zero_step_shard(ctx, hp, state: StateHandle, grads, owner_lo, owner_hi, partial, stream=None):
    """Fused step on shards [owner_lo, owner_hi); partial: device buffer of 2 float64."""
    if isinstance(hp, dict):
        hp = zero_adamw(hp["lr"], hp["beta1"], hp["beta2"], hp["eps"], hp["weight_decay"])
    g, ga = _ptr_array(grads)
    _check(_lib.zero_step_shard(ctx, C.byref(hp), C.byref(state.c), g, owner_lo, owner_hi,
                                _addr(partial), _stream(stream)))


def zero_step_shard_ex(ctx, hp, state: StateHandle, grads, owner_lo, owner_hi, partial,
                       grad_divisor=1.0, max_grad_norm=0.0, global_norm_sq=None, stream=None, flags=0):
    """Sharded step with options; grads=None steps from state's accumulators.
    global_norm_sq: device float64 holding the cross-rank norm (clipping)."""
    if isinstance(hp, dict):
        hp = zero_adamw(hp["lr"], hp["beta1"], hp["beta2"], hp["eps"], hp["weight_decay"])
    g = _ptr_array(grads)
    opts = zero_step_opts(grad_divisor, max_grad_norm, flags)
    _check(_lib.zero_step_shard_ex(ctx, C.byref(hp), C.byref(state.c), g[0] if g else None, owner_lo,
                                   owner_hi, C.byref(opts), _addr(global_norm_sq), _addr(partial),
                                   _stream(stream)))


def zero_reduce_scatter_shard(ctx, bucket, grads, acc, owner_lo, owner_hi, flags=0, stream=None):
    """Bucket `bucket` (-1: all) reduce-scattered into the owners [lo, hi)'s accumulators."""
    g, ga = _ptr_array(grads)
    a, aa = _ptr_array(acc)
    _check(_lib.zero_reduce_scatter_shard(ctx, bucket, g, a, owner_lo, owner_hi, flags, _stream(stream)))


def zero_grad_norm_shard(ctx, grads, acc, owner_lo, owner_hi, partial, grad_divisor=1.0, stream=None):
    """Owners [lo, hi)'s sum of unscaled g^2 into partial[0] (from grads, from
    acc, or with both None from the reduce-scatters' ZERO_RS_NORM shares)."""
    g = _ptr_array(grads)
    a = _ptr_array(acc)
    _check(_lib.zero_grad_norm_shard(ctx, g[0] if g else None, a[0] if a else None, grad_divisor,
                                     owner_lo, owner_hi, _addr(partial), _stream(stream)))


def zero_step_commit(ctx, reduced, stream=None):
    """Loss-scale update from reduced totals (device buffer of 2 float64)."""
    _check(_lib.zero_step_commit(ctx, _addr(reduced), _stream(stream)))


def zero_debug_bounds(reset=False):
    """(count, first_site, first_index) of the out-of-range accesses the
    debug build's kernels skipped; count is -1 in the release build."""
    n, site, idx = C.c_int64(), C.c_int64(), C.c_int64()
    _check(_lib.zero_debug_bounds(C.byref(n), C.byref(site), C.byref(idx), 1 if reset else 0))
    return n.value, site.value, idx.value


def zero_sync(ctx, stream=None):
    _check(_lib.zero_sync(ctx, _stream(stream)))


def zero_last_error():
    buf = C.create_string_buffer(1024)
    _lib.zero_last_error(buf, 1024)
    return buf.value.decode(errors="replace")


def zero_version():
    return _lib.zero_version().decode()
