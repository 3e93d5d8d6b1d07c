"""TEST INFRASTRUCTURE: ctypes binding of the plain CPU oracle (zero_oracle.c).

Only tests/, __graft_entry__.smoke() and bench.py's CPU-baseline / reference
legs may import this package. The CUDA library never imports it and shares
no code with it.
"""
import ctypes as C
import os

import numpy as np

from . import build as _build

BF16, FP16 = 0, 1
SCALE_NONE, SCALE_STATIC, SCALE_DYNAMIC = 0, 1, 2

_lib = None


class AdamW(C.Structure):
    _fields_ = [("lr", C.c_double), ("beta1", C.c_double), ("beta2", C.c_double),
                ("eps", C.c_double), ("weight_decay", C.c_double)]


class FSM(C.Structure):
    _fields_ = [("mode", C.c_int32), ("scale", C.c_float), ("growth_interval", C.c_int64),
                ("growth_factor", C.c_float), ("backoff_factor", C.c_float),
                ("min_scale", C.c_float), ("good", C.c_int64), ("t", C.c_int64),
                ("last_overflow", C.c_int32), ("last_skipped", C.c_int32),
                ("grad_norm_sq", C.c_double)]


class StepOpts(C.Structure):
    _fields_ = [("grad_divisor", C.c_double), ("max_grad_norm", C.c_double)]


def lib():
    """Load (building first if needed) the oracle shared library."""
    global _lib
    if _lib is None:
        # ZERO_ORACLE_LIB points the tests at another build of this oracle
        # (used to check that the pins catch planted mistakes)
        path = os.environ.get("ZERO_ORACLE_LIB") or _build.build()
        L = C.CDLL(path)
        P = C.c_void_p
        L.oracle_half_to_float.restype = C.c_float
        L.oracle_half_to_float.argtypes = [C.c_uint16, C.c_int32]
        L.oracle_float_to_half.restype = C.c_uint16
        L.oracle_float_to_half.argtypes = [C.c_float, C.c_int32]
        L.oracle_half_to_float_n.argtypes = [P, P, C.c_int64, C.c_int32]
        L.oracle_float_to_half_n.argtypes = [P, P, C.c_int64, C.c_int32]
        L.oracle_layout.restype = C.c_int32
        L.oracle_layout.argtypes = [P, C.c_int64, C.c_int32, C.c_int32, C.c_int64, P,
                                    P, P, P, P, P, P, P]
        L.oracle_fsm_update.restype = C.c_int32
        L.oracle_fsm_update.argtypes = [C.POINTER(FSM), C.c_int32]
        L.oracle_allreduce_sum.restype = C.c_int32
        L.oracle_allreduce_sum.argtypes = [C.c_int64, C.c_int32, C.c_int32, P, P]
        L.oracle_step.restype = C.c_int32
        L.oracle_step.argtypes = [C.c_int64, C.c_int32, C.c_int32, P, P, P, P, P,
                                  C.POINTER(AdamW), C.POINTER(FSM)]
        L.oracle_step_sharded.restype = C.c_int32
        L.oracle_step_sharded.argtypes = [C.c_int64, C.c_int32, C.c_int32, P, P, P, P, P, P,
                                          C.POINTER(AdamW), C.POINTER(FSM)]
        L.oracle_step_ex.restype = C.c_int32
        L.oracle_step_ex.argtypes = [C.c_int64, C.c_int32, C.c_int32, C.c_int32, P, P, P, P, P,
                                     C.POINTER(AdamW), C.POINTER(StepOpts), C.POINTER(FSM)]
        L.oracle_step_ex_sample.restype = C.c_int32
        L.oracle_step_ex_sample.argtypes = [C.c_int64, C.c_int32, C.c_int32, C.c_int32, P, P, P, P, P,
                                            C.POINTER(AdamW), C.POINTER(StepOpts), C.POINTER(FSM),
                                            C.c_double]
        L.oracle_model_state_bytes.restype = C.c_double
        L.oracle_model_state_bytes.argtypes = [C.c_int32, C.c_double, C.c_double]
        L.oracle_fp32_weight_bytes.restype = C.c_double
        L.oracle_fp32_weight_bytes.argtypes = [C.c_double]
        _lib = L
    return _lib


def _ptr(a: np.ndarray):
    assert a.flags["C_CONTIGUOUS"]
    return a.ctypes.data_as(C.c_void_p)


# ---- half formats ---------------------------------------------------------

def half_to_float(h: np.ndarray, dtype: int) -> np.ndarray:
    h = np.ascontiguousarray(h, dtype=np.uint16)
    out = np.empty(h.shape, np.float32)
    lib().oracle_half_to_float_n(_ptr(h), _ptr(out), h.size, dtype)
    return out


def float_to_half(x: np.ndarray, dtype: int) -> np.ndarray:
    x = np.ascontiguousarray(x, dtype=np.float32)
    out = np.empty(x.shape, np.uint16)
    lib().oracle_float_to_half_n(_ptr(x), _ptr(out), x.size, dtype)
    return out


# ---- layout ----------------------------------------------------------------

class Layout:
    """The oracle's own derivation of the flat layout, buckets and layers."""

    def __init__(self, numels, R, align=8, bucket_elems=0, layer_ids=None):
        numels = np.ascontiguousarray(numels, dtype=np.int64)
        n = numels.size
        self.offsets = np.zeros(n, np.int64)
        sizes = np.zeros(6, np.int64)
        self.tensor_bucket = np.zeros(n, np.int64)
        blo, bhi = np.zeros(n, np.int64), np.zeros(n, np.int64)
        llo, lhi = np.zeros(n, np.int64), np.zeros(n, np.int64)
        lid = None
        if layer_ids is not None:
            lid = np.ascontiguousarray(layer_ids, dtype=np.int32)
        rc = lib().oracle_layout(_ptr(numels), n, R, align, bucket_elems,
                                 None if lid is None else _ptr(lid),
                                 _ptr(self.offsets), _ptr(sizes), _ptr(self.tensor_bucket),
                                 _ptr(blo), _ptr(bhi), _ptr(llo), _ptr(lhi))
        if rc != 0:
            raise ValueError(f"oracle_layout rejected the input (code {rc})")
        self.numels = numels
        self.R = R
        self.P, self.L, self.S, self.T, nb, nl = (int(v) for v in sizes)
        self.buckets = list(zip(blo[:nb].tolist(), bhi[:nb].tolist()))
        self.layers = list(zip(llo[:nl].tolist(), lhi[:nl].tolist()))

    def flat_index(self) -> np.ndarray:
        """Flat (padded) index of every unpadded element, in tensor order."""
        return np.concatenate([np.arange(o, o + n, dtype=np.int64)
                               for o, n in zip(self.offsets.tolist(), self.numels.tolist())])


# ---- steps -----------------------------------------------------------------

def make_fsm(mode, scale=1.0, interval=1000, growth=2.0, backoff=0.5, min_scale=1.0,
             good=0, t=0) -> FSM:
    return FSM(mode, scale, interval, growth, backoff, min_scale, good, t, 0, 0, 0.0)


def allreduce_sum(grads: np.ndarray, dtype: int):
    """grads: (R, P) uint16. Returns (acc float32[P], overflow)."""
    g = np.ascontiguousarray(grads, dtype=np.uint16)
    R, P = g.shape
    acc = np.empty(P, np.float32)
    ovf = lib().oracle_allreduce_sum(P, R, dtype, _ptr(g), _ptr(acc))
    return acc, bool(ovf)


class State:
    """Unpartitioned model state: master, m, v (float32) and param (uint16)."""

    def __init__(self, master: np.ndarray, dtype: int, param=None):
        self.master = np.ascontiguousarray(master, dtype=np.float32).copy()
        self.m = np.zeros_like(self.master)
        self.v = np.zeros_like(self.master)
        self.param = (float_to_half(self.master, dtype) if param is None
                      else np.ascontiguousarray(param, dtype=np.uint16).copy())
        self.dtype = dtype

    def copy(self):
        s = State.__new__(State)
        s.master, s.m, s.v, s.param = (self.master.copy(), self.m.copy(), self.v.copy(),
                                       self.param.copy())
        s.dtype = self.dtype
        return s


def step(state: State, grads: np.ndarray, hp: AdamW, fsm: FSM) -> bool:
    """One unpartitioned step in place. grads: (R, P) uint16. Returns skipped."""
    g = np.ascontiguousarray(grads, dtype=np.uint16)
    R, P = g.shape
    assert P == state.master.size
    rc = lib().oracle_step(P, R, state.dtype, _ptr(g), _ptr(state.master), _ptr(state.m),
                           _ptr(state.v), _ptr(state.param), C.byref(hp), C.byref(fsm))
    if rc < 0:
        raise MemoryError("oracle_step")
    return bool(rc)


def step_ex(state: State, micro_grads: np.ndarray, hp: AdamW, fsm: FSM, grad_divisor=1.0,
            max_grad_norm=0.0) -> bool:
    """Step with accumulation over micro-batches and optional global-norm
    clipping. micro_grads: (n_micro, R, P) uint16. Returns skipped."""
    g = np.ascontiguousarray(micro_grads, dtype=np.uint16)
    n_micro, R, P = g.shape
    opts = StepOpts(grad_divisor, max_grad_norm)
    rc = lib().oracle_step_ex(P, R, state.dtype, n_micro, _ptr(g), _ptr(state.master),
                              _ptr(state.m), _ptr(state.v), _ptr(state.param), C.byref(hp),
                              C.byref(opts), C.byref(fsm))
    if rc < 0:
        raise ValueError("oracle_step_ex rejected its arguments")
    return bool(rc)


def step_ex_sample(state: State, micro_grads: np.ndarray, hp: AdamW, fsm: FSM, grad_divisor,
                   max_grad_norm, norm_sq_all) -> bool:
    """step_ex on a sample of a model's elements, clipping with the whole
    model's squared norm norm_sq_all. Returns skipped."""
    g = np.ascontiguousarray(micro_grads, dtype=np.uint16)
    n_micro, R, P = g.shape
    opts = StepOpts(grad_divisor, max_grad_norm)
    rc = lib().oracle_step_ex_sample(P, R, state.dtype, n_micro, _ptr(g), _ptr(state.master),
                                     _ptr(state.m), _ptr(state.v), _ptr(state.param), C.byref(hp),
                                     C.byref(opts), C.byref(fsm), float(norm_sq_all))
    if rc < 0:
        raise ValueError("oracle_step_ex_sample rejected its arguments")
    return bool(rc)


def step_sharded(S: int, R: int, dtype: int, grads, master, m, v, param, hp, fsm):
    """The partitioned step over the padded layout (all arrays length R*S;
    grads (R, R*S)). Returns (skipped, gathered params)."""
    gathered = np.empty(R * S, np.uint16)
    rc = lib().oracle_step_sharded(S, R, dtype, _ptr(grads), _ptr(master), _ptr(m), _ptr(v),
                                   _ptr(param), _ptr(gathered), C.byref(hp), C.byref(fsm))
    if rc < 0:
        raise MemoryError("oracle_step_sharded")
    return bool(rc), gathered


def fsm_update(fsm: FSM, overflow: bool) -> bool:
    return bool(lib().oracle_fsm_update(C.byref(fsm), int(overflow)))


def model_state_bytes(stage: int, psi: float, N: float) -> float:
    return lib().oracle_model_state_bytes(stage, float(psi), float(N))


def fp32_weight_bytes(psi: float) -> float:
    return lib().oracle_fp32_weight_bytes(float(psi))
