"""ZeRO data-parallel hot path for B200 (sm_100a): partitioned mixed-precision
AdamW over a flat sharded state, R data-parallel ranks simulated on one GPU.

The compute is in libzero_b200.so (hand-written CUDA, C ABI in
include/zero_b200.h); this package binds it with ctypes and uses PyTorch
only for device memory and streams.
"""
from ._capi import (  # noqa: F401
    ZERO_OK, ZERO_ERR_INVALID_ARG, ZERO_ERR_ALIGN, ZERO_ERR_CUDA, ZERO_ERR_OOM, ZERO_ERR_RANGE,
    ZERO_ERR_TIMEOUT, ZERO_ERR_STATE, STATUS_NAMES,
    ZERO_BF16, ZERO_FP16, ZERO_LOSS_SCALE_GET, ZERO_LOSS_SCALE_SET, ZERO_MAX_RANKS,
    ZERO_SCALE_DYNAMIC, ZERO_SCALE_NONE, ZERO_SCALE_STATIC, LIB_PATH, StateHandle, ZeroError,
    zero_adamw, zero_ctx_create, zero_ctx_destroy, zero_gather_layer, zero_gather_layers,
    ZERO_GATHER_MAX_LAYERS, zero_last_error,
    zero_loss_scale, zero_plan, zero_plan_bucket, zero_plan_destroy, zero_plan_get_info,
    zero_plan_layer, zero_plan_memory, zero_plan_step_tiles, zero_plan_tensor, zero_reduce_scatter_bucket, zero_step,
    zero_reduce_scatter_bucket_ex, zero_step_ex, ZERO_RS_ACCUMULATE, ZERO_STEP_ADD_ACC,
    zero_step_noalloc, ZERO_NOALLOC_MAX_ELEMS, zero_sync, zero_version, zero_grads_ready,
    zero_grads_join, zero_prefetch_begin, zero_layer_acquire, zero_layer_release, zero_cpu_step,
    zero_step_shard, zero_step_commit, zero_ctx_reserve_steps, zero_test_drop_tile,
    zero_sched_set_comm_sms, zero_step_shard_ex, zero_reduce_scatter_shard, zero_grad_norm_shard,
    zero_debug_bounds, zero_cpu_scan, zero_cpu_update, zero_cpu_commit, zero_ctx_set_grad_divisor,
    ZERO_RS_NORM, ZERO_STEP_NORM_FROM_RS, zero_reduce_scatter_buckets, zero_trace_start, zero_trace_read,
    zero_trace_stop, TRACE_NAMES, zero_cpu_scan_shard, zero_cpu_decide, zero_cpu_update_shard,
    zero_ipc_export, zero_ipc_open, zero_ipc_close, zero_ctx_set_param_push, ZERO_STEP_PUSH_PARAMS,
    zero_take_overflow, ZERO_STEP_CLEAN)
from .state import Plan, ShardedState  # noqa: F401
