// C ABI of libzero_b200.so: context lifecycle, argument validation, kernel
// launches and the loss-scale state. See include/zero_b200.h for the
// contract of every call.
#include <algorithm>
#include <cmath>
#include <cstring>
#include <exception>
#include <new>
#include <string>
#include <vector>

#include "internal.h"

namespace {

thread_local std::string g_last_error;

}  // namespace

zero_status zb_fail(zero_status code, const std::string& msg) noexcept {
    try {
        g_last_error = msg;
    } catch (...) {
        g_last_error.clear();  // no room for the message: the status still tells
    }
    return code;
}

zero_status zb_exception(const char* where) noexcept {
    try {
        try {
            throw;
        } catch (const std::exception& e) {
            return zb_fail(ZERO_ERR_OOM, std::string(where) + ": host resources exhausted: " + e.what());
        } catch (...) {
            return zb_fail(ZERO_ERR_OOM, std::string(where) + ": host resources exhausted");
        }
    } catch (...) {
        g_last_error.clear();  // not even the message fits
        return ZERO_ERR_OOM;
    }
}

namespace {

zero_status cuda_fail(const char* where, cudaError_t e) {
    return zb_fail(ZERO_ERR_CUDA, std::string(where) + ": " + cudaGetErrorName(e) + ": " +
                                      cudaGetErrorString(e));
}

zero_status check_device(const zero_ctx_t* ctx, const char* where) {
    int dev = -1;
    cudaError_t e = cudaGetDevice(&dev);
    if (e != cudaSuccess) return cuda_fail(where, e);
    if (dev != ctx->device)
        return zb_fail(ZERO_ERR_INVALID_ARG, std::string(where) + ": context belongs to device " +
                                                 std::to_string(ctx->device) +
                                                 " but device " + std::to_string(dev) +
                                                 " is current");
    // surface errors of earlier asynchronous work
    e = cudaPeekAtLastError();
    if (e != cudaSuccess) {
        cudaGetLastError();
        return cuda_fail(where, e);
    }
    return ZERO_OK;
}

bool aligned(const void* p, uintptr_t a) { return (reinterpret_cast<uintptr_t>(p) % a) == 0; }

template <typename Ptr>
zero_status check_ranks(Ptr const* arr, int R, uintptr_t align, const char* where,
                        const char* what) {
    if (!arr) return zb_fail(ZERO_ERR_INVALID_ARG, std::string(where) + ": " + what + " is NULL");
    for (int r = 0; r < R; ++r) {
        if (!arr[r])
            return zb_fail(ZERO_ERR_INVALID_ARG, std::string(where) + ": " + what + "[" +
                                                     std::to_string(r) + "] is NULL");
        if (!aligned(arr[r], align))
            return zb_fail(ZERO_ERR_ALIGN, std::string(where) + ": " + what + "[" +
                                               std::to_string(r) + "] is not " +
                                               std::to_string(align) + "-byte aligned");
    }
    return ZERO_OK;
}

// Validate the state sets; returns the number of sets (1 or 2) in *sets.
zero_status check_state(const zero_ctx_t* ctx, const zero_state* st, const char* where, int* sets,
                        bool params_only) {
    if (!st) return zb_fail(ZERO_ERR_INVALID_ARG, std::string(where) + ": state is NULL");
    const int R = ctx->R;
    zero_status s;
    const bool set1_any = st->master[1] || st->m[1] || st->v[1] || st->param[1];
    const bool set1_all = st->master[1] && st->m[1] && st->v[1] && st->param[1];
    if (params_only) {
        if ((s = check_ranks(st->param[0], R, 16, where, "param[0]")) != ZERO_OK) return s;
        if (st->param[1] && (s = check_ranks(st->param[1], R, 16, where, "param[1]")) != ZERO_OK)
            return s;
        *sets = st->param[1] ? 2 : 1;
        return ZERO_OK;
    }
    if (set1_any && !set1_all)
        return zb_fail(ZERO_ERR_INVALID_ARG,
                       std::string(where) + ": state set 1 must be given completely or not at all");
    for (int k = 0; k < (set1_all ? 2 : 1); ++k) {
        if ((s = check_ranks(st->master[k], R, 32, where, k ? "master[1]" : "master[0]")) != ZERO_OK) return s;
        if ((s = check_ranks(st->m[k], R, 32, where, k ? "m[1]" : "m[0]")) != ZERO_OK) return s;
        if ((s = check_ranks(st->v[k], R, 32, where, k ? "v[1]" : "v[0]")) != ZERO_OK) return s;
        if ((s = check_ranks(st->param[k], R, 16, where, k ? "param[1]" : "param[0]")) != ZERO_OK) return s;
    }
    *sets = set1_all ? 2 : 1;
    return ZERO_OK;
}

void fill_state_ptrs(const zero_ctx_t* ctx, const zero_state* st, int sets, zb::RankPtrs* p) {
    for (int r = 0; r < ctx->R; ++r)
        for (int k = 0; k < 2; ++k) {
            const int from = (k < sets) ? k : 0;  // one set: both slots alias set 0
            p->master[k][r] = st->master[from] ? st->master[from][r] : nullptr;
            p->m[k][r] = st->m[from] ? st->m[from][r] : nullptr;
            p->v[k][r] = st->v[from] ? st->v[from][r] : nullptr;
            p->param[k][r] = st->param[from] ? st->param[from][r] : nullptr;
        }
}

// Host-built table of (beta1^t, beta2^t), t = 0..len-1, computed with the C
// library's pow in double; the device forms the bias corrections from it.
zero_status ensure_powtab(zero_ctx_t* ctx, double b1, double b2, int64_t need_t, cudaStream_t s) {
    if (ctx->powtab && ctx->pow_valid && ctx->pow_b1 == b1 && ctx->pow_b2 == b2 &&
        need_t < ctx->powtab_len)
        return ZERO_OK;
    // growing the table allocates and copies synchronously, which a stream capture forbids
    cudaStreamCaptureStatus cap = cudaStreamCaptureStatusNone;
    if (cudaStreamIsCapturing(s, &cap) == cudaSuccess && cap != cudaStreamCaptureStatusNone)
        return zb_fail(ZERO_ERR_STATE,
                       "zero_step: the bias-correction table must grow, which cannot happen inside a "
                       "stream capture; call zero_ctx_reserve_steps before capturing");
    int64_t len = 1024;
    while (len <= need_t) len *= 2;
    std::vector<double2> host(static_cast<size_t>(len));
    for (int64_t t = 0; t < len; ++t)
        host[t] = make_double2(std::pow(b1, static_cast<double>(t)), std::pow(b2, static_cast<double>(t)));
    // Kernels already queued, and kernels captured into CUDA graphs, hold the
    // old table's address: keep it allocated until the context is destroyed.
    // A replay that outruns its table reads the last entry and raises the
    // device error flag instead of reading past the end.
    if (ctx->powtab) ctx->powtab_retired.push_back(ctx->powtab);
    ctx->powtab = nullptr;
    ctx->powtab_len = 0;
    cudaError_t e;
    e = cudaMalloc(&ctx->powtab, sizeof(double2) * static_cast<size_t>(len));
    if (e != cudaSuccess) {
        cudaGetLastError();
        return zb_fail(ZERO_ERR_OOM, "zero_step: cannot allocate the power table");
    }
    e = cudaMemcpy(ctx->powtab, host.data(), sizeof(double2) * host.size(), cudaMemcpyHostToDevice);
    if (e != cudaSuccess) return cuda_fail("zero_step: power table upload", e);
    ctx->powtab_len = len;
    ctx->pow_b1 = b1;
    ctx->pow_b2 = b2;
    ctx->pow_valid = true;
    return ZERO_OK;
}

}  // namespace

extern "C" zero_status zero_ctx_create(const zero_plan_t* plan, const zero_loss_scale_config* cfg,
                                       zero_ctx_t** out) {
    return zb_guarded("zero_ctx_create", [&]() -> zero_status {
        if (!out) return zb_fail(ZERO_ERR_INVALID_ARG, "zero_ctx_create: out is NULL");
        *out = nullptr;
        if (!plan || !cfg) return zb_fail(ZERO_ERR_INVALID_ARG, "zero_ctx_create: NULL plan or cfg");
        if (cfg->mode < ZERO_SCALE_NONE || cfg->mode > ZERO_SCALE_DYNAMIC)
            return zb_fail(ZERO_ERR_INVALID_ARG, "zero_ctx_create: bad loss-scale mode");
        if (cfg->mode != ZERO_SCALE_NONE && !(cfg->init_scale > 0.0f && std::isfinite(cfg->init_scale)))
            return zb_fail(ZERO_ERR_INVALID_ARG, "zero_ctx_create: init_scale must be finite and > 0");
        if (cfg->mode == ZERO_SCALE_DYNAMIC) {
            if (cfg->growth_interval < 1)
                return zb_fail(ZERO_ERR_INVALID_ARG, "zero_ctx_create: growth_interval must be >= 1");
            if (!(cfg->growth_factor > 1.0f) || !(cfg->backoff_factor > 0.0f && cfg->backoff_factor < 1.0f) ||
                !(cfg->min_scale > 0.0f))
                return zb_fail(ZERO_ERR_INVALID_ARG,
                               "zero_ctx_create: need growth_factor > 1, 0 < backoff_factor < 1, min_scale > 0");
        }
        if (cfg->reserved != 0) return zb_fail(ZERO_ERR_INVALID_ARG, "zero_ctx_create: reserved must be 0");

        zero_ctx_t* ctx = new (std::nothrow) zero_ctx_t();
        if (!ctx) return zb_fail(ZERO_ERR_OOM, "zero_ctx_create: out of host memory");
        cudaError_t e = cudaGetDevice(&ctx->device);
        if (e != cudaSuccess) {
            delete ctx;
            cudaGetLastError();
            return cuda_fail("zero_ctx_create", e);
        }
        ctx->R = plan->R;
        ctx->dtype = plan->dtype;
        ctx->S = plan->S;
        ctx->T = plan->T;
        ctx->bucket_lo = plan->bucket_lo;
        ctx->bucket_hi = plan->bucket_hi;
        ctx->layer_lo = plan->layer_lo;
        ctx->layer_hi = plan->layer_hi;
        ctx->tensor_bucket = plan->tensor_bucket;
        ctx->bucket_ntensors.assign(plan->bucket_lo.size(), 0);
        for (int64_t b : plan->tensor_bucket) ctx->bucket_ntensors[b] += 1;
        ctx->cfg = *cfg;
        ctx->grid_cap = zb::step_grid_cap(ctx->device);

        // norm-share slots: one per bucket and one for the whole range
        const size_t slots = ctx->bucket_lo.size() + 1;
        ctx->rs_norm_valid.assign(slots, 0);
        ctx->rs_norm_div.assign(slots, 1.0);
        ctx->rs_norm_owner.assign(slots, 0);
        auto free_scratch = [ctx] {
            cudaFree(ctx->st);
            cudaFree(ctx->partials);
            cudaFree(ctx->rs_norm_partials);
            cudaFree(ctx->rs_norm_done);
            cudaFree(ctx->rs_norm);
        };
        e = cudaMalloc(&ctx->st, sizeof(zb::DevState));
        if (e == cudaSuccess) e = cudaMalloc(&ctx->partials, sizeof(double) * ctx->grid_cap);
        if (e == cudaSuccess) e = cudaMalloc(&ctx->rs_norm_partials, sizeof(double) * ctx->grid_cap * slots);
        if (e == cudaSuccess) e = cudaMalloc(&ctx->rs_norm_done, sizeof(uint32_t) * slots);
        if (e == cudaSuccess) e = cudaMalloc(&ctx->rs_norm, sizeof(double) * slots);
        if (e != cudaSuccess) {
            cudaGetLastError();
            free_scratch();
            delete ctx;
            return zb_fail(ZERO_ERR_OOM, "zero_ctx_create: cannot allocate device scratch");
        }
        zb::DevState init{};
        init.scale = cfg->mode == ZERO_SCALE_NONE ? 1.0f : cfg->init_scale;
        e = cudaMemcpy(ctx->st, &init, sizeof(init), cudaMemcpyHostToDevice);
        if (e == cudaSuccess) e = cudaMemset(ctx->partials, 0, sizeof(double) * ctx->grid_cap);
        if (e == cudaSuccess) e = cudaMemset(ctx->rs_norm_done, 0, sizeof(uint32_t) * slots);
        if (e == cudaSuccess) e = cudaMemset(ctx->rs_norm, 0, sizeof(double) * slots);
        if (e != cudaSuccess) {
            free_scratch();
            delete ctx;
            return cuda_fail("zero_ctx_create", e);
        }
        *out = ctx;
        return ZERO_OK;
    });
}

extern "C" zero_status zero_ctx_set_grad_divisor(zero_ctx_t* ctx, double grad_divisor) {
    return zb_guarded("zero_ctx_set_grad_divisor", [&]() -> zero_status {
        if (!ctx) return zb_fail(ZERO_ERR_INVALID_ARG, "zero_ctx_set_grad_divisor: ctx is NULL");
        if (!(grad_divisor >= 1.0) || !std::isfinite(grad_divisor))
            return zb_fail(ZERO_ERR_INVALID_ARG, "zero_ctx_set_grad_divisor: need a finite divisor >= 1");
        ctx->grad_divisor = grad_divisor;
        return ZERO_OK;
    });
}

zb::RsNorm zb_rs_norm_note(zero_ctx_t* ctx, int64_t first, int64_t count, bool norm, int32_t owner_lo,
                           int32_t owner_hi) {
    const size_t whole = ctx->bucket_lo.size();
    const size_t slot = first < 0 ? whole : static_cast<size_t>(first);
    if (owner_hi < 0) owner_hi = ctx->R;
    const int64_t owner = (static_cast<int64_t>(owner_lo) << 32) | static_cast<int64_t>(owner_hi);
    if (first < 0) {
        // the whole range is rewritten: every per-bucket share is stale
        std::fill(ctx->rs_norm_valid.begin(), ctx->rs_norm_valid.end(), 0);
        ctx->rs_norm_valid[whole] = norm ? 1 : 0;
        ctx->rs_norm_div[whole] = ctx->grad_divisor;
        ctx->rs_norm_owner[whole] = owner;
    } else {
        ctx->rs_norm_valid[whole] = 0;
        for (int64_t b = first; b < first + count; ++b) {
            ctx->rs_norm_valid[static_cast<size_t>(b)] = norm ? 1 : 0;
            ctx->rs_norm_div[static_cast<size_t>(b)] = ctx->grad_divisor;
            ctx->rs_norm_owner[static_cast<size_t>(b)] = owner;
        }
    }
    zb::RsNorm n;
    if (!norm) return n;
    n.partials = ctx->rs_norm_partials + slot * static_cast<size_t>(ctx->grid_cap);
    n.done = ctx->rs_norm_done + slot;
    n.out = ctx->rs_norm + slot;
    n.cap = static_cast<uint32_t>(ctx->grid_cap);
    n.mode = ctx->cfg.mode;
    n.divisor = ctx->grad_divisor;
    return n;
}

cudaError_t zb_rs_launch(zero_ctx_t* ctx, int64_t first, int64_t count, const zb::RankPtrs& p,
                         cudaStream_t s, int32_t flags, int max_sms) {
    int64_t lo = 0, hi = ctx->T;
    if (first >= 0) {
        lo = ctx->bucket_lo[static_cast<size_t>(first + count - 1)];
        hi = ctx->bucket_hi[static_cast<size_t>(first)];
    }
    const bool with_norm = (flags & ZERO_RS_NORM) != 0;
    const zb::RsNorm norm = zb_rs_norm_note(ctx, first, count, with_norm);
    ZbTraceScope trace(ctx, ZERO_TRACE_REDUCE_SCATTER, s, first);
    cudaError_t e = cudaSuccess;
    // a group's share lands in its first bucket's slot; the others hold 0
    if (with_norm && first >= 0 && count > 1)
        e = cudaMemsetAsync(ctx->rs_norm + first + 1, 0, sizeof(double) * static_cast<size_t>(count - 1), s);
    if (e == cudaSuccess)
        e = zb::launch_reduce_scatter(ctx->R, ctx->dtype, ctx->S, lo, hi, ctx->st, p, s,
                                      (flags & ZERO_RS_ACCUMULATE) != 0, max_sms,
                                      with_norm ? &norm : nullptr);
    if (e != cudaSuccess) {
        const size_t whole = ctx->bucket_lo.size();
        if (first < 0) ctx->rs_norm_valid[whole] = 0;
        for (int64_t b = first; first >= 0 && b < first + count; ++b) ctx->rs_norm_valid[static_cast<size_t>(b)] = 0;
    }
    return e;
}

extern "C" zero_status zero_ctx_destroy(zero_ctx_t* ctx) {
    return zb_guarded("zero_ctx_destroy", [&]() -> zero_status {
        if (!ctx) return ZERO_OK;
        int prev = -1;
        cudaGetDevice(&prev);
        cudaSetDevice(ctx->device);
        cudaError_t e = cudaDeviceSynchronize();
        zb_sched_destroy(ctx);
        zb_trace_destroy(ctx);
        cudaFree(ctx->st);
        cudaFree(ctx->partials);
        cudaFree(ctx->rs_norm_partials);
        cudaFree(ctx->rs_norm_done);
        cudaFree(ctx->rs_norm);
        if (ctx->powtab) cudaFree(ctx->powtab);
        for (double2* old : ctx->powtab_retired) cudaFree(old);
        if (prev >= 0) cudaSetDevice(prev);
        delete ctx;
        if (e != cudaSuccess) return cuda_fail("zero_ctx_destroy", e);
        return ZERO_OK;
    });
}

extern "C" zero_status zero_ctx_reserve_steps(zero_ctx_t* ctx, int64_t steps, double beta1, double beta2,
                                              void* stream) {
    return zb_guarded("zero_ctx_reserve_steps", [&]() -> zero_status {
        if (!ctx) return zb_fail(ZERO_ERR_INVALID_ARG, "zero_ctx_reserve_steps: ctx is NULL");
        zero_status s = check_device(ctx, "zero_ctx_reserve_steps");
        if (s != ZERO_OK) return s;
        if (steps < 0 || !(beta1 >= 0.0 && beta1 < 1.0) || !(beta2 >= 0.0 && beta2 < 1.0))
            return zb_fail(ZERO_ERR_INVALID_ARG, "zero_ctx_reserve_steps: need steps >= 0 and 0 <= beta < 1");
        return ensure_powtab(ctx, beta1, beta2, ctx->t_bound + 1 + steps, static_cast<cudaStream_t>(stream));
    });
}

extern "C" zero_status zero_test_drop_tile(zero_ctx_t* ctx, int64_t tile) {
    return zb_guarded("zero_test_drop_tile", [&]() -> zero_status {
        if (!ctx) return zb_fail(ZERO_ERR_INVALID_ARG, "zero_test_drop_tile: ctx is NULL");
        if (tile < 0 || tile >= 0xffffffffLL)
            return zb_fail(ZERO_ERR_INVALID_ARG, "zero_test_drop_tile: need 0 <= tile < 2^32 - 1");
        ctx->drop_tile = static_cast<uint32_t>(tile);
        return ZERO_OK;
    });
}

extern "C" zero_status zero_reduce_scatter_bucket(zero_ctx_t* ctx, int64_t bucket,
                                                  const void* const* grads, float* const* acc,
                                                  void* stream) {
    return zb_guarded("zero_reduce_scatter_bucket", [&]() -> zero_status {
        return zero_reduce_scatter_bucket_ex(ctx, bucket, grads, acc, 0, stream);
    });
}

extern "C" zero_status zero_reduce_scatter_bucket_ex(zero_ctx_t* ctx, int64_t bucket,
                                                     const void* const* grads, float* const* acc,
                                                     int32_t flags, void* stream) {
    return zb_guarded("zero_reduce_scatter_bucket_ex", [&]() -> zero_status {
        if (bucket == -1) return zero_reduce_scatter_buckets(ctx, -1, 1, grads, acc, flags, stream);
        if (ctx && (bucket < 0 || bucket >= static_cast<int64_t>(ctx->bucket_lo.size())))
            return zb_fail(ZERO_ERR_RANGE, "zero_reduce_scatter_bucket: bucket index out of range");
        return zero_reduce_scatter_buckets(ctx, bucket, 1, grads, acc, flags, stream);
    });
}

extern "C" zero_status zero_reduce_scatter_buckets(zero_ctx_t* ctx, int64_t first, int64_t count,
                                                   const void* const* grads, float* const* acc,
                                                   int32_t flags, void* stream) {
    return zb_guarded("zero_reduce_scatter_buckets", [&]() -> zero_status {
        const char* where = "zero_reduce_scatter_bucket";
        if (flags & ~(ZERO_RS_ACCUMULATE | ZERO_RS_NORM))
            return zb_fail(ZERO_ERR_INVALID_ARG, "zero_reduce_scatter_bucket_ex: unknown flags");
        if (!ctx) return zb_fail(ZERO_ERR_INVALID_ARG, "zero_reduce_scatter_bucket: ctx is NULL");
        zero_status s = check_device(ctx, where);
        if (s != ZERO_OK) return s;
        const int64_t nb = static_cast<int64_t>(ctx->bucket_lo.size());
        if (!(first == -1 && count == 1) && (first < 0 || count < 1 || first > nb - count))
            return zb_fail(ZERO_ERR_RANGE, "zero_reduce_scatter_buckets: need 0 <= first, 1 <= count and "
                                           "first + count <= n_buckets (or first = -1, count = 1)");
        if ((s = check_ranks(grads, ctx->R, 16, where, "grads")) != ZERO_OK) return s;
        if ((s = check_ranks(acc, ctx->R, 32, where, "acc")) != ZERO_OK) return s;
        zb::RankPtrs p;
        for (int r = 0; r < ctx->R; ++r) {
            p.g[r] = grads[r];
            p.acc[r] = acc[r];
        }
        cudaError_t e = zb_rs_launch(ctx, first, count, p, static_cast<cudaStream_t>(stream), flags, 0);
        if (e != cudaSuccess) return cuda_fail(where, e);
        return ZERO_OK;
    });
}

extern "C" zero_status zero_step(zero_ctx_t* ctx, const zero_adamw* hp, const zero_state* state,
                                 const void* const* grads, void* stream) {
    return zb_guarded("zero_step", [&]() -> zero_status {
        return zero_step_ex(ctx, hp, state, grads, nullptr, stream);
    });
}

namespace {

// Parameters shared by the sharded calls (everything but the AdamW hyper-parameters).
zb::StepParams shard_params(const zero_ctx_t* ctx, int32_t owner_lo, int32_t owner_hi, double divisor,
                            double* partial) {
    zb::StepParams sp;
    sp.R = ctx->R;
    sp.dtype = ctx->dtype;
    sp.mode = ctx->cfg.mode;
    sp.S8 = static_cast<uint32_t>(ctx->S / 8);
    sp.T8 = static_cast<uint32_t>(ctx->T / 8);
    sp.divisor = divisor;
    sp.interval = ctx->cfg.growth_interval;
    sp.growth = ctx->cfg.growth_factor;
    sp.backoff = ctx->cfg.backoff_factor;
    sp.min_scale = ctx->cfg.min_scale;
    sp.st = ctx->st;
    sp.partials = ctx->partials;
    sp.powtab = ctx->powtab;
    sp.powtab_len = ctx->powtab_len;
    sp.grid_cap = ctx->grid_cap;
    sp.obeg = owner_lo;
    sp.oend = owner_hi;
    sp.partial_out = partial;
    return sp;
}

zero_status check_owner_range(const zero_ctx_t* ctx, int32_t lo, int32_t hi, const char* where) {
    if (lo < 0 || lo >= hi || hi > ctx->R)
        return zb_fail(ZERO_ERR_RANGE, std::string(where) + ": need 0 <= owner_lo < owner_hi <= R");
    return ZERO_OK;
}

zero_status check_all_grads(const zero_ctx_t* ctx, const void* const* grads, const char* where) {
    for (int r = 0; r < ctx->R; ++r) {
        if (!grads[r]) return zb_fail(ZERO_ERR_INVALID_ARG, std::string(where) + ": grads[" + std::to_string(r) + "] is NULL");
        if (!aligned(grads[r], 16)) return zb_fail(ZERO_ERR_ALIGN, std::string(where) + ": grads misaligned");
    }
    return ZERO_OK;
}

zero_status check_owned_acc(const zero_ctx_t* ctx, float* const* acc, int32_t lo, int32_t hi, const char* where) {
    if (!acc) return zb_fail(ZERO_ERR_INVALID_ARG, std::string(where) + ": acc is NULL");
    for (int r = lo; r < hi; ++r) {
        if (!acc[r]) return zb_fail(ZERO_ERR_INVALID_ARG, std::string(where) + ": acc[" + std::to_string(r) + "] is NULL");
        if (!aligned(acc[r], 32)) return zb_fail(ZERO_ERR_ALIGN, std::string(where) + ": acc misaligned");
    }
    (void)ctx;
    return ZERO_OK;
}

// Options of zero_step_ex / zero_step_shard_ex, validated; *out receives them.
zero_status check_step_opts(const zero_step_opts* opts, bool fused, const char* where, zero_step_opts* out) {
    zero_step_opts o{1.0, 0.0, 0, 0};
    if (opts) o = *opts;
    if (!(o.grad_divisor >= 1.0) || !std::isfinite(o.grad_divisor) || !(o.max_grad_norm >= 0.0) ||
        !std::isfinite(o.max_grad_norm) || o.reserved != 0)
        return zb_fail(ZERO_ERR_INVALID_ARG,
                       std::string(where) + ": need grad_divisor >= 1, finite max_grad_norm >= 0, reserved 0");
    if (o.flags & ~static_cast<int64_t>(ZERO_STEP_ADD_ACC | ZERO_STEP_NORM_FROM_RS | ZERO_STEP_PUSH_PARAMS))
        return zb_fail(ZERO_ERR_INVALID_ARG, std::string(where) + ": unknown flags");
    if ((o.flags & ZERO_STEP_ADD_ACC) && (!fused || o.max_grad_norm > 0.0))
        return zb_fail(ZERO_ERR_INVALID_ARG,
                       std::string(where) + ": ZERO_STEP_ADD_ACC needs the fused path (grads) and no clipping");
    if ((o.flags & ZERO_STEP_NORM_FROM_RS) && (fused || !(o.max_grad_norm > 0.0)))
        return zb_fail(ZERO_ERR_INVALID_ARG, std::string(where) +
                                                 ": ZERO_STEP_NORM_FROM_RS needs the two-pass path "
                                                 "(no grads) and clipping");
    *out = o;
    return ZERO_OK;
}

zero_status check_hp(const zero_adamw* hp, const char* where) {
    if (!(hp->lr >= 0.0) || !(hp->beta1 >= 0.0 && hp->beta1 < 1.0) || !(hp->beta2 >= 0.0 && hp->beta2 < 1.0) ||
        !(hp->eps > 0.0) || !(hp->weight_decay >= 0.0) || !std::isfinite(hp->lr) ||
        !std::isfinite(hp->weight_decay) || !std::isfinite(hp->eps))
        return zb_fail(ZERO_ERR_INVALID_ARG,
                       std::string(where) + ": need finite lr >= 0, 0 <= beta < 1, eps > 0, weight_decay >= 0");
    return ZERO_OK;
}

// ZERO_STEP_PUSH_PARAMS: the registered full-model buffers of every set the
// step may write (both with ping-pong state) into p->full; none without it.
zero_status fill_push_ptrs(const zero_ctx_t* ctx, const zero_step_opts& o, int sets, const char* where,
                           zb::RankPtrs* p) {
    const bool push = (o.flags & ZERO_STEP_PUSH_PARAMS) != 0;
    for (int k = 0; k < 2; ++k)
        for (int r = 0; r < ctx->R; ++r) p->full[k][r] = nullptr;
    if (!push) return ZERO_OK;
    for (int k = 0; k < sets; ++k)
        if (ctx->push_full[k].size() != static_cast<size_t>(ctx->R))
            return zb_fail(ZERO_ERR_STATE, std::string(where) + ": ZERO_STEP_PUSH_PARAMS, but no full-model buffers of "
                                                                 "state set " + std::to_string(k) +
                                                                 " are registered (zero_ctx_set_param_push)");
    for (int k = 0; k < 2; ++k) {
        const int from = k < sets ? k : 0;  // one set: both slots alias set 0
        for (int r = 0; r < ctx->R; ++r) p->full[k][r] = ctx->push_full[from][static_cast<size_t>(r)];
    }
    return ZERO_OK;
}

// Everything a step launch needs, for owners [owner_lo, owner_hi).
zb::StepParams step_params(const zero_ctx_t* ctx, const zero_adamw* hp, const zero_step_opts& o, int sets,
                           int32_t owner_lo, int32_t owner_hi, double* partial) {
    zb::StepParams sp = shard_params(ctx, owner_lo, owner_hi, o.grad_divisor, partial);
    sp.pingpong = sets == 2 ? 1 : 0;
    sp.dec = static_cast<float>(1.0 - hp->lr * hp->weight_decay);
    sp.b1f = static_cast<float>(hp->beta1);
    sp.omb1 = static_cast<float>(1.0 - hp->beta1);
    sp.b2f = static_cast<float>(hp->beta2);
    sp.omb2 = static_cast<float>(1.0 - hp->beta2);
    sp.epsf = static_cast<float>(hp->eps);
    sp.lr = hp->lr;
    sp.max_norm = o.max_grad_norm;
    sp.clip = o.max_grad_norm > 0.0 ? 1 : 0;
    sp.add_acc = (o.flags & ZERO_STEP_ADD_ACC) ? 1 : 0;
    sp.push = (o.flags & ZERO_STEP_PUSH_PARAMS) ? 1 : 0;
    return sp;
}

}  // namespace

extern "C" zero_status zero_step_ex(zero_ctx_t* ctx, const zero_adamw* hp, const zero_state* state,
                                    const void* const* grads, const zero_step_opts* opts,
                                    void* stream) {
    return zb_guarded("zero_step_ex", [&]() -> zero_status {
        const char* where = "zero_step";
        const bool fused = grads != nullptr;
        zero_step_opts o;
        zero_status s = check_step_opts(opts, fused, "zero_step_ex", &o);
        if (s != ZERO_OK) return s;
        const bool add_acc = (o.flags & ZERO_STEP_ADD_ACC) != 0;
        if (!ctx || !hp) return zb_fail(ZERO_ERR_INVALID_ARG, "zero_step: NULL ctx or hyper-parameters");
        if ((s = check_device(ctx, where)) != ZERO_OK) return s;
        if ((s = check_hp(hp, where)) != ZERO_OK) return s;
        int sets = 1;
        if ((s = check_state(ctx, state, where, &sets, false)) != ZERO_OK) return s;
        if (add_acc && (s = check_ranks(state->acc, ctx->R, 32, where, "acc")) != ZERO_OK) return s;
        if (fused) {
            if ((s = check_ranks(grads, ctx->R, 16, where, "grads")) != ZERO_OK) return s;
            if (sets == 1 && ctx->cfg.mode == ZERO_SCALE_DYNAMIC)
                return zb_fail(ZERO_ERR_INVALID_ARG,
                               "zero_step: a fused step with dynamic loss scaling needs state set 1 "
                               "(ping-pong) so that a skipped step can be undone; or use the two-pass path");
        } else {
            if ((s = check_ranks(state->acc, ctx->R, 32, where, "acc")) != ZERO_OK) return s;
        }
        if (sets == 1 && ctx->two_sets)
            return zb_fail(ZERO_ERR_STATE,
                           "zero_step: the current model may live in state set 1; pass both sets");

        cudaStream_t cs = static_cast<cudaStream_t>(stream);
        if ((s = ensure_powtab(ctx, hp->beta1, hp->beta2, ctx->t_bound + 1, cs)) != ZERO_OK) return s;

        zb::StepParams sp = step_params(ctx, hp, o, sets, 0, ctx->R, nullptr);
        if (fused) sp.drop_tile = ctx->drop_tile;

        zb::RankPtrs p;
        fill_state_ptrs(ctx, state, sets, &p);
        for (int r = 0; r < ctx->R; ++r) {
            p.g[r] = fused ? grads[r] : nullptr;
            p.acc[r] = (!fused || add_acc) ? state->acc[r] : nullptr;
        }
        if ((s = fill_push_ptrs(ctx, o, sets, "zero_step", &p)) != ZERO_OK) return s;
        // with ZERO_STEP_NORM_FROM_RS: the current norm slots, whole range or
        // every bucket, each taken with this step's divisor
        const size_t nb = ctx->bucket_lo.size();
        int64_t slot_first = 0, slot_count = 0;
        if (o.flags & ZERO_STEP_NORM_FROM_RS) {
            const int64_t all_owners = static_cast<int64_t>(ctx->R);  // owner range [0, R)
            auto ok = [&](size_t k) {
                return ctx->rs_norm_valid[k] && ctx->rs_norm_div[k] == o.grad_divisor &&
                       ctx->rs_norm_owner[k] == all_owners;
            };
            bool all = true;
            for (size_t b = 0; b < nb && all; ++b) all = ok(b);
            if (ok(nb)) {
                slot_first = static_cast<int64_t>(nb);
                slot_count = 1;
            } else if (all) {
                slot_count = static_cast<int64_t>(nb);
            } else {
                return zb_fail(ZERO_ERR_STATE,
                               "zero_step: ZERO_STEP_NORM_FROM_RS, but the reduce-scatters since the last step did "
                               "not record a current norm share of every bucket with this grad_divisor");
            }
        }
        ZbTraceScope trace(ctx, ZERO_TRACE_STEP, cs, -1);
        cudaError_t e = cudaSuccess;
        // clipping needs the global norm before any element is updated: the
        // reduce-scatters' shares, or one read-only pass over the accumulators,
        // or over the replicas when fused
        if (sp.clip) {
            if (slot_count > 0)
                e = zb::launch_clip_from_rs_norm(sp, ctx->rs_norm, slot_first, slot_count, cs);
            else
                e = fused ? zb::launch_grad_norm(sp, p, cs) : zb::launch_clip_norm(sp, p, cs);
        }
        if (e == cudaSuccess)
            e = fused ? zb::launch_fused_step(sp, p, cs) : zb::launch_step_from_acc(sp, p, cs);
        // the accumulators are consumed: the next step's shares start afresh
        std::fill(ctx->rs_norm_valid.begin(), ctx->rs_norm_valid.end(), 0);
        if (e != cudaSuccess) return cuda_fail(where, e);
        ctx->t_bound += 1;
        if (fused) ctx->drop_tile = 0xffffffffu;
        if (sp.pingpong) ctx->two_sets = true;
        return ZERO_OK;
    });
}

namespace {

// Shard-range variant of check_state: only owners [lo, hi) need pointers.
zero_status check_state_range(const zero_ctx_t* ctx, const zero_state* st, int lo, int hi,
                              const char* where, int* sets) {
    if (!st) return zb_fail(ZERO_ERR_INVALID_ARG, std::string(where) + ": state is NULL");
    const bool any1 = st->master[1] || st->m[1] || st->v[1] || st->param[1];
    const bool all1 = st->master[1] && st->m[1] && st->v[1] && st->param[1];
    if (any1 && !all1)
        return zb_fail(ZERO_ERR_INVALID_ARG, std::string(where) + ": state set 1 must be complete or absent");
    for (int k = 0; k < (all1 ? 2 : 1); ++k) {
        if (!st->master[k] || !st->m[k] || !st->v[k] || !st->param[k])
            return zb_fail(ZERO_ERR_INVALID_ARG, std::string(where) + ": NULL state array");
        for (int r = lo; r < hi; ++r) {
            const void* f[3] = {st->master[k][r], st->m[k][r], st->v[k][r]};
            for (const void* q : f) {
                if (!q) return zb_fail(ZERO_ERR_INVALID_ARG, std::string(where) + ": NULL state pointer");
                if (!aligned(q, 32)) return zb_fail(ZERO_ERR_ALIGN, std::string(where) + ": fp32 state misaligned");
            }
            if (!st->param[k][r]) return zb_fail(ZERO_ERR_INVALID_ARG, std::string(where) + ": NULL param pointer");
            if (!aligned(st->param[k][r], 16)) return zb_fail(ZERO_ERR_ALIGN, std::string(where) + ": param misaligned");
        }
    }
    *sets = all1 ? 2 : 1;
    (void)ctx;
    return ZERO_OK;
}

}  // namespace


extern "C" zero_status zero_reduce_scatter_shard(zero_ctx_t* ctx, int64_t bucket, const void* const* grads,
                                                 float* const* acc, int32_t owner_lo, int32_t owner_hi,
                                                 int32_t flags, void* stream) {
    return zb_guarded("zero_reduce_scatter_shard", [&]() -> zero_status {
        const char* where = "zero_reduce_scatter_shard";
        if (!ctx || !grads) return zb_fail(ZERO_ERR_INVALID_ARG, "zero_reduce_scatter_shard: NULL ctx or grads");
        if (flags & ~(ZERO_RS_ACCUMULATE | ZERO_RS_NORM))
            return zb_fail(ZERO_ERR_INVALID_ARG, "zero_reduce_scatter_shard: unknown flags");
        zero_status s = check_device(ctx, where);
        if (s != ZERO_OK) return s;
        if ((s = check_owner_range(ctx, owner_lo, owner_hi, where)) != ZERO_OK) return s;
        int64_t lo, hi;
        if (bucket == -1) {
            lo = 0;
            hi = ctx->T;
        } else if (bucket < 0 || bucket >= static_cast<int64_t>(ctx->bucket_lo.size())) {
            return zb_fail(ZERO_ERR_RANGE, "zero_reduce_scatter_shard: bucket index out of range");
        } else {
            lo = ctx->bucket_lo[bucket];
            hi = ctx->bucket_hi[bucket];
        }
        if ((s = check_all_grads(ctx, grads, where)) != ZERO_OK) return s;
        if ((s = check_owned_acc(ctx, acc, owner_lo, owner_hi, where)) != ZERO_OK) return s;
        // the bucket's part inside the owners' flat range [owner_lo * S, owner_hi * S)
        lo = std::max<int64_t>(lo, static_cast<int64_t>(owner_lo) * ctx->S);
        hi = std::min<int64_t>(hi, static_cast<int64_t>(owner_hi) * ctx->S);
        const bool with_norm = (flags & ZERO_RS_NORM) != 0;
        const zb::RsNorm norm = zb_rs_norm_note(ctx, bucket, 1, with_norm, owner_lo, owner_hi);
        cudaStream_t cs = static_cast<cudaStream_t>(stream);
        const size_t slot = bucket < 0 ? ctx->bucket_lo.size() : static_cast<size_t>(bucket);
        if (lo >= hi) {
            // no element of this bucket is owned here: its share is 0
            if (!with_norm) return ZERO_OK;
            cudaError_t e = cudaMemsetAsync(norm.out, 0, sizeof(double), cs);
            if (e != cudaSuccess) {
                ctx->rs_norm_valid[slot] = 0;
                return cuda_fail(where, e);
            }
            return ZERO_OK;
        }
        zb::RankPtrs p{};
        for (int r = 0; r < ctx->R; ++r) {
            p.g[r] = grads[r];
            p.acc[r] = (r >= owner_lo && r < owner_hi) ? acc[r] : nullptr;
        }
        ZbTraceScope trace(ctx, ZERO_TRACE_REDUCE_SCATTER, cs, bucket);
        cudaError_t e = zb::launch_reduce_scatter(ctx->R, ctx->dtype, ctx->S, lo, hi, ctx->st, p, cs,
                                                  (flags & ZERO_RS_ACCUMULATE) != 0, 0,
                                                  with_norm ? &norm : nullptr);
        if (e != cudaSuccess) {
            ctx->rs_norm_valid[slot] = 0;
            return cuda_fail(where, e);
        }
        return ZERO_OK;
    });
}

extern "C" zero_status zero_grad_norm_shard(zero_ctx_t* ctx, const void* const* grads, float* const* acc,
                                            double grad_divisor, int32_t owner_lo, int32_t owner_hi,
                                            double* partial, void* stream) {
    return zb_guarded("zero_grad_norm_shard", [&]() -> zero_status {
        const char* where = "zero_grad_norm_shard";
        if (!ctx || !partial) return zb_fail(ZERO_ERR_INVALID_ARG, "zero_grad_norm_shard: NULL ctx or partial");
        if (grads && acc) return zb_fail(ZERO_ERR_INVALID_ARG, "zero_grad_norm_shard: give at most one of grads and acc");
        if (!(grad_divisor >= 1.0) || !std::isfinite(grad_divisor))
            return zb_fail(ZERO_ERR_INVALID_ARG, "zero_grad_norm_shard: need a finite grad_divisor >= 1");
        zero_status s = check_device(ctx, where);
        if (s != ZERO_OK) return s;
        if ((s = check_owner_range(ctx, owner_lo, owner_hi, where)) != ZERO_OK) return s;
        if (!aligned(partial, 8)) return zb_fail(ZERO_ERR_ALIGN, "zero_grad_norm_shard: partial not 8-byte aligned");
        if (!grads && !acc) {
            // the sum of the shares this owner range's ZERO_RS_NORM reduce-scatters took
            const size_t nb = ctx->bucket_lo.size();
            const int64_t owner = (static_cast<int64_t>(owner_lo) << 32) | static_cast<int64_t>(owner_hi);
            auto ok = [&](size_t k) {
                return ctx->rs_norm_valid[k] && ctx->rs_norm_div[k] == grad_divisor && ctx->rs_norm_owner[k] == owner;
            };
            bool all = true;
            for (size_t b = 0; b < nb && all; ++b) all = ok(b);
            int64_t first = 0, count = 0;
            if (ok(nb)) {
                first = static_cast<int64_t>(nb);
                count = 1;
            } else if (all) {
                count = static_cast<int64_t>(nb);
            } else {
                return zb_fail(ZERO_ERR_STATE,
                               "zero_grad_norm_shard: no current ZERO_RS_NORM share of every bucket for this owner "
                               "range and grad_divisor");
            }
            cudaStream_t cs = static_cast<cudaStream_t>(stream);
            ZbTraceScope trace(ctx, ZERO_TRACE_NORM, cs, owner_lo);
            cudaError_t e = zb::launch_sum_norm_slots(ctx->rs_norm, first, count, partial, cs);
            if (e != cudaSuccess) return cuda_fail(where, e);
            return ZERO_OK;
        }
        if (grads && (s = check_all_grads(ctx, grads, where)) != ZERO_OK) return s;
        if (acc && (s = check_owned_acc(ctx, acc, owner_lo, owner_hi, where)) != ZERO_OK) return s;
        zb::StepParams sp = shard_params(ctx, owner_lo, owner_hi, grad_divisor, partial);
        zb::RankPtrs p{};
        for (int r = 0; r < ctx->R; ++r) {
            p.g[r] = grads ? grads[r] : nullptr;
            p.acc[r] = (acc && r >= owner_lo && r < owner_hi) ? acc[r] : nullptr;
        }
        cudaStream_t cs = static_cast<cudaStream_t>(stream);
        ZbTraceScope trace(ctx, ZERO_TRACE_NORM, cs, owner_lo);
        cudaError_t e = grads ? zb::launch_grad_norm(sp, p, cs) : zb::launch_clip_norm(sp, p, cs);
        if (e != cudaSuccess) return cuda_fail(where, e);
        return ZERO_OK;
    });
}

extern "C" zero_status zero_step_shard_ex(zero_ctx_t* ctx, const zero_adamw* hp, const zero_state* state,
                                          const void* const* grads, int32_t owner_lo, int32_t owner_hi,
                                          const zero_step_opts* opts, const double* global_norm_sq,
                                          double* partial, void* stream) {
    return zb_guarded("zero_step_shard_ex", [&]() -> zero_status {
        const char* where = "zero_step_shard";
        if (!ctx || !hp || !partial)
            return zb_fail(ZERO_ERR_INVALID_ARG, "zero_step_shard: NULL ctx, hp or partial");
        const bool fused = grads != nullptr;
        zero_step_opts o;
        zero_status s = check_step_opts(opts, fused, where, &o);
        if (s != ZERO_OK) return s;
        const bool add_acc = (o.flags & ZERO_STEP_ADD_ACC) != 0;
        const bool clip = o.max_grad_norm > 0.0;
        if (clip && !global_norm_sq)
            return zb_fail(ZERO_ERR_INVALID_ARG,
                           "zero_step_shard: clipping needs global_norm_sq (the cross-rank sum of the "
                           "zero_grad_norm_shard partials)");
        if (global_norm_sq && !aligned(global_norm_sq, 8))
            return zb_fail(ZERO_ERR_ALIGN, "zero_step_shard: global_norm_sq not 8-byte aligned");
        if ((s = check_device(ctx, where)) != ZERO_OK) return s;
        if ((s = check_owner_range(ctx, owner_lo, owner_hi, where)) != ZERO_OK) return s;
        if (!aligned(partial, 8)) return zb_fail(ZERO_ERR_ALIGN, "zero_step_shard: partial not 8-byte aligned");
        if ((s = check_hp(hp, where)) != ZERO_OK) return s;
        int sets = 1;
        if ((s = check_state_range(ctx, state, owner_lo, owner_hi, where, &sets)) != ZERO_OK) return s;
        if (fused && (s = check_all_grads(ctx, grads, where)) != ZERO_OK) return s;
        if ((!fused || add_acc) && (s = check_owned_acc(ctx, state->acc, owner_lo, owner_hi, where)) != ZERO_OK)
            return s;
        if (sets == 1 && ctx->cfg.mode == ZERO_SCALE_DYNAMIC)
            return zb_fail(ZERO_ERR_INVALID_ARG, "zero_step_shard: dynamic loss scaling needs state set 1 (ping-pong)");
        if (sets == 1 && ctx->two_sets)
            return zb_fail(ZERO_ERR_STATE, "zero_step_shard: the current model may live in state set 1");
        cudaStream_t cs = static_cast<cudaStream_t>(stream);
        if ((s = ensure_powtab(ctx, hp->beta1, hp->beta2, ctx->t_bound + 1, cs)) != ZERO_OK) return s;
        zb::StepParams sp = step_params(ctx, hp, o, sets, owner_lo, owner_hi, partial);
        if (fused) sp.drop_tile = ctx->drop_tile;
        zb::RankPtrs p{};
        for (int r = 0; r < ctx->R; ++r) {
            const bool owned = r >= owner_lo && r < owner_hi;
            p.g[r] = fused ? grads[r] : nullptr;
            p.acc[r] = ((!fused || add_acc) && owned) ? state->acc[r] : nullptr;
            for (int k = 0; k < 2; ++k) {
                const int from = k < sets ? k : 0;
                p.master[k][r] = owned ? state->master[from][r] : nullptr;
                p.m[k][r] = owned ? state->m[from][r] : nullptr;
                p.v[k][r] = owned ? state->v[from][r] : nullptr;
                p.param[k][r] = owned ? state->param[from][r] : nullptr;
            }
        }
        if ((s = fill_push_ptrs(ctx, o, sets, where, &p)) != ZERO_OK) return s;
        ZbTraceScope trace(ctx, ZERO_TRACE_STEP, cs, owner_lo);
        cudaError_t e = cudaSuccess;
        if (clip) e = zb::launch_clip_from_norm(sp, global_norm_sq, cs);
        if (e == cudaSuccess) e = fused ? zb::launch_fused_step(sp, p, cs) : zb::launch_step_from_acc(sp, p, cs);
        if (e != cudaSuccess) return cuda_fail(where, e);
        ctx->t_bound += 1;
        if (fused) ctx->drop_tile = 0xffffffffu;
        ctx->shard_pingpong = sp.pingpong;
        if (sp.pingpong) ctx->two_sets = true;
        return ZERO_OK;
    });
}

extern "C" zero_status zero_take_overflow(zero_ctx_t* ctx, int32_t* flag, void* stream) {
    return zb_guarded("zero_take_overflow", [&]() -> zero_status {
        const char* where = "zero_take_overflow";
        if (!ctx || !flag) return zb_fail(ZERO_ERR_INVALID_ARG, "zero_take_overflow: NULL ctx or flag");
        zero_status s = check_device(ctx, where);
        if (s != ZERO_OK) return s;
        if (!aligned(flag, 4)) return zb_fail(ZERO_ERR_ALIGN, "zero_take_overflow: flag not 4-byte aligned");
        cudaError_t e = zb::launch_take_overflow(ctx->st, flag, static_cast<cudaStream_t>(stream));
        if (e != cudaSuccess) return cuda_fail(where, e);
        return ZERO_OK;
    });
}

extern "C" zero_status zero_ctx_set_param_push(zero_ctx_t* ctx, void* const* full0, void* const* full1) {
    return zb_guarded("zero_ctx_set_param_push", [&]() -> zero_status {
        if (!ctx) return zb_fail(ZERO_ERR_INVALID_ARG, "zero_ctx_set_param_push: ctx is NULL");
        if (!full0) {
            ctx->push_full[0].clear();
            ctx->push_full[1].clear();
            return ZERO_OK;
        }
        void* const* sets[2] = {full0, full1};
        std::vector<void*> got[2];
        for (int k = 0; k < 2; ++k) {
            if (!sets[k]) continue;
            for (int r = 0; r < ctx->R; ++r) {
                if (!sets[k][r])
                    return zb_fail(ZERO_ERR_INVALID_ARG, "zero_ctx_set_param_push: full" + std::to_string(k) + "[" +
                                                             std::to_string(r) + "] is NULL");
                if (!aligned(sets[k][r], 16))
                    return zb_fail(ZERO_ERR_ALIGN, "zero_ctx_set_param_push: a buffer is not 16-byte aligned");
                got[k].push_back(sets[k][r]);
            }
        }
        ctx->push_full[0] = std::move(got[0]);
        ctx->push_full[1] = std::move(got[1]);
        return ZERO_OK;
    });
}

extern "C" zero_status zero_step_shard(zero_ctx_t* ctx, const zero_adamw* hp, const zero_state* state,
                                       const void* const* grads, int32_t owner_lo, int32_t owner_hi,
                                       double* partial, void* stream) {
    return zb_guarded("zero_step_shard", [&]() -> zero_status {
        if (!grads) return zb_fail(ZERO_ERR_INVALID_ARG, "zero_step_shard: grads is NULL (use zero_step_shard_ex)");
        return zero_step_shard_ex(ctx, hp, state, grads, owner_lo, owner_hi, nullptr, nullptr, partial, stream);
    });
}

extern "C" zero_status zero_step_commit(zero_ctx_t* ctx, const double* reduced, void* stream) {
    return zb_guarded("zero_step_commit", [&]() -> zero_status {
        const char* where = "zero_step_commit";
        if (!ctx || !reduced) return zb_fail(ZERO_ERR_INVALID_ARG, "zero_step_commit: NULL argument");
        zero_status s = check_device(ctx, where);
        if (s != ZERO_OK) return s;
        if (!aligned(reduced, 8)) return zb_fail(ZERO_ERR_ALIGN, "zero_step_commit: reduced not 8-byte aligned");
        zb::StepParams sp;
        sp.R = ctx->R;
        sp.mode = ctx->cfg.mode;
        sp.pingpong = ctx->shard_pingpong;
        sp.interval = ctx->cfg.growth_interval;
        sp.growth = ctx->cfg.growth_factor;
        sp.backoff = ctx->cfg.backoff_factor;
        sp.min_scale = ctx->cfg.min_scale;
        sp.st = ctx->st;
        ZbTraceScope trace(ctx, ZERO_TRACE_COMMIT, static_cast<cudaStream_t>(stream), -1);
        cudaError_t e = zb::launch_fsm_commit(sp, reduced, static_cast<cudaStream_t>(stream));
        if (e != cudaSuccess) return cuda_fail(where, e);
        return ZERO_OK;
    });
}

extern "C" zero_status zero_gather_layer(zero_ctx_t* ctx, int64_t layer, const zero_state* state,
                                         void* out, void* stream) {
    return zb_guarded("zero_gather_layer", [&]() -> zero_status {
        const char* where = "zero_gather_layer";
        if (!ctx) return zb_fail(ZERO_ERR_INVALID_ARG, "zero_gather_layer: ctx is NULL");
        zero_status s = check_device(ctx, where);
        if (s != ZERO_OK) return s;
        if (layer < 0 || layer >= static_cast<int64_t>(ctx->layer_lo.size()))
            return zb_fail(ZERO_ERR_RANGE, "zero_gather_layer: layer index out of range");
        if (!out) return zb_fail(ZERO_ERR_INVALID_ARG, "zero_gather_layer: out is NULL");
        if (!aligned(out, 16)) return zb_fail(ZERO_ERR_ALIGN, "zero_gather_layer: out is not 16-byte aligned");
        int sets = 1;
        if ((s = check_state(ctx, state, where, &sets, true)) != ZERO_OK) return s;
        if (sets == 1 && ctx->two_sets)
            return zb_fail(ZERO_ERR_STATE,
                           "zero_gather_layer: the current parameters may live in set 1; pass param[1]");
        zb::RankPtrs p;
        for (int r = 0; r < ctx->R; ++r) {
            p.param[0][r] = state->param[0][r];
            p.param[1][r] = sets == 2 ? state->param[1][r] : state->param[0][r];
        }
        ZbTraceScope trace(ctx, ZERO_TRACE_GATHER, static_cast<cudaStream_t>(stream), layer);
        cudaError_t e = zb::launch_gather(ctx->R, ctx->S, ctx->layer_lo[layer], ctx->layer_hi[layer],
                                          ctx->st, p, out, static_cast<cudaStream_t>(stream));
        if (e != cudaSuccess) return cuda_fail(where, e);
        return ZERO_OK;
    });
}

extern "C" zero_status zero_gather_layers(zero_ctx_t* ctx, int64_t first, int64_t count,
                                          const zero_state* state, void* const* outs,
                                          void* stream) {
    return zb_guarded("zero_gather_layers", [&]() -> zero_status {
        const char* where = "zero_gather_layers";
        if (!ctx) return zb_fail(ZERO_ERR_INVALID_ARG, "zero_gather_layers: ctx is NULL");
        zero_status s = check_device(ctx, where);
        if (s != ZERO_OK) return s;
        const int64_t nl = static_cast<int64_t>(ctx->layer_lo.size());
        if (count < 1 || count > ZERO_GATHER_MAX_LAYERS || first < 0 || first >= nl || count > nl - first)
            return zb_fail(ZERO_ERR_RANGE, "zero_gather_layers: need 0 <= first, 1 <= count <= 64 and "
                                           "first + count <= n_layers");
        if (!outs) return zb_fail(ZERO_ERR_INVALID_ARG, "zero_gather_layers: outs is NULL");
        for (int64_t i = 0; i < count; ++i) {
            if (!outs[i])
                return zb_fail(ZERO_ERR_INVALID_ARG, "zero_gather_layers: outs[" + std::to_string(i) + "] is NULL");
            if (!aligned(outs[i], 16))
                return zb_fail(ZERO_ERR_ALIGN, "zero_gather_layers: outs[" + std::to_string(i) +
                                                   "] is not 16-byte aligned");
        }
        int sets = 1;
        if ((s = check_state(ctx, state, where, &sets, true)) != ZERO_OK) return s;
        if (sets == 1 && ctx->two_sets)
            return zb_fail(ZERO_ERR_STATE,
                           "zero_gather_layers: the current parameters may live in set 1; pass param[1]");
        zb::RankPtrs p;
        for (int r = 0; r < ctx->R; ++r) {
            p.param[0][r] = state->param[0][r];
            p.param[1][r] = sets == 2 ? state->param[1][r] : state->param[0][r];
        }
        ZbTraceScope trace(ctx, ZERO_TRACE_GATHER, static_cast<cudaStream_t>(stream), first);
        cudaError_t e = zb::launch_gather_many(ctx->R, ctx->S, static_cast<int>(count),
                                               ctx->layer_lo.data() + first, ctx->layer_hi.data() + first,
                                               ctx->st, p, outs, static_cast<cudaStream_t>(stream));
        if (e != cudaSuccess) return cuda_fail(where, e);
        return ZERO_OK;
    });
}

extern "C" zero_status zero_loss_scale(zero_ctx_t* ctx, zero_loss_scale_state* inout, int32_t op,
                                       void* stream) {
    return zb_guarded("zero_loss_scale", [&]() -> zero_status {
        const char* where = "zero_loss_scale";
        if (!ctx || !inout) return zb_fail(ZERO_ERR_INVALID_ARG, "zero_loss_scale: NULL argument");
        zero_status s = check_device(ctx, where);
        if (s != ZERO_OK) return s;
        cudaStream_t cs = static_cast<cudaStream_t>(stream);
        zb::DevState d{};
        if (op == ZERO_LOSS_SCALE_GET) {
            cudaError_t e = cudaMemcpyAsync(&d, ctx->st, sizeof(d), cudaMemcpyDeviceToHost, cs);
            if (e == cudaSuccess) e = cudaStreamSynchronize(cs);
            if (e != cudaSuccess) return cuda_fail(where, e);
            if (d.err == 2)
                return zb_fail(ZERO_ERR_TIMEOUT, "zero_loss_scale: a step kernel gave up waiting for its "
                                                 "tile copies (2 s); the step's results are incomplete");
            if (d.err != 0)
                return zb_fail(ZERO_ERR_STATE, "zero_loss_scale: device reported an inconsistent step "
                                               "counter (power table behind t)");
            inout->scale = d.scale;
            inout->cur = d.cur;
            inout->good = d.good;
            inout->t = d.t;
            inout->last_overflow = d.last_overflow;
            inout->last_skipped = d.last_skipped;
            inout->grad_norm_sq = d.grad_norm_sq;
            ctx->t_bound = d.t;
            return ZERO_OK;
        }
        if (op != ZERO_LOSS_SCALE_SET)
            return zb_fail(ZERO_ERR_INVALID_ARG, "zero_loss_scale: op must be GET or SET");
        if ((inout->cur != 0 && inout->cur != 1) || !(inout->scale > 0.0f) ||
            !std::isfinite(inout->scale) || inout->t < 0 || inout->good < 0)
            return zb_fail(ZERO_ERR_INVALID_ARG,
                           "zero_loss_scale: need cur in {0,1}, finite scale > 0, t >= 0, good >= 0");
        d.scale = ctx->cfg.mode == ZERO_SCALE_NONE ? 1.0f : inout->scale;
        d.cur = inout->cur;
        d.good = inout->good;
        d.t = inout->t;
        d.last_overflow = inout->last_overflow;
        d.last_skipped = inout->last_skipped;
        d.grad_norm_sq = inout->grad_norm_sq;
        cudaError_t e = cudaMemcpyAsync(ctx->st, &d, sizeof(d), cudaMemcpyHostToDevice, cs);
        if (e == cudaSuccess) e = cudaStreamSynchronize(cs);
        if (e != cudaSuccess) return cuda_fail(where, e);
        ctx->t_bound = inout->t;
        if (inout->cur == 1) ctx->two_sets = true;
        return ZERO_OK;
    });
}

extern "C" zero_status zero_sync(zero_ctx_t* ctx, void* stream) {
    return zb_guarded("zero_sync", [&]() -> zero_status {
        if (!ctx) return zb_fail(ZERO_ERR_INVALID_ARG, "zero_sync: ctx is NULL");
        cudaError_t e = cudaStreamSynchronize(static_cast<cudaStream_t>(stream));
        if (e == cudaSuccess) e = cudaGetLastError();
        if (e != cudaSuccess) return cuda_fail("zero_sync", e);
        return ZERO_OK;
    });
}

extern "C" size_t zero_last_error(char* buf, size_t n) {
    if (buf && n > 0) {
        const size_t k = g_last_error.size() < n - 1 ? g_last_error.size() : n - 1;
        std::memcpy(buf, g_last_error.data(), k);
        buf[k] = '\0';
    }
    return g_last_error.size();
}

extern "C" const char* zero_version(void) { return "zero_b200 0.1.0 (sm_100a)"; }
