// Per-call tracing: each traced call of a context brackets the work it queues
// on its stream with two timing events, so a caller can read back how long
// every reduce-scatter, step and gather took on the device, in call order,
// without a profiler. Off by default; while it is off a call pays one pointer
// test. Calls made while their stream is being captured into a CUDA graph are
// not traced (a graph replays without the host, so there is nothing to pair
// the events with).
#include <memory>
#include <string>
#include <vector>

#include "internal.h"

struct zero_trace {
    int32_t capacity = 0;
    std::vector<cudaEvent_t> ev;  // 2 per record: start, end
    std::vector<zero_trace_record> rec;
    int64_t dropped = 0;
};

namespace {

void free_trace(zero_trace* t) {
    for (cudaEvent_t e : t->ev)
        if (e) cudaEventDestroy(e);
    delete t;
}

}  // namespace

void zb_trace_destroy(zero_ctx_t* ctx) {
    if (ctx->trace) free_trace(ctx->trace);
    ctx->trace = nullptr;
}

ZbTraceScope::ZbTraceScope(zero_ctx_t* ctx, int32_t call, cudaStream_t s, int64_t arg)
    : t_(ctx ? ctx->trace : nullptr), s_(s), slot_(-1) {
    if (!t_) return;
    cudaStreamCaptureStatus cap = cudaStreamCaptureStatusNone;
    if (cudaStreamIsCapturing(s, &cap) != cudaSuccess) {
        cudaGetLastError();
        t_ = nullptr;
        return;
    }
    if (cap != cudaStreamCaptureStatusNone) {
        t_ = nullptr;
        return;
    }
    if (static_cast<int32_t>(t_->rec.size()) >= t_->capacity) {
        t_->dropped += 1;
        t_ = nullptr;
        return;
    }
    slot_ = static_cast<int32_t>(t_->rec.size());
    zero_trace_record r{};
    r.call = call;
    r.arg = arg;
    r.ms = -1.0f;
    t_->rec.push_back(r);
    if (cudaEventRecord(t_->ev[2 * slot_], s) != cudaSuccess) {
        cudaGetLastError();
        t_->rec.pop_back();
        t_ = nullptr;
    }
}

ZbTraceScope::~ZbTraceScope() {
    if (!t_) return;
    if (cudaEventRecord(t_->ev[2 * slot_ + 1], s_) != cudaSuccess) {
        cudaGetLastError();
        t_->rec[slot_].call = 0;  // no end event: reported as untimed
    }
}

extern "C" zero_status zero_trace_start(zero_ctx_t* ctx, int32_t capacity) {
    return zb_guarded("zero_trace_start", [&]() -> zero_status {
        if (!ctx) return zb_fail(ZERO_ERR_INVALID_ARG, "zero_trace_start: ctx is NULL");
        if (capacity < 1 || capacity > (1 << 20))
            return zb_fail(ZERO_ERR_INVALID_ARG, "zero_trace_start: need 1 <= capacity <= 2^20");
        int dev = -1;
        if (cudaGetDevice(&dev) != cudaSuccess || dev != ctx->device) {
            cudaGetLastError();
            return zb_fail(ZERO_ERR_INVALID_ARG, "zero_trace_start: context belongs to another device");
        }
        zb_trace_destroy(ctx);
        std::unique_ptr<zero_trace, void (*)(zero_trace*)> t(new zero_trace(), free_trace);
        t->capacity = capacity;
        t->ev.assign(2 * static_cast<size_t>(capacity), nullptr);
        t->rec.reserve(capacity);
        for (cudaEvent_t& e : t->ev) {
            cudaError_t err = cudaEventCreate(&e);
            if (err != cudaSuccess) {
                cudaGetLastError();
                return zb_fail(ZERO_ERR_CUDA, std::string("zero_trace_start: ") + cudaGetErrorString(err));
            }
        }
        ctx->trace = t.release();
        return ZERO_OK;
    });
}

extern "C" zero_status zero_trace_read(zero_ctx_t* ctx, zero_trace_record* out, int32_t max, int32_t* count,
                                       int64_t* dropped) {
    return zb_guarded("zero_trace_read", [&]() -> zero_status {
        if (!ctx || !count || (max > 0 && !out))
            return zb_fail(ZERO_ERR_INVALID_ARG, "zero_trace_read: NULL argument");
        zero_trace* t = ctx->trace;
        if (!t) return zb_fail(ZERO_ERR_STATE, "zero_trace_read: tracing is not started");
        const int32_t n = static_cast<int32_t>(t->rec.size());
        if (max < n)
            return zb_fail(ZERO_ERR_RANGE, "zero_trace_read: " + std::to_string(n) + " records, room for " +
                                               std::to_string(max));
        for (int32_t i = 0; i < n; ++i) {
            zero_trace_record r = t->rec[i];
            if (r.call != 0) {
                cudaError_t e = cudaEventSynchronize(t->ev[2 * i + 1]);
                float ms = -1.0f;
                if (e == cudaSuccess) e = cudaEventElapsedTime(&ms, t->ev[2 * i], t->ev[2 * i + 1]);
                if (e != cudaSuccess) {
                    cudaGetLastError();
                    return zb_fail(ZERO_ERR_CUDA, std::string("zero_trace_read: ") + cudaGetErrorString(e));
                }
                r.ms = ms;
            }
            out[i] = r;
        }
        *count = n;
        if (dropped) *dropped = t->dropped;
        t->rec.clear();
        t->dropped = 0;
        return ZERO_OK;
    });
}

extern "C" zero_status zero_trace_stop(zero_ctx_t* ctx) {
    return zb_guarded("zero_trace_stop", [&]() -> zero_status {
        if (!ctx) return zb_fail(ZERO_ERR_INVALID_ARG, "zero_trace_stop: ctx is NULL");
        if (ctx->trace) {
            // events still queued must complete before they are destroyed
            for (size_t i = 0; i < ctx->trace->rec.size(); ++i) cudaEventSynchronize(ctx->trace->ev[2 * i + 1]);
            cudaGetLastError();
        }
        zb_trace_destroy(ctx);
        return ZERO_OK;
    });
}
