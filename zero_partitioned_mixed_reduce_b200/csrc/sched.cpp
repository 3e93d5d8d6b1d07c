// Overlap and prefetch scheduling on a context-owned communication stream.
//
// Gradient reduction overlapped with backward (inferensys legal pre-training
// glossary, "Communication Overlap": as soon as a layer's gradients exist,
// their reduction starts; genomic glossary, "Reduce-Scatter Overlap"): the
// caller reports tensors whose gradients are written; a bucket is
// reduce-scattered on the communication stream as soon as all of its tensors
// are reported, ordered after the caller's work by an event, while the
// caller's stream goes on with the next layer.
//
// ZeRO-3 look-ahead gathering (legal glossary, ZeRO-3 "Prefetching
// Scheduler"; genomic glossary, "Bucketed All-Gather" / "Prefetch
// Scheduling"): layers are gathered into a ring of caller buffers on the
// communication stream, `depth` layers ahead of the one in use; a slot is
// refilled only after the caller released the layer it held.
#include <algorithm>
#include <string>
#include <vector>

#include "internal.h"

struct zero_sched {
    cudaStream_t comm = nullptr;
    int comm_sms = 0;  // SMs the communication stream's kernels may fill (0 = all)
    // gradient readiness, per step (or micro-batch)
    std::vector<uint8_t> tensor_ready;
    std::vector<int64_t> bucket_ready;
    std::vector<cudaEvent_t> bucket_event;
    int64_t buckets_issued = 0;
    cudaEvent_t join_event = nullptr;
    // look-ahead gathering
    bool pf_active = false;
    int nbufs = 0, depth = 0, dir = 1;
    std::vector<void*> bufs;
    zb::RankPtrs params{};
    std::vector<cudaEvent_t> slot_ready, slot_free;
    std::vector<int64_t> slot_pos;         // sequence position held by each slot (-1: none)
    std::vector<uint8_t> slot_released;    // the held position has been released
    int64_t next_issue = 0;                // next sequence position to gather
    cudaEvent_t begin_event = nullptr;
};

namespace {

zero_status cuda_err(const char* where, cudaError_t e) {
    cudaGetLastError();
    return zb_fail(ZERO_ERR_CUDA, std::string(where) + ": " + cudaGetErrorString(e));
}

zero_status ensure_sched(zero_ctx_t* ctx, const char* where) {
    int dev = -1;
    cudaError_t e = cudaGetDevice(&dev);
    if (e != cudaSuccess) return cuda_err(where, e);
    if (dev != ctx->device)
        return zb_fail(ZERO_ERR_INVALID_ARG, std::string(where) + ": context belongs to another device");
    if (ctx->sched) return ZERO_OK;
    zero_sched* s = new zero_sched();
    int lo = 0, hi = 0;
    cudaDeviceGetStreamPriorityRange(&lo, &hi);
    // the communication stream gets the highest priority so that its short,
    // bandwidth-bound kernels start as soon as their inputs are ready
    e = cudaStreamCreateWithPriority(&s->comm, cudaStreamNonBlocking, hi);
    const size_t nb = ctx->bucket_lo.size();
    s->tensor_ready.assign(ctx->tensor_bucket.size(), 0);
    s->bucket_ready.assign(nb, 0);
    s->bucket_event.assign(nb, nullptr);
    for (size_t b = 0; e == cudaSuccess && b < nb; ++b)
        e = cudaEventCreateWithFlags(&s->bucket_event[b], cudaEventDisableTiming);
    if (e == cudaSuccess) e = cudaEventCreateWithFlags(&s->join_event, cudaEventDisableTiming);
    if (e == cudaSuccess) e = cudaEventCreateWithFlags(&s->begin_event, cudaEventDisableTiming);
    ctx->sched = s;  // destroyed with the context even if creation failed half-way
    if (e != cudaSuccess) return cuda_err(where, e);
    return ZERO_OK;
}

}  // namespace

void zb_sched_destroy(zero_ctx_t* ctx) {
    zero_sched* s = ctx->sched;
    if (!s) return;
    for (cudaEvent_t ev : s->bucket_event)
        if (ev) cudaEventDestroy(ev);
    for (cudaEvent_t ev : s->slot_ready)
        if (ev) cudaEventDestroy(ev);
    for (cudaEvent_t ev : s->slot_free)
        if (ev) cudaEventDestroy(ev);
    if (s->join_event) cudaEventDestroy(s->join_event);
    if (s->begin_event) cudaEventDestroy(s->begin_event);
    if (s->comm) cudaStreamDestroy(s->comm);
    delete s;
    ctx->sched = nullptr;
}

extern "C" zero_status zero_sched_set_comm_sms(zero_ctx_t* ctx, int32_t sms) {
    return zb_guarded("zero_sched_set_comm_sms", [&]() -> zero_status {
        const char* where = "zero_sched_set_comm_sms";
        if (!ctx) return zb_fail(ZERO_ERR_INVALID_ARG, "zero_sched_set_comm_sms: ctx is NULL");
        if (sms < 0) return zb_fail(ZERO_ERR_INVALID_ARG, "zero_sched_set_comm_sms: need sms >= 0");
        zero_status st = ensure_sched(ctx, where);
        if (st != ZERO_OK) return st;
        ctx->sched->comm_sms = sms;
        return ZERO_OK;
    });
}

extern "C" zero_status zero_grads_ready(zero_ctx_t* ctx, int64_t first, int64_t count,
                                        const void* const* grads, float* const* acc, int32_t flags,
                                        void* stream) {
    return zb_guarded("zero_grads_ready", [&]() -> zero_status {
        const char* where = "zero_grads_ready";
        if (!ctx) return zb_fail(ZERO_ERR_INVALID_ARG, "zero_grads_ready: ctx is NULL");
        zero_status st = ensure_sched(ctx, where);
        if (st != ZERO_OK) return st;
        const int64_t n = static_cast<int64_t>(ctx->tensor_bucket.size());
        if (first < 0 || count < 1 || first > n - count)
            return zb_fail(ZERO_ERR_RANGE, "zero_grads_ready: tensor range out of bounds");
        if (flags & ~(ZERO_RS_ACCUMULATE | ZERO_RS_NORM))
            return zb_fail(ZERO_ERR_INVALID_ARG, "zero_grads_ready: unknown flags");
        if (!grads || !acc) return zb_fail(ZERO_ERR_INVALID_ARG, "zero_grads_ready: NULL grads or acc");
        for (int r = 0; r < ctx->R; ++r) {
            if (!grads[r] || !acc[r]) return zb_fail(ZERO_ERR_INVALID_ARG, "zero_grads_ready: NULL rank pointer");
            if (reinterpret_cast<uintptr_t>(grads[r]) % 16 || reinterpret_cast<uintptr_t>(acc[r]) % 32)
                return zb_fail(ZERO_ERR_ALIGN, "zero_grads_ready: misaligned rank pointer");
        }
        zero_sched* s = ctx->sched;
        for (int64_t k = first; k < first + count; ++k)
            if (s->tensor_ready[k])
                return zb_fail(ZERO_ERR_STATE, "zero_grads_ready: tensor " + std::to_string(k) +
                                                   " was already reported since the last join");
        zb::RankPtrs p;
        for (int r = 0; r < ctx->R; ++r) {
            p.g[r] = grads[r];
            p.acc[r] = acc[r];
        }
        cudaStream_t cs = static_cast<cudaStream_t>(stream);
        // the buckets this call completes, in ascending order
        std::vector<int64_t> done;
        for (int64_t k = first; k < first + count; ++k) {
            s->tensor_ready[k] = 1;
            const int64_t b = ctx->tensor_bucket[k];
            if (++s->bucket_ready[b] == ctx->bucket_ntensors[b]) done.push_back(b);
        }
        std::sort(done.begin(), done.end());
        const int64_t nb = static_cast<int64_t>(ctx->bucket_lo.size());
        // each run of consecutive buckets is one contiguous flat range: one
        // launch behind the caller's work so far
        for (size_t i = 0; i < done.size();) {
            size_t j = i + 1;
            while (j < done.size() && done[j] == done[j - 1] + 1) ++j;
            const int64_t b0 = done[i], cnt = static_cast<int64_t>(j - i);
            // the step's last buckets have no compute left to hide behind: whole GPU
            const bool last = s->buckets_issued + cnt == nb;
            cudaError_t e = cudaEventRecord(s->bucket_event[b0], cs);
            if (e == cudaSuccess) e = cudaStreamWaitEvent(s->comm, s->bucket_event[b0], 0);
            if (e == cudaSuccess) e = zb_rs_launch(ctx, b0, cnt, p, s->comm, flags, last ? 0 : s->comm_sms);
            if (e != cudaSuccess) return cuda_err(where, e);
            s->buckets_issued += cnt;
            i = j;
        }
        return ZERO_OK;
    });
}

extern "C" zero_status zero_grads_join(zero_ctx_t* ctx, void* stream) {
    return zb_guarded("zero_grads_join", [&]() -> zero_status {
        const char* where = "zero_grads_join";
        if (!ctx) return zb_fail(ZERO_ERR_INVALID_ARG, "zero_grads_join: ctx is NULL");
        zero_status st = ensure_sched(ctx, where);
        if (st != ZERO_OK) return st;
        zero_sched* s = ctx->sched;
        if (s->buckets_issued != static_cast<int64_t>(ctx->bucket_lo.size()))
            return zb_fail(ZERO_ERR_STATE, "zero_grads_join: " +
                                               std::to_string(static_cast<int64_t>(ctx->bucket_lo.size()) -
                                                              s->buckets_issued) +
                                               " bucket(s) still have tensors not reported ready");
        cudaError_t e = cudaEventRecord(s->join_event, s->comm);
        if (e == cudaSuccess) e = cudaStreamWaitEvent(static_cast<cudaStream_t>(stream), s->join_event, 0);
        if (e != cudaSuccess) return cuda_err(where, e);
        std::fill(s->tensor_ready.begin(), s->tensor_ready.end(), 0);
        std::fill(s->bucket_ready.begin(), s->bucket_ready.end(), 0);
        s->buckets_issued = 0;
        return ZERO_OK;
    });
}

extern "C" zero_status zero_prefetch_begin(zero_ctx_t* ctx, const zero_state* state, void* const* bufs,
                                           int32_t nbufs, int32_t depth, int32_t direction, void* stream) {
    return zb_guarded("zero_prefetch_begin", [&]() -> zero_status {
        const char* where = "zero_prefetch_begin";
        if (!ctx || !state || !bufs) return zb_fail(ZERO_ERR_INVALID_ARG, "zero_prefetch_begin: NULL argument");
        zero_status st = ensure_sched(ctx, where);
        if (st != ZERO_OK) return st;
        if (nbufs < 1 || nbufs > 64 || depth < 0 || depth >= nbufs || (direction != 1 && direction != -1))
            return zb_fail(ZERO_ERR_INVALID_ARG,
                           "zero_prefetch_begin: need 1 <= nbufs <= 64, 0 <= depth < nbufs, direction +1 or -1");
        for (int i = 0; i < nbufs; ++i) {
            if (!bufs[i]) return zb_fail(ZERO_ERR_INVALID_ARG, "zero_prefetch_begin: NULL buffer");
            if (reinterpret_cast<uintptr_t>(bufs[i]) % 16)
                return zb_fail(ZERO_ERR_ALIGN, "zero_prefetch_begin: buffer not 16-byte aligned");
        }
        if (!state->param[0]) return zb_fail(ZERO_ERR_INVALID_ARG, "zero_prefetch_begin: param[0] is NULL");
        const bool two = state->param[1] != nullptr;
        if (!two && ctx->two_sets)
            return zb_fail(ZERO_ERR_STATE, "zero_prefetch_begin: the current parameters may live in set 1");
        zero_sched* s = ctx->sched;
        for (int r = 0; r < ctx->R; ++r) {
            if (!state->param[0][r] || (two && !state->param[1][r]))
                return zb_fail(ZERO_ERR_INVALID_ARG, "zero_prefetch_begin: NULL param pointer");
            s->params.param[0][r] = state->param[0][r];
            s->params.param[1][r] = two ? state->param[1][r] : state->param[0][r];
        }
        // fresh ring
        for (cudaEvent_t ev : s->slot_ready) cudaEventDestroy(ev);
        for (cudaEvent_t ev : s->slot_free) cudaEventDestroy(ev);
        s->slot_ready.assign(nbufs, nullptr);
        s->slot_free.assign(nbufs, nullptr);
        cudaError_t e = cudaSuccess;
        for (int i = 0; e == cudaSuccess && i < nbufs; ++i) {
            e = cudaEventCreateWithFlags(&s->slot_ready[i], cudaEventDisableTiming);
            if (e == cudaSuccess) e = cudaEventCreateWithFlags(&s->slot_free[i], cudaEventDisableTiming);
        }
        if (e != cudaSuccess) return cuda_err(where, e);
        s->bufs.assign(bufs, bufs + nbufs);
        s->nbufs = nbufs;
        s->depth = depth;
        s->dir = direction;
        s->slot_pos.assign(nbufs, -1);
        s->slot_released.assign(nbufs, 1);
        s->next_issue = 0;
        s->pf_active = true;
        // every gather of this pass comes after the work already queued on `stream`
        // (for example the optimizer step that produced the parameters)
        e = cudaEventRecord(s->begin_event, static_cast<cudaStream_t>(stream));
        if (e == cudaSuccess) e = cudaStreamWaitEvent(s->comm, s->begin_event, 0);
        if (e != cudaSuccess) return cuda_err(where, e);
        return ZERO_OK;
    });
}

namespace {

// Gather sequence positions up to `upto` whose slots are free.
zero_status issue_upto(zero_ctx_t* ctx, int64_t upto) {
    zero_sched* s = ctx->sched;
    const int64_t nl = static_cast<int64_t>(ctx->layer_lo.size());
    if (upto > nl - 1) upto = nl - 1;
    while (s->next_issue <= upto) {
        const int64_t pos = s->next_issue;
        const int slot = static_cast<int>(pos % s->nbufs);
        if (!s->slot_released[slot]) break;  // still in use by an unreleased layer
        cudaError_t e = cudaSuccess;
        if (s->slot_pos[slot] >= 0) e = cudaStreamWaitEvent(s->comm, s->slot_free[slot], 0);
        const int64_t layer = s->dir > 0 ? pos : nl - 1 - pos;
        void* out = s->bufs[slot];
        if (e == cudaSuccess) {
            ZbTraceScope trace(ctx, ZERO_TRACE_GATHER, s->comm, layer);
            // the pass's first gather has nothing before it to hide behind: whole GPU
            e = zb::launch_gather_many(ctx->R, ctx->S, 1, &ctx->layer_lo[layer], &ctx->layer_hi[layer], ctx->st,
                                       s->params, &out, s->comm, pos == 0 ? 0 : s->comm_sms);
        }
        if (e == cudaSuccess) e = cudaEventRecord(s->slot_ready[slot], s->comm);
        if (e != cudaSuccess) return cuda_err("zero_layer_acquire", e);
        s->slot_pos[slot] = pos;
        s->slot_released[slot] = 0;
        s->next_issue += 1;
    }
    return ZERO_OK;
}

int64_t position_of(const zero_ctx_t* ctx, int64_t layer) {
    const int64_t nl = static_cast<int64_t>(ctx->layer_lo.size());
    return ctx->sched->dir > 0 ? layer : nl - 1 - layer;
}

}  // namespace

extern "C" zero_status zero_layer_acquire(zero_ctx_t* ctx, int64_t layer, void** buf, void* stream) {
    return zb_guarded("zero_layer_acquire", [&]() -> zero_status {
        const char* where = "zero_layer_acquire";
        if (!ctx || !buf) return zb_fail(ZERO_ERR_INVALID_ARG, "zero_layer_acquire: NULL argument");
        zero_status st = ensure_sched(ctx, where);
        if (st != ZERO_OK) return st;
        zero_sched* s = ctx->sched;
        if (!s->pf_active) return zb_fail(ZERO_ERR_STATE, "zero_layer_acquire: call zero_prefetch_begin first");
        const int64_t nl = static_cast<int64_t>(ctx->layer_lo.size());
        if (layer < 0 || layer >= nl) return zb_fail(ZERO_ERR_RANGE, "zero_layer_acquire: layer out of range");
        const int64_t pos = position_of(ctx, layer);
        if ((st = issue_upto(ctx, pos + s->depth)) != ZERO_OK) return st;
        const int slot = static_cast<int>(pos % s->nbufs);
        if (s->slot_pos[slot] != pos)
            return zb_fail(ZERO_ERR_STATE, "zero_layer_acquire: layer " + std::to_string(layer) +
                                               " is not in the ring (acquire layers in order and release "
                                               "each one after use)");
        cudaError_t e = cudaStreamWaitEvent(static_cast<cudaStream_t>(stream), s->slot_ready[slot], 0);
        if (e != cudaSuccess) return cuda_err(where, e);
        *buf = s->bufs[slot];
        return ZERO_OK;
    });
}

extern "C" zero_status zero_layer_release(zero_ctx_t* ctx, int64_t layer, void* stream) {
    return zb_guarded("zero_layer_release", [&]() -> zero_status {
        const char* where = "zero_layer_release";
        if (!ctx) return zb_fail(ZERO_ERR_INVALID_ARG, "zero_layer_release: ctx is NULL");
        zero_status st = ensure_sched(ctx, where);
        if (st != ZERO_OK) return st;
        zero_sched* s = ctx->sched;
        if (!s->pf_active) return zb_fail(ZERO_ERR_STATE, "zero_layer_release: call zero_prefetch_begin first");
        const int64_t nl = static_cast<int64_t>(ctx->layer_lo.size());
        if (layer < 0 || layer >= nl) return zb_fail(ZERO_ERR_RANGE, "zero_layer_release: layer out of range");
        const int64_t pos = position_of(ctx, layer);
        const int slot = static_cast<int>(pos % s->nbufs);
        if (s->slot_pos[slot] != pos || s->slot_released[slot])
            return zb_fail(ZERO_ERR_STATE, "zero_layer_release: layer " + std::to_string(layer) + " is not held");
        cudaError_t e = cudaEventRecord(s->slot_free[slot], static_cast<cudaStream_t>(stream));
        if (e != cudaSuccess) return cuda_err(where, e);
        s->slot_released[slot] = 1;
        // the freed slot can take the next layer of the look-ahead window
        return issue_upto(ctx, pos + s->depth + 1);
    });
}
