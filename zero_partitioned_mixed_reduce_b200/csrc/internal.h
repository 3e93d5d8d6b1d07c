// Internal declarations shared by the host C++ (plan, C ABI) and the CUDA
// kernels of libzero_b200.so. Not installed; the public ABI is
// include/zero_b200.h.
#pragma once

#include <cstdint>
#include <string>
#include <vector>

#include <cuda_runtime.h>

#include "zero_b200.h"

struct zero_plan_s {
    int32_t R = 0, dtype = 0, align = 0;
    int64_t bucket_elems = 0;
    int64_t P = 0, L = 0, S = 0, T = 0;
    std::vector<int64_t> numel, offset, tensor_bucket, tensor_layer;
    std::vector<int64_t> bucket_lo, bucket_hi;
    std::vector<int64_t> layer_lo, layer_hi;
};

namespace zb {

// The staged fused step's tile: each shard is cut into tiles of this many
// elements (the last tile of a shard shorter), in 64-bit arithmetic.
constexpr int64_t kStagedTile = 4096;
inline int64_t staged_tiles_per_shard(int64_t S) { return (S + kStagedTile - 1) / kStagedTile; }

// Device-resident loss-scale / step state. One per context, in the
// context's device scratch. Written by the last block of every step kernel.
struct alignas(64) DevState {
    float scale;
    int32_t cur;
    int64_t good;
    int64_t t;
    int32_t last_overflow;
    int32_t last_skipped;
    double grad_norm_sq;
    uint32_t flag;  // OR of "some reduced gradient is inf/NaN" for the step in progress
    uint32_t done;  // blocks of the running step kernel that have finished
    int32_t err;    // device-side consistency error (0 = none)
    float clip;     // clipping coefficient of the step in progress
};

// Everything a step kernel needs besides the rank pointers. Filled on the host.
struct StepParams {
    int32_t R = 0, dtype = 0, mode = 0, pingpong = 0;
    uint32_t S8 = 0, T8 = 0;  // shard and total length in 8-element vectors
    float dec = 0, b1f = 0, omb1 = 0, b2f = 0, omb2 = 0, epsf = 0;
    double lr = 0;
    double divisor = 1;       // grad divisor k: unscale by 1 / ((R * k) * scale)
    double max_norm = 0;      // > 0: clipping on
    int32_t clip = 0;
    int32_t add_acc = 0;      // fused step adds the accumulators (ZERO_STEP_ADD_ACC)
    int64_t interval = 1;
    float growth = 2, backoff = 0.5f, min_scale = 1;
    DevState* st = nullptr;
    double* partials = nullptr;
    const double2* powtab = nullptr;  // powtab[t] = (beta1^t, beta2^t)
    int64_t powtab_len = 0;
    int grid_cap = 0;  // capacity of `partials`
    // step or norm pass over shards [obeg, oend) only (default: all R)
    int32_t obeg = 0, oend = 0;
    // non-null: the step's last block writes {sum of g^2, overflow 0/1} here and
    // leaves the loss-scale update to a later commit (sharded multi-rank step)
    double* partial_out = nullptr;
    // test support (zero_test_drop_tile): the staged kernel issues no copy
    // for this tile, so the block waiting for it gives up after its limit
    uint32_t drop_tile = 0xffffffffu;
    // the step also writes each updated parameter vector into every rank's
    // full-model buffer RankPtrs::full[dst][r] (ZERO_STEP_PUSH_PARAMS)
    int32_t push = 0;
};

// Rank pointer tables, sized for the largest R.
struct RankPtrs {
    const void* g[ZERO_MAX_RANKS];
    float* acc[ZERO_MAX_RANKS];
    float* master[2][ZERO_MAX_RANKS];
    float* m[2][ZERO_MAX_RANKS];
    float* v[2][ZERO_MAX_RANKS];
    void* param[2][ZERO_MAX_RANKS];
    void* full[2][ZERO_MAX_RANKS];  // full-model parameter buffers of the push
};

// A reduce-scatter's share of the clipping norm (ZERO_RS_NORM): the launch
// adds up sum((float)(acc * inv))^2 over the accumulator values it writes,
// inv = 1 / ((R * divisor) * scale), one partial per block in `partials`
// (grid capacity entries), the last block storing the total in *out.
struct RsNorm {
    double* partials = nullptr;
    uint32_t* done = nullptr;
    double* out = nullptr;
    uint32_t cap = 0;      // entries of `partials`
    int32_t mode = 0;
    double divisor = 1.0;
};

// Kernel launchers (kernels.cu). Each returns the launch's cudaError_t.
cudaError_t launch_fused_step(const StepParams& sp, const RankPtrs& p, cudaStream_t s);
cudaError_t launch_step_from_acc(const StepParams& sp, const RankPtrs& p, cudaStream_t s);
// max_sms > 0 caps the grid at that many SMs' worth of resident blocks (the
// communication stream's kernels, so that they leave the rest of the GPU to
// concurrent compute); 0 = the whole GPU.
cudaError_t launch_reduce_scatter(int32_t R, int32_t dtype, int64_t S, int64_t lo, int64_t hi,
                                  DevState* st, const RankPtrs& p, cudaStream_t s,
                                  bool accumulate = false, int max_sms = 0, const RsNorm* norm = nullptr);
// A sharded rank's norm part from norm slots [first, first + count) into
// out[0] (out[1] = 0) (norm_slots.cu).
cudaError_t launch_sum_norm_slots(const double* slots, int64_t first, int64_t count, double* out,
                                  cudaStream_t s);
// *out = the reduce-scatters' overflow flag (0/1), which is cleared (norm_slots.cu).
cudaError_t launch_take_overflow(DevState* st, int32_t* out, cudaStream_t s);
// The clipping coefficient from norm slots [first, first + count).
cudaError_t launch_clip_from_rs_norm(const StepParams& sp, const double* slots, int64_t first, int64_t count,
                                     cudaStream_t s);
// Norm passes over owners [obeg, oend): the last block stores the clipping
// coefficient, or, with partial_out, the range's sum of g^2 in partial_out[0].
cudaError_t launch_grad_norm(const StepParams& sp, const RankPtrs& p, cudaStream_t s);
cudaError_t launch_clip_from_norm(const StepParams& sp, const double* norm_sq, cudaStream_t s);
cudaError_t launch_clip_norm(const StepParams& sp, const RankPtrs& p, cudaStream_t s);
// Loss-scale update from globally reduced totals {sum of g^2, overflow count}.
cudaError_t launch_fsm_commit(const StepParams& sp, const double* reduced, cudaStream_t s);
cudaError_t launch_gather(int32_t R, int64_t S, int64_t lo, int64_t hi, const DevState* st,
                          const RankPtrs& p, void* out, cudaStream_t s);

cudaError_t launch_gather_many(int32_t R, int64_t S, int nl, const int64_t* lo, const int64_t* hi,
                               const DevState* st, const RankPtrs& p, void* const* outs,
                               cudaStream_t s, int max_sms = 0);

// Grid the step kernels use for a given problem (for sizing `partials`).
int step_grid_cap(int device);

#ifdef ZERO_DEBUG_BOUNDS
// The bounds record of the static-scratch step's module (noalloc.cu), zero
// when that step never ran in this process; optionally cleared.
cudaError_t noalloc_bounds_record(unsigned long long* count, unsigned long long* first, bool reset);
#endif

}  // namespace zb

// Context: the plan's layout, the loss-scale config, the device scratch, and
// the overlap / prefetch scheduler (sched.cpp).
struct zero_sched;  // scheduler state, sched.cpp
struct zero_trace;  // per-call trace, trace.cpp

struct zero_ctx_s {
    int device = 0;
    int32_t R = 0, dtype = 0;
    int64_t S = 0, T = 0;
    std::vector<int64_t> bucket_lo, bucket_hi, layer_lo, layer_hi;
    std::vector<int64_t> tensor_bucket;  // bucket of each tensor
    std::vector<int64_t> bucket_ntensors;
    zero_loss_scale_config cfg{};
    zb::DevState* st = nullptr;   // device
    double* partials = nullptr;   // device, grid_cap entries
    int grid_cap = 0;
    uint32_t drop_tile = 0xffffffffu;  // one-shot, for the next fused step
    double2* powtab = nullptr;    // device, powtab_len entries
    std::vector<double2*> powtab_retired;  // outgrown tables, freed with the context
    int64_t powtab_len = 0;
    double pow_b1 = 0.0, pow_b2 = 0.0;
    bool pow_valid = false;
    int64_t t_bound = 0;          // upper bound of the device step count
    bool two_sets = false;        // a ping-pong step has run (or cur was set to 1)
    int32_t shard_pingpong = 0;   // the last zero_step_shard wrote set 1-cur
    zero_sched* sched = nullptr;  // created on first use
    // reduce-scatter norm shares (ZERO_RS_NORM): one slot per bucket, and
    // slot n_buckets for a whole-range call; device partials (grid_cap per
    // slot), counters and totals; on the host, whether each slot holds the
    // norm of the accumulators as they now stand, and its divisor
    double* rs_norm_partials = nullptr;
    uint32_t* rs_norm_done = nullptr;
    double* rs_norm = nullptr;
    std::vector<uint8_t> rs_norm_valid;
    std::vector<double> rs_norm_div;
    std::vector<int64_t> rs_norm_owner;  // owner range of each share: lo << 32 | hi
    double grad_divisor = 1.0;    // the divisor ZERO_RS_NORM unscales by
    std::vector<void*> push_full[2];  // zero_ctx_set_param_push: R buffers per state set (empty: none)
    zero_trace* trace = nullptr;  // per-call trace while started
};

void zb_trace_destroy(zero_ctx_t* ctx);

// Brackets the work a traced call queues on `s` with the trace's two events
// (nothing while the trace is off, the ring is full or `s` is capturing).
class ZbTraceScope {
public:
    ZbTraceScope(zero_ctx_t* ctx, int32_t call, cudaStream_t s, int64_t arg);
    ~ZbTraceScope();
    ZbTraceScope(const ZbTraceScope&) = delete;
    ZbTraceScope& operator=(const ZbTraceScope&) = delete;

private:
    zero_trace* t_;
    cudaStream_t s_;
    int32_t slot_;
};

// Bookkeeping of a reduce-scatter of buckets [first, first + count) (first
// -1: the whole range), with or without its norm share; returns the launch's
// norm arguments for the first bucket's slot (capi.cpp).
zb::RsNorm zb_rs_norm_note(zero_ctx_t* ctx, int64_t first, int64_t count, bool norm, int32_t owner_lo = 0,
                           int32_t owner_hi = -1);
// One reduce-scatter launch over buckets [first, first + count), a
// contiguous flat range (first -1, count 1: every element), flags as for
// zero_reduce_scatter_bucket_ex, grid capped at max_sms SMs (0: all).
cudaError_t zb_rs_launch(zero_ctx_t* ctx, int64_t first, int64_t count, const zb::RankPtrs& p,
                         cudaStream_t s, int32_t flags, int max_sms);

void zb_sched_destroy(zero_ctx_t* ctx);

// Set the calling thread's last error message; returns `code`.
zero_status zb_fail(zero_status code, const std::string& msg) noexcept;

// No exception crosses the C ABI: every entry point runs its body through
// zb_guarded, which turns an exception in flight (host memory or threads
// exhausted) into ZERO_ERR_OOM with the exception's message.
zero_status zb_exception(const char* where) noexcept;
template <typename F>
zero_status zb_guarded(const char* where, F&& body) noexcept {
    try {
        return body();
    } catch (...) {
        return zb_exception(where);
    }
}
