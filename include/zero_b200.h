/*
 * zero_b200.h -- C ABI of libzero_b200.so: the data-parallel hot path of ZeRO
 * (partitioned mixed-precision AdamW over a flat, sharded model state) on one
 * NVIDIA B200 (sm_100a). R data-parallel ranks are simulated as R gradient
 * buffers and R state shards in the HBM of one GPU.
 *
 * Sources are four web pages titled "ZeRO Optimization":
 *   [legal]    inferensys glossary, domain-specific legal pre-training
 *   [instr]    inferensys glossary, instruction-tuning methodologies
 *   [intro]    mbrenndoerfer, "ZeRO Optimization: Optimizer, Gradient, and
 *              Parameter Partitioning", introduction
 *   [genomic]  inferensys glossary, genomic MLOps
 * Each entry point cites the passage that defines its operation.
 *
 * Conventions for every call:
 *  - Every call returns a zero_status; nothing throws across the ABI. On an
 *    error, zero_last_error() gives a message for the calling thread.
 *  - Device pointers are owned by the caller (for example allocated by
 *    PyTorch) and must stay valid until the work enqueued on the stream has
 *    finished. Half buffers (gradients, parameters, gather output) must be
 *    16-byte aligned; fp32 buffers (master, m, v, accumulators) must be
 *    32-byte aligned. A misaligned pointer returns ZERO_ERR_ALIGN and
 *    nothing is launched.
 *  - `stream` is a cudaStream_t passed as void* (NULL = legacy default
 *    stream). Every GPU call is asynchronous on that stream, except where a
 *    call says it synchronizes. A CUDA error raised by earlier asynchronous
 *    work surfaces as ZERO_ERR_CUDA on a later call or on zero_sync.
 *  - A context is bound to the CUDA device that was current when it was
 *    created; calls with another device current return ZERO_ERR_INVALID_ARG.
 *  - No C++ exception crosses this interface: a call that runs out of host
 *    memory or threads returns ZERO_ERR_OOM.
 *  - Threads: a plan is read-only after zero_plan and may be shared. A
 *    context holds host-side state (the step count bound, the scheduler's
 *    readiness counters, the prefetch ring), so calls on one context must
 *    not overlap in time; different contexts may be used from different
 *    threads. The CPU step (zero_cpu_step, zero_cpu_scan, zero_cpu_update)
 *    runs on a pool of worker threads that the library keeps between calls;
 *    a call that finds the pool busy with another thread's step starts
 *    threads of its own, so concurrent CPU steps on different buffers are
 *    safe.
 *  - The library owns only the plan (host memory) and the context's small
 *    device scratch (loss-scale state, overflow flag, per-block norm
 *    partials, bias-correction power table).
 */
#ifndef ZERO_B200_H
#define ZERO_B200_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

#define ZERO_MAX_RANKS 64

typedef enum {
    ZERO_OK = 0,
    ZERO_ERR_INVALID_ARG = 1, /* a bad argument value (null, out-of-range config, ...) */
    ZERO_ERR_ALIGN = 2,       /* a device pointer violates the alignment rule above */
    ZERO_ERR_CUDA = 3,        /* a CUDA runtime error (launch, async fault, no device) */
    ZERO_ERR_OOM = 4,         /* host or device allocation failed */
    ZERO_ERR_RANGE = 5,       /* a bucket / layer / tensor index or a size out of range */
    ZERO_ERR_TIMEOUT = 6,     /* a bounded device wait gave up; the step was abandoned */
    ZERO_ERR_STATE = 7        /* the call does not fit the context's state */
} zero_status;

typedef enum { ZERO_BF16 = 0, ZERO_FP16 = 1 } zero_dtype;

typedef enum {
    ZERO_SCALE_NONE = 0,    /* no loss scaling (bf16; [legal] "BFloat16 Compatibility") */
    ZERO_SCALE_STATIC = 1,  /* fixed scale, never skips */
    ZERO_SCALE_DYNAMIC = 2  /* skip + back off on overflow, grow after clean steps */
} zero_scale_mode;

typedef struct zero_plan_s zero_plan_t;
typedef struct zero_ctx_s zero_ctx_t;

/* ------------------------------------------------------------------------ */
/* Partition plan (host only; no GPU needed).                               */
/* ------------------------------------------------------------------------ */

typedef struct {
    int32_t R;            /* simulated data-parallel ranks, 1..ZERO_MAX_RANKS */
    int32_t dtype;        /* zero_dtype of gradients and parameters */
    int32_t tensor_align; /* each tensor starts at a multiple of this many
                             elements, 1..4096 (8 = 16 bytes of half) */
    int32_t reserved;     /* must be 0 */
    int64_t bucket_elems; /* reduce-scatter bucket capacity in raw elements;
                             <= 0 means one bucket for the whole model */
} zero_plan_config;

typedef struct {
    int64_t P;         /* raw parameter count (sum of numels) */
    int64_t L;         /* flat length: end of the last tensor */
    int64_t S;         /* shard length, a multiple of 8 */
    int64_t T;         /* padded total R*S */
    int64_t n_tensors, n_buckets, n_layers;
    int32_t R, dtype, tensor_align, reserved;
} zero_plan_info;

/*
 * zero_plan -- lay n parameter tensors into one flat buffer cut into R equal
 * shards, and group them into reduce-scatter buckets and gather layers.
 *
 * Defines: [instr] ZeRO-1/2/3 "Mechanism" bullets (each data-parallel
 * process owns and updates one partition of optimizer state, gradients and
 * parameters); [legal] "Bandwidth Optimization" bullet (small parameter
 * groups are fused to cope with irregular transformer tensor sizes);
 * [legal] ZeRO-3 "All-Gather on Demand" bullet (parameters are gathered per
 * layer before the layer runs).
 *
 * Layout: tensors are placed back to back in list order, tensor k at the
 * smallest multiple of tensor_align at or after the end of tensor k-1
 * (tensor 0 at 0); L is the end of the last tensor; S is the smallest
 * multiple of 8 that is >= ceil(L/R); T = R*S; rank r owns flat range
 * [r*S, (r+1)*S). Padding elements carry zero gradients and stay zero.
 * Buckets: greedy over tensors in reverse list order (the order gradients
 * become ready); a tensor joins the open bucket while the bucket's raw
 * element count stays <= bucket_elems; a larger tensor forms its own bucket;
 * tensors are never split. Bucket 0 holds the last tensor. A bucket's flat
 * range runs from its first tensor's offset to the next tensor's offset (the
 * bucket holding the last tensor ends at T), so the buckets partition
 * [0, T). Layers: layer_ids[k] gives tensor k's layer; ids start at 0 and
 * step by 0 or +1; layer l spans its first tensor's offset up to the next
 * layer's first offset, and the last layer ends at L. layer_ids == NULL makes
 * every tensor its own layer.
 *
 * numels: n counts (each >= 1), host memory, read during the call only.
 * Errors: ZERO_ERR_INVALID_ARG for n < 1, a count < 1, R or tensor_align out
 * of range, a bad dtype or layer id sequence; ZERO_ERR_RANGE if T/8 does not
 * fit in 31 bits; ZERO_ERR_OOM. On success *out owns a plan that the caller
 * frees with zero_plan_destroy.
 */
zero_status zero_plan(const int64_t* numels, const int32_t* layer_ids, int64_t n,
                      const zero_plan_config* cfg, zero_plan_t** out);
void zero_plan_destroy(zero_plan_t* plan);

zero_status zero_plan_get_info(const zero_plan_t* plan, zero_plan_info* info);
/* Tensor k: flat offset, numel, owning bucket and layer (any output may be NULL). */
zero_status zero_plan_tensor(const zero_plan_t* plan, int64_t k, int64_t* offset, int64_t* numel,
                             int64_t* bucket, int64_t* layer);
/* Bucket b's flat range [lo, hi). */
zero_status zero_plan_bucket(const zero_plan_t* plan, int64_t b, int64_t* lo, int64_t* hi);
/* Layer l's flat range [lo, hi). */
zero_status zero_plan_layer(const zero_plan_t* plan, int64_t l, int64_t* lo, int64_t* hi);

/*
 * zero_plan_memory -- model-state bytes one rank holds under this plan at a
 * given ZeRO stage (0 = plain data parallel, 1, 2, 3), counting 2 bytes of
 * half parameters, 2 of half gradients and 12 of fp32 master + momentum +
 * variance per element of the padded layout: stage 0: 16T; stage 1:
 * 4T + 12S; stage 2: 2T + 14S; stage 3: 16S.
 * Defines: [genomic] memory-breakdown bullets (2 + 2 + 12 bytes per
 * parameter) and the stage bullets of [legal] and [genomic] (ZeRO-1 shards
 * the optimizer state, ZeRO-2 adds gradients, ZeRO-3 adds parameters).
 * Errors: ZERO_ERR_INVALID_ARG for another stage or a NULL output.
 */
zero_status zero_plan_memory(const zero_plan_t* plan, int32_t stage, int64_t* bytes_per_rank);

/*
 * zero_plan_step_tiles -- how the staged steps (the fused step zero_step
 * runs for R <= 2, and the step from the accumulators at every R; their reads
 * are bulk copies into shared memory) cut this plan's shards: each shard
 * of S elements into *tiles_per_shard tiles of *tile_elems elements, the
 * last tile of a shard holding the rest,
 * S - (tiles_per_shard - 1) * tile_elems (a multiple of 8, at least 8); the
 * step's work is *tiles_total = R * tiles_per_shard tiles. Host arithmetic
 * in 64 bits, the same the launch uses, so a shard longer than 2^32
 * elements is tiled completely. Any output may be NULL.
 * Defines: [instr] ZeRO-1/2 "Mechanism" bullets (each owner updates every
 * element of its partition).
 * Errors: ZERO_ERR_INVALID_ARG for a NULL plan.
 */
zero_status zero_plan_step_tiles(const zero_plan_t* plan, int64_t* tile_elems, int64_t* tiles_per_shard,
                                 int64_t* tiles_total);

/* ------------------------------------------------------------------------ */
/* Context: device scratch and the loss-scale state.                        */
/* ------------------------------------------------------------------------ */

typedef struct {
    int32_t mode;            /* zero_scale_mode */
    float init_scale;        /* starting scale (STATIC, DYNAMIC); > 0, power of two advised */
    int64_t growth_interval; /* DYNAMIC: clean steps in a row before growth, >= 1 */
    float growth_factor;     /* DYNAMIC: multiplier on growth, > 1 (2) */
    float backoff_factor;    /* DYNAMIC: multiplier on overflow, in (0, 1) (0.5) */
    float min_scale;         /* DYNAMIC: floor of the scale, > 0 (1) */
    int32_t reserved;        /* must be 0 */
} zero_loss_scale_config;

/*
 * zero_ctx_create -- bind a context to the current CUDA device and allocate
 * its device scratch. The plan's layout is copied; the plan may be destroyed
 * afterwards. Defines the loss-scale state of [legal] "Dynamic Loss
 * Scaling" and [instr] "Loss Scaling": the scale starts at init_scale (1 in
 * NONE mode), the step count t at 0.
 * Errors: ZERO_ERR_INVALID_ARG (bad config), ZERO_ERR_CUDA (no device),
 * ZERO_ERR_OOM. Free with zero_ctx_destroy (which synchronizes the device).
 */
zero_status zero_ctx_create(const zero_plan_t* plan, const zero_loss_scale_config* cfg,
                            zero_ctx_t** out);
zero_status zero_ctx_destroy(zero_ctx_t* ctx);

/*
 * zero_ctx_reserve_steps -- make the context's bias-correction table
 * (beta1^t, beta2^t for the given betas) cover `steps` more optimizer steps
 * than the host has issued. zero_step grows the table by itself, with a
 * synchronous allocation and upload. A step captured into a CUDA graph and
 * replayed advances the device step count without the host seeing it, so
 * reserve at least the number of replays before capturing:
 *   - a captured zero_step that would have to grow the table returns
 *     ZERO_ERR_STATE and launches nothing;
 *   - a replay beyond the reserve reads the table's last entry (never past
 *     its end) and sets the device error flag, which the next
 *     zero_loss_scale reports as ZERO_ERR_STATE.
 * Outgrown tables stay allocated until zero_ctx_destroy, so no captured
 * graph ever holds a freed table. `stream` is only checked for a capture in
 * progress. Blocks the host while the table is uploaded; not capturable.
 */
zero_status zero_ctx_reserve_steps(zero_ctx_t* ctx, int64_t steps, double beta1, double beta2,
                                   void* stream);

/*
 * zero_test_drop_tile -- test support for the error path of the staged
 * fused step (R <= 2): the next zero_step / zero_step_shard with gradients
 * issues no copy for tile `tile` (tiles are 4096-element pieces of the
 * shards, numbered shard after shard), so the block that waits for it gives
 * up after its 2 s limit, as it would if a copy never arrived. The step is
 * then abandoned and reported as ZERO_ERR_TIMEOUT (see zero_loss_scale);
 * nothing faults and the context stays usable. One-shot; no effect on the
 * register kernel (R >= 4). Not part of the method; the pages have no
 * counterpart. Errors: ZERO_ERR_INVALID_ARG.
 */
zero_status zero_test_drop_tile(zero_ctx_t* ctx, int64_t tile);

/* ------------------------------------------------------------------------ */
/* The step.                                                                */
/* ------------------------------------------------------------------------ */

typedef struct {
    double lr, beta1, beta2, eps, weight_decay;
} zero_adamw;

/*
 * Sharded model state. Each array holds R device pointers (host memory, read
 * during the call only); entry r points at rank r's shard of S elements.
 * master/m/v are fp32, param is the plan's half dtype. Set 0 is required;
 * set 1 (all four arrays non-NULL, or all NULL) enables ping-pong steps:
 * the step (fused, or from the accumulators) then reads set `cur` and
 * writes set 1-cur, and flips `cur` only if the step is applied, so a
 * skipped step costs no extra traffic. Ping-pong also measured faster than
 * updating in place (writes never alias the lines being read), at the cost
 * of a second state set.
 * acc holds R fp32 accumulators of S elements for the two-pass path (may be
 * NULL for the fused path and for gathers).
 */
typedef struct {
    float* const* master[2];
    float* const* m[2];
    float* const* v[2];
    void* const* param[2];
    float* const* acc;
} zero_state;

/*
 * zero_reduce_scatter_bucket -- sum the R gradient replicas of one bucket
 * into the owning ranks' fp32 accumulators:
 *   acc[o][i - o*S] = ((f32(g_0[i]) + f32(g_1[i])) + ...) + f32(g_{R-1}[i])
 * for every flat index i of the bucket, o = i / S; the overflow flag of the
 * current step is OR-ed with "some sum is inf or NaN". Accumulators are
 * overwritten, not added to. bucket = -1 reduces the whole range [0, T) in
 * one launch.
 * Defines: [legal] "Reduce-Scatter" bullet and [instr] ZeRO-2
 * "Communication" bullet (a reduce-scatter aggregates and averages the
 * gradients and leaves each partition on its owner, replacing DP's
 * all-reduce); the division by R is folded into the step's unscale.
 * grads: R device pointers to full replicas of T half elements in the plan's
 * flat layout (zero in padding). acc: R device pointers, S fp32 each.
 * Errors: ZERO_ERR_RANGE (bucket), ZERO_ERR_INVALID_ARG, ZERO_ERR_ALIGN,
 * ZERO_ERR_CUDA.
 */
zero_status zero_reduce_scatter_bucket(zero_ctx_t* ctx, int64_t bucket, const void* const* grads,
                                       float* const* acc, void* stream);

/*
 * zero_reduce_scatter_bucket_ex -- zero_reduce_scatter_bucket with flags.
 * ZERO_RS_ACCUMULATE adds the bucket's rank-order sum to the accumulators
 * instead of overwriting them, for gradient accumulation over micro-batches:
 *   acc[o][i - o*S] = acc[o][i - o*S] + (((f32(g_0[i]) + f32(g_1[i])) + ...) + f32(g_{R-1}[i]))
 * The overflow flag is OR-ed with "some accumulator is inf or NaN". The
 * first micro-batch of a step must not accumulate (it initializes).
 * ZERO_RS_NORM also takes the call's share of the squared norm that global
 * clipping needs, from the accumulator values it writes, as the step would
 * form the unscaled gradient:
 *   sum over the range of (double)((float)(acc * inv))^2,
 *   inv = (float)(1 / ((R * d) * scale)),
 * d the context's gradient divisor (zero_ctx_set_grad_divisor, default 1)
 * and scale the loss scale at launch time (1 without loss scaling). The
 * share lands in a device slot of the bucket (of the whole range for
 * bucket -1), which a two-pass zero_step_ex with ZERO_STEP_NORM_FROM_RS
 * sums instead of re-reading every accumulator. Give the flag to the last
 * micro-batch's call, the one that leaves the accumulator final; a later
 * call on the bucket without it (or a call on the whole range) makes the
 * slot stale, and the step refuses stale or missing slots.
 * Defines: gradient accumulation is not on the pages, which only note that
 * ZeRO frees memory for larger effective batches ([instr], large-batch
 * paragraph); the reduce-scatter itself is [legal] "Reduce-Scatter".
 * Clipping is not on the pages either.
 * Errors: as zero_reduce_scatter_bucket, plus ZERO_ERR_INVALID_ARG for
 * unknown flags.
 */
#define ZERO_RS_ACCUMULATE 1
#define ZERO_RS_NORM 2
zero_status zero_reduce_scatter_bucket_ex(zero_ctx_t* ctx, int64_t bucket, const void* const* grads,
                                          float* const* acc, int32_t flags, void* stream);

/*
 * zero_reduce_scatter_buckets -- zero_reduce_scatter_bucket_ex over the
 * consecutive buckets [first, first + count) in one launch. Consecutive
 * buckets are adjacent in the flat layout (bucket b + 1 ends where bucket b
 * begins), so this is one reduce-scatter of the flat range from the start of
 * bucket first + count - 1 to the end of bucket first: the same bytes as
 * count separate calls, with one launch instead of count. For small buckets
 * the launches, not the bytes, bound the separate calls. first = -1 with
 * count = 1 is the whole range. With ZERO_RS_NORM the group's norm share
 * lands in the slot of bucket `first` and the other buckets' slots hold 0,
 * so the step's sum over every slot is the same norm.
 * Defines: [legal] "Bandwidth Optimization" (fusing small parameter groups
 * into larger transfers) applied to launches.
 * Errors: as zero_reduce_scatter_bucket_ex; ZERO_ERR_RANGE unless
 * 0 <= first, 1 <= count and first + count <= n_buckets.
 */
zero_status zero_reduce_scatter_buckets(zero_ctx_t* ctx, int64_t first, int64_t count, const void* const* grads,
                                        float* const* acc, int32_t flags, void* stream);

/*
 * zero_ctx_set_grad_divisor -- the gradient divisor d (>= 1, finite) that
 * later ZERO_RS_NORM reduce-scatters unscale by; the step checks that its
 * own grad_divisor equals the one each slot was taken with. Host state
 * only. Errors: ZERO_ERR_INVALID_ARG.
 */
zero_status zero_ctx_set_grad_divisor(zero_ctx_t* ctx, double grad_divisor);

/*
 * zero_step -- one optimizer step on every shard, then the loss-scale update.
 *
 * With g = acc * (1 / (R * scale)) the unscaled, averaged gradient (scale = 1
 * in NONE mode), t the step count after this step, and every operation one
 * rounded fp32 operation without fused multiply-add:
 *   p = p * (1 - lr*wd)
 *   m = b1*m + (1-b1)*g
 *   v = b2*v + (1-b2)*(g*g)
 *   p = p - (lr / (1 - b1^t)) * (m / (sqrt(v) / sqrt(1 - b2^t) + eps))
 *   param = round-to-nearest-even half(p)
 * Scalar coefficients are formed in double and rounded once to float. The
 * step is skipped (state untouched, t unchanged) only in DYNAMIC mode when
 * the step's overflow flag is set. The loss-scale update then runs on the
 * device without a host round trip: DYNAMIC overflow -> scale = max(scale *
 * backoff, min_scale), clean count 0; DYNAMIC clean -> t += 1, count += 1,
 * and at growth_interval the scale grows and the count clears; NONE/STATIC
 * -> t += 1. The squared L2 norm of g is recorded (diagnostic).
 *
 * Defines: [instr] ZeRO-1 "Mechanism" (each process updates only its
 * partition of the Adam state), [genomic] memory breakdown (fp32 master,
 * momentum and variance), [instr] "Precision Management" (fp32 update on
 * upcast gradients, weights cast back to half), [legal] "Dynamic Loss
 * Scaling" and [instr] "Loss Scaling" (unscale before the update; the scale
 * adjusts itself). The Adam formula itself is not printed on the pages; the
 * one above is bias-corrected Adam with decoupled weight decay.
 *
 * grads == NULL: two-pass path; g comes from the accumulators written by
 * zero_reduce_scatter_bucket for this step (state->acc), the step is done in
 * place on set cur when the state has one set, from set cur into set 1-cur
 * when it has two (a skipped step writes nothing either way). grads != NULL: fused path; the R replicas are reduced,
 * checked, and applied in one pass with no accumulator: in place when the
 * state has one set (NONE or STATIC mode only, since an in-place fused step
 * cannot be undone), ping-pong when it has two.
 * Errors: ZERO_ERR_INVALID_ARG (a NULL pointer, DYNAMIC fused in place,
 * bad hyper-parameters), ZERO_ERR_ALIGN, ZERO_ERR_STATE (one state set
 * given after ping-pong steps), ZERO_ERR_CUDA, ZERO_ERR_OOM.
 */
zero_status zero_step(zero_ctx_t* ctx, const zero_adamw* hp, const zero_state* state,
                      const void* const* grads, void* stream);

/*
 * zero_step_ex -- zero_step with options (opts == NULL: the defaults, i.e.
 * exactly zero_step).
 *  grad_divisor k (>= 1, default 1): the unscale multiplies by
 *    (float)(1 / ((R * k) * scale)); k = the number of accumulated
 *    micro-batches gives their mean.
 *  max_grad_norm (> 0 turns clipping on, 0 = off): with ||g|| the L2 norm of
 *    the unscaled gradient, c = (float) min(1, max_norm / (||g|| + 1e-6)) in
 *    double, and the update uses g * c (one fp32 multiply). Clipping needs
 *    the norm before any element is updated, so one read-only pass comes
 *    first: over the accumulators on the two-pass path (4 bytes per
 *    element; none with ZERO_STEP_NORM_FROM_RS), over the R replicas on the
 *    fused path (2R bytes per element; they are summed in rank order as the
 *    step sums them). The fused path with clipping moves 4R + 26 bytes per
 *    element against 2R + 34 for the two-pass path with the reduce-scatters'
 *    norm shares (2R + 38 with the pass), so it is the cheaper one for
 *    R <= 3 and even at R = 4. The recorded grad_norm_sq is the norm before
 *    clipping.
 *  flags & ZERO_STEP_ADD_ACC (fused path, the last micro-batch of an
 *    accumulation): the reduced gradient is state->acc[o] plus this
 *    micro-batch's rank-order sum of the replicas,
 *      acc + (((f32(g_0) + f32(g_1)) + ...) + f32(g_{R-1})),
 *    exactly what zero_reduce_scatter_bucket_ex(ZERO_RS_ACCUMULATE) followed
 *    by the two-pass step computes, in one pass that neither writes nor
 *    re-reads the accumulator: 2R + 30 bytes per element instead of
 *    (2R + 8) + 30. The accumulator is read only. Not combinable with
 *    clipping (whose norm needs the sum before the update): use the two-pass
 *    path for that.
 *  flags & ZERO_STEP_NORM_FROM_RS (two-pass path with clipping): the
 *    global norm is the sum, in slot order, of the norm shares that this
 *    step's ZERO_RS_NORM reduce-scatters recorded (every bucket's slot, or
 *    the whole-range slot), instead of a read-only pass over the
 *    accumulators: 2R + 34 bytes per element instead of 2R + 38. Refused
 *    (ZERO_ERR_STATE) unless every slot it needs is current and was taken
 *    with this call's grad_divisor. Every zero_step_ex marks the slots
 *    used up.
 *  flags & ZERO_STEP_PUSH_PARAMS: the step also writes every updated half
 *    parameter vector into the full-model parameter buffers registered with
 *    zero_ctx_set_param_push, one per rank (the ZeRO-1/2 all-gather of the
 *    updated parameters, done by the step itself): buffer [dst][r] for every
 *    rank r, where dst is the state set the step writes (1-cur with
 *    ping-pong, else cur), at the element's flat index. After the step (and,
 *    for a sharded step, the commit), each rank's buffer of set cur holds
 *    the whole updated model, padding zero. 2 more bytes per element per
 *    rank are written; with one process per GPU the peers' buffers are
 *    peer-mapped (zero_ipc_open) and written with plain stores, so the
 *    all-gather's NVLink traffic leaves while the step streams HBM.
 * Defines: not on the pages (clipping and accumulation are common practice
 * around ZeRO training loops, not part of the method the pages describe);
 * the parameter push follows [instr] ZeRO-1 "Mechanism" (the updated
 * partitions are all-gathered so that every process holds the full model).
 * Errors: as zero_step, plus ZERO_ERR_INVALID_ARG for a divisor < 1, a
 * negative or non-finite max norm, unknown flags, ZERO_STEP_ADD_ACC
 * without grads, without state->acc or with clipping, or
 * ZERO_STEP_NORM_FROM_RS with grads or without clipping; ZERO_ERR_STATE for
 * ZERO_STEP_NORM_FROM_RS without current norm slots, or for
 * ZERO_STEP_PUSH_PARAMS without registered buffers for the set written.
 */
#define ZERO_STEP_ADD_ACC 1
#define ZERO_STEP_NORM_FROM_RS 2
#define ZERO_STEP_PUSH_PARAMS 4
typedef struct {
    double grad_divisor;
    double max_grad_norm;
    int64_t flags;    /* ZERO_STEP_* bits, 0 for none */
    int64_t reserved; /* must be 0 */
} zero_step_opts;
zero_status zero_step_ex(zero_ctx_t* ctx, const zero_adamw* hp, const zero_state* state,
                         const void* const* grads, const zero_step_opts* opts, void* stream);

/*
 * zero_ctx_set_param_push -- register the full-model parameter buffers that
 * steps with ZERO_STEP_PUSH_PARAMS write: full0[r] (state set 0) and
 * full1[r] (set 1, needed once ping-pong state is used), for r in [0, R),
 * each T half elements, 16-byte aligned, caller-owned; with one process per
 * GPU, rank r's buffers as this process maps them (its own, or a peer's
 * through zero_ipc_open). full0 == NULL clears the registration. The
 * pointers are copied; the buffers must outlive the steps that write them.
 * Defines: [instr] ZeRO-1 "Mechanism" (every process ends the step with the
 * full updated parameters).
 * Errors: ZERO_ERR_INVALID_ARG (a NULL entry), ZERO_ERR_ALIGN.
 */
zero_status zero_ctx_set_param_push(zero_ctx_t* ctx, void* const* full0, void* const* full1);

/*
 * zero_step_shard -- the fused step (grads != NULL path of zero_step) on
 * shards [owner_lo, owner_hi) only, with the loss-scale update left to
 * zero_step_commit: the step's last block writes partial[0] = sum of g^2 and
 * partial[1] = 1 if some reduced gradient of these shards is inf/NaN, else 0.
 * This is the per-rank half of a multi-GPU ZeRO step: rank o calls it with
 * [o, o+1) and grads[r] pointing at rank r's gradient buffer (peer-mapped,
 * read with plain loads or bulk copies without multicast); the ranks then
 * all-reduce `partial` (sum) and each calls zero_step_commit with the
 * result, so every rank takes the same skip and loss-scale decision. In one
 * process, calling it for every shard and summing the partials gives exactly
 * zero_step. Only the owned shards' state pointers are read (others may be
 * NULL); DYNAMIC mode needs the ping-pong set, as for zero_step.
 * Defines: [instr] ZeRO-2 "Mechanism" and "Communication" (each process
 * reduces and updates only its own partition) and [instr] "Baseline (DP)" /
 * ZeRO-2 (the reduce-scatter replaces the all-reduce); the overflow and norm
 * are the small all-reduce every rank needs for the shared decision.
 * partial: device, 2 doubles, 8-byte aligned, caller-owned.
 * Errors: ZERO_ERR_RANGE (owner range), ZERO_ERR_INVALID_ARG, ZERO_ERR_ALIGN,
 * ZERO_ERR_STATE, ZERO_ERR_CUDA.
 */
zero_status zero_step_shard(zero_ctx_t* ctx, const zero_adamw* hp, const zero_state* state,
                            const void* const* grads, int32_t owner_lo, int32_t owner_hi,
                            double* partial, void* stream);

/*
 * zero_step_shard_ex -- zero_step_shard with the options of zero_step_ex,
 * and the two-pass path:
 *  - grads != NULL: the fused step over the owners' shards, as zero_step_shard;
 *  - grads == NULL: the step from the owners' accumulators state->acc[o]
 *    (written by zero_reduce_scatter_shard), from set cur into set 1-cur
 *    with ping-pong state, else in place. The skip is decided only by
 *    zero_step_commit, so DYNAMIC mode needs the ping-pong set here too.
 *  - opts->max_grad_norm > 0: global-norm clipping. Its norm spans every
 *    rank, so global_norm_sq (device, 1 double) must hold the cross-rank sum
 *    of the zero_grad_norm_shard partials of this step; the coefficient
 *    min(1, max_norm / (sqrt(global_norm_sq) + 1e-6)) is formed from it on
 *    the device. global_norm_sq may be NULL without clipping.
 *  - opts->flags may hold ZERO_STEP_ADD_ACC (fused path, as for
 *    zero_step_ex): only the owners' accumulators are read; and
 *    ZERO_STEP_PUSH_PARAMS: the owners' updated parameters are written into
 *    every rank's registered full-model buffer of the set the step writes,
 *    so that after the commit each rank holds the whole model in set cur.
 * partial and the commit are as for zero_step_shard. Running every owner
 * range in one process, with the partials summed, gives exactly zero_step_ex.
 * Defines: [instr] ZeRO-2 "Mechanism"; clipping and accumulation are not on
 * the pages (see zero_step_ex).
 * Errors: as zero_step_shard, plus ZERO_ERR_INVALID_ARG for bad options or a
 * missing global_norm_sq.
 */
zero_status zero_step_shard_ex(zero_ctx_t* ctx, const zero_adamw* hp, const zero_state* state,
                               const void* const* grads, int32_t owner_lo, int32_t owner_hi,
                               const zero_step_opts* opts, const double* global_norm_sq,
                               double* partial, void* stream);

/*
 * zero_reduce_scatter_shard -- zero_reduce_scatter_bucket_ex restricted to
 * owners [owner_lo, owner_hi): the part of bucket `bucket` (-1: every
 * element) inside their flat range [owner_lo*S, owner_hi*S) is summed from
 * all R replicas in rank order into acc[o] (or added to it, with
 * ZERO_RS_ACCUMULATE), and the context's overflow flag is OR-ed as usual.
 * This is rank o's part of a multi-GPU bucketed reduce-scatter: grads[r] is
 * rank r's gradient buffer (peer-mapped; plain loads, no multicast) and only
 * acc[o] for the owned ranks is touched (other entries may be NULL). A
 * bucket with no owned element launches nothing. ZERO_RS_NORM takes the
 * owned part's norm share as zero_reduce_scatter_bucket_ex does (0 for a
 * bucket with no owned element), recorded for this owner range; a context
 * that several owner ranges share keeps only the last range's shares, so
 * use one context per rank for it.
 * Defines: [legal] "Reduce-Scatter" and [instr] ZeRO-2 "Communication".
 * Errors: ZERO_ERR_RANGE (bucket, owner range), ZERO_ERR_INVALID_ARG,
 * ZERO_ERR_ALIGN, ZERO_ERR_CUDA.
 */
zero_status zero_reduce_scatter_shard(zero_ctx_t* ctx, int64_t bucket, const void* const* grads,
                                      float* const* acc, int32_t owner_lo, int32_t owner_hi,
                                      int32_t flags, void* stream);

/*
 * zero_grad_norm_shard -- owners [owner_lo, owner_hi)'s part of the global
 * gradient norm for clipping: partial[0] = sum over their elements of
 * (float)(x * inv)^2 in double, inv = (float)(1 / ((R * grad_divisor) *
 * scale)), where x is the element's reduced gradient read either from the
 * R replicas (grads != NULL, summed in rank order as the fused step sums
 * them) or from the owners' accumulators (acc != NULL); partial[1] = 0.
 * With grads and acc both NULL, partial[0] is instead the sum, in slot
 * order, of the norm shares that this owner range's ZERO_RS_NORM
 * reduce-scatters (zero_reduce_scatter_shard) took with this grad_divisor
 * (the context's, zero_ctx_set_grad_divisor): no accumulator is read.
 * The ranks all-reduce partial[0] (sum) and pass it to zero_step_shard_ex
 * as global_norm_sq.
 * partial: device, 2 doubles, 8-byte aligned.
 * Errors: ZERO_ERR_RANGE, ZERO_ERR_INVALID_ARG (both grads and acc given),
 * ZERO_ERR_ALIGN, ZERO_ERR_CUDA; ZERO_ERR_STATE when the shares are stale,
 * missing, or were taken with another owner range or divisor.
 */
zero_status zero_grad_norm_shard(zero_ctx_t* ctx, const void* const* grads, float* const* acc,
                                 double grad_divisor, int32_t owner_lo, int32_t owner_hi,
                                 double* partial, void* stream);

/*
 * zero_step_commit -- the loss-scale update after zero_step_shard, from
 * totals reduced over every shard: reduced[0] = sum of g^2 (recorded as
 * grad_norm_sq), reduced[1] > 0 means overflow. Skip, backoff, growth, t and
 * the ping-pong flip follow zero_step.
 * reduced: device, 2 doubles, 8-byte aligned.
 */
zero_status zero_step_commit(zero_ctx_t* ctx, const double* reduced, void* stream);

/*
 * zero_gather_layer -- assemble one layer's half parameters from the R
 * shards of the current set into a contiguous buffer:
 *   out[j] = param[cur][o][lo + j - o*S],  o = (lo + j) / S,  0 <= j < hi - lo.
 * Defines: [legal] ZeRO-3 "All-Gather on Demand" and [instr] ZeRO-3 forward /
 * backward bullets (a layer's parameters are all-gathered just before use
 * and released afterwards; the backward pass gathers again); [genomic]
 * "Bucketed All-Gather".
 * out: device buffer of (hi - lo) half elements, 16-byte aligned; the
 * caller owns and releases it.
 * Errors: ZERO_ERR_RANGE (layer), ZERO_ERR_INVALID_ARG, ZERO_ERR_ALIGN,
 * ZERO_ERR_STATE, ZERO_ERR_CUDA.
 */
zero_status zero_gather_layer(zero_ctx_t* ctx, int64_t layer, const zero_state* state, void* out,
                              void* stream);

/*
 * zero_gather_layers -- gather `count` consecutive layers in one launch:
 * layer first+i into outs[i], for 0 <= i < count, with exactly the result of
 * count calls of zero_gather_layer.
 * Defines: [genomic] "Bucketed All-Gather" bullet (parameter shards are
 * grouped into buckets and a whole bucket is all-gathered at once, ahead of
 * the layers that use it) and [legal] ZeRO-3 "Prefetching Scheduler"
 * (upcoming layers are fetched ahead of use).
 * count: 1..ZERO_GATHER_MAX_LAYERS. outs: count device pointers (host
 * array, read during the call), each 16-byte aligned and holding its layer's
 * (hi - lo) half elements; caller-owned.
 * Errors: ZERO_ERR_RANGE (first/count), ZERO_ERR_INVALID_ARG, ZERO_ERR_ALIGN,
 * ZERO_ERR_STATE, ZERO_ERR_CUDA.
 */
#define ZERO_GATHER_MAX_LAYERS 64
zero_status zero_gather_layers(zero_ctx_t* ctx, int64_t first, int64_t count,
                               const zero_state* state, void* const* outs, void* stream);

typedef struct {
    float scale;           /* current loss scale */
    int32_t cur;           /* state set holding the current model (0 or 1) */
    int64_t good;          /* clean steps since the last scale change */
    int64_t t;             /* applied optimizer steps */
    int32_t last_overflow; /* the last step saw an inf/NaN gradient sum */
    int32_t last_skipped;  /* the last step was skipped */
    double grad_norm_sq;   /* squared L2 norm of the last step's unscaled, averaged gradient */
} zero_loss_scale_state;

#define ZERO_LOSS_SCALE_GET 0
#define ZERO_LOSS_SCALE_SET 1

/*
 * zero_loss_scale -- read (GET) or overwrite (SET) the device-resident
 * loss-scale state; SET is how a run resumes from a checkpoint. Both
 * synchronize `stream` (GET reads the state after all work queued on it).
 * Defines: the state of [legal] "Dynamic Loss Scaling".
 * A step during which the device raised an error is abandoned: t, scale,
 * good and cur keep their values from before it, so with ping-pong state
 * the current set still holds the model from before the step (an in-place
 * step may have updated part of its set). GET then returns
 * ZERO_ERR_TIMEOUT (a step kernel's bounded wait for its tile copies ran
 * out) or ZERO_ERR_STATE (the bias-correction table was behind t) until a
 * SET, which clears the error.
 * Errors: ZERO_ERR_INVALID_ARG (op, NULL, cur not 0/1, scale <= 0, t < 0),
 * ZERO_ERR_TIMEOUT, ZERO_ERR_STATE, ZERO_ERR_CUDA.
 */
zero_status zero_loss_scale(zero_ctx_t* ctx, zero_loss_scale_state* inout, int32_t op,
                            void* stream);

/*
 * zero_step_noalloc -- the two-pass step (reduce-scatter of all R replicas
 * into fp32 accumulators, then the AdamW step above, in place on one state
 * set) for callers that cannot allocate device memory: processes whose GPU
 * memory is owned by another allocator that has already reserved it, and
 * loops that may not call cudaMalloc or cudaFree because those calls
 * synchronize the device or can fail mid-run. This call allocates nothing
 * and needs no context: its scratch (the accumulators, the per-block norm
 * partials and a control word) lives in one static device array of
 * 16 MiB + 32 KiB + 256 B. A device reserves the array when the library's
 * code module that holds it is loaded there; under CUDA's default lazy
 * module loading that is the first zero_step_noalloc call on the device
 * (its set-up, below), and the device then holds the array until the
 * process exits. So make the first call on each device before another
 * allocator has taken all of its memory; later calls reserve nothing. The
 * pages have no counterpart to this entry point; it is a deployment variant
 * of zero_reduce_scatter_bucket(-1) + zero_step (grads == NULL) and gives
 * the same results.
 *
 * plan: the layout (host only); its padded length T must be at most
 * ZERO_NOALLOC_MAX_ELEMS, else ZERO_ERR_RANGE. cfg: loss-scale mode and
 * rules as for zero_ctx_create. inout: HOST memory; the loss-scale state
 * before the step (cur must be 0), overwritten with the state after it.
 * grads: R device pointers to full half replicas of T elements; master, m, v
 * (fp32, 32-byte aligned) and param (half, 16-byte aligned): R device
 * pointers to the shards of S elements, updated in place.
 *
 * Set-up: the first call on each device (with that device current) looks up
 * the device address of the static scratch, again after the device's
 * context has been replaced (a device reset); make that first call before
 * any stream capture begins. Every call shares the same scratch and leaves the
 * last call's contents in it (the control word is cleared at the start of
 * each call). Calls whose work overlaps on the GPU -- two streams, two host
 * threads, or two devices' calls racing on one device -- race on the
 * scratch and give wrong results; serialize them. The call synchronizes
 * `stream` before it returns (it reads the overflow flag and the norm back
 * to update `inout`).
 * Errors: ZERO_ERR_RANGE (model too large), ZERO_ERR_INVALID_ARG,
 * ZERO_ERR_ALIGN, ZERO_ERR_CUDA.
 */
#define ZERO_NOALLOC_MAX_ELEMS 4194304
zero_status zero_step_noalloc(const zero_plan_t* plan, const zero_loss_scale_config* cfg,
                              zero_loss_scale_state* inout, const zero_adamw* hp,
                              const void* const* grads, float* const* master, float* const* m,
                              float* const* v, void* const* param, void* stream);

/* ------------------------------------------------------------------------ */
/* Buffers shared across the processes of a multi-GPU job (CUDA IPC).       */
/* ------------------------------------------------------------------------ */

/*
 * One rank's device buffer as its peers need it to map it: the IPC handle of
 * the cudaMalloc allocation that holds the buffer, the buffer's byte offset
 * in that allocation and the allocation's size. Plain bytes: a job passes it
 * between its processes with any collective.
 */
typedef struct {
    uint8_t handle[64];
    int64_t offset;
    int64_t alloc_bytes;
} zero_ipc_handle;

/*
 * zero_ipc_export -- describe the device buffer at `ptr` for the other
 * processes of the job. With one process per GPU, rank o's fused step and
 * gathers read every peer's gradient replica and parameter shard; the peers
 * reach those buffers through zero_ipc_open.
 * Defines: the exchanges of [legal] "Reduce-Scatter" and "All-Gather on
 * Demand" (each rank reads its partition of every peer's gradients, and
 * every layer's parameters from their owners) as peer reads over NVLink.
 * ptr: any address inside a device allocation made with cudaMalloc (for
 * example a PyTorch tensor from its default allocator); an allocation from
 * a virtual-memory pool cannot be exported and returns ZERO_ERR_CUDA. Call
 * with the device that owns `ptr` current. The caller keeps the allocation
 * alive until every peer has closed its handle.
 * Errors: ZERO_ERR_INVALID_ARG (NULL, or host memory), ZERO_ERR_CUDA.
 */
zero_status zero_ipc_export(const void* ptr, zero_ipc_handle* out);

/*
 * zero_ipc_open -- map a buffer that another process exported (on another
 * GPU of this node) into this process: *out is its device address here,
 * which the entry points above accept as a peer's buffer (plain loads and
 * 1-D bulk copies; never a multicast load). The allocation is mapped once
 * per process and device however many of its buffers are opened; peer access to the
 * exporting GPU is enabled for this mapping. Call with the device that will
 * read the buffer current.
 * Errors: ZERO_ERR_INVALID_ARG, ZERO_ERR_RANGE (an offset outside the
 * allocation), ZERO_ERR_CUDA (for instance a handle from this process).
 */
zero_status zero_ipc_open(const zero_ipc_handle* h, void** out);

/*
 * zero_ipc_close -- end one zero_ipc_open of this handle (with the same
 * device current); the allocation is unmapped when its last open buffer is
 * closed. Nothing may still read the buffer (synchronize first). Errors: ZERO_ERR_INVALID_ARG, ZERO_ERR_STATE
 * (the handle is not open here), ZERO_ERR_CUDA.
 */
zero_status zero_ipc_close(const zero_ipc_handle* h);

/* ------------------------------------------------------------------------ */
/* Overlap and prefetch scheduling (a communication stream owned by the     */
/* context, created on first use with the highest stream priority).         */
/* ------------------------------------------------------------------------ */

/*
 * zero_sched_set_comm_sms -- cap the kernels that the scheduler launches on
 * its communication stream (the reduce-scatters of zero_grads_ready, the
 * gathers of the prefetch ring) at `sms` SMs' worth of resident blocks, so
 * that they run beside the caller's compute instead of taking every SM a
 * finishing compute kernel frees; 0 (the default) lets them fill the GPU.
 * Two launches always get the whole GPU, having no compute to hide behind: a
 * step's last reduce-scatter bucket and the first gather of a prefetch pass.
 * The kernels loop over their range with whatever grid they get, so results
 * do not depend on the setting. Pair it with keeping as many SMs free of the
 * compute kernels. Defines: [legal] "Communication Overlap" (the reduction
 * runs while the backward pass continues). Errors: ZERO_ERR_INVALID_ARG.
 */
zero_status zero_sched_set_comm_sms(zero_ctx_t* ctx, int32_t sms);

/*
 * zero_grads_ready -- report that tensors [first, first+count) have their
 * gradients written in `grads` by the work queued on `stream` so far. Each
 * bucket whose tensors have then all been reported is reduce-scattered at
 * once (as zero_reduce_scatter_bucket_ex with `flags`) on the communication
 * stream, ordered after that work by an event, so the reduction of early
 * buckets overlaps the caller's next work on `stream`. Buckets that one call
 * completes and that are consecutive go in one launch, as
 * zero_reduce_scatter_buckets (a caller reporting a whole layer at a time
 * pays one launch per layer, however small the buckets).
 * Defines: [legal] "Communication Overlap" (a layer's gradient reduction
 * starts as soon as its gradients are computed, hidden behind the backward
 * pass) and [genomic] "Reduce-Scatter Overlap".
 * grads / acc: as zero_reduce_scatter_bucket; they must stay the same
 * buffers until zero_grads_join.
 * Errors: ZERO_ERR_RANGE, ZERO_ERR_INVALID_ARG, ZERO_ERR_ALIGN,
 * ZERO_ERR_STATE (a tensor reported twice before the join), ZERO_ERR_CUDA.
 */
zero_status zero_grads_ready(zero_ctx_t* ctx, int64_t first, int64_t count, const void* const* grads,
                             float* const* acc, int32_t flags, void* stream);

/*
 * zero_grads_join -- make `stream` wait for every reduce-scatter issued by
 * zero_grads_ready, and start a new round of reports (the next micro-batch
 * or step). Every tensor must have been reported, else ZERO_ERR_STATE.
 * A two-pass zero_step / zero_step_ex (grads == NULL) on `stream` follows.
 */
zero_status zero_grads_join(zero_ctx_t* ctx, void* stream);

/*
 * zero_prefetch_begin -- start one pass over the layers (direction +1:
 * layer 0 first, the forward pass; -1: the last layer first, the backward
 * pass) with look-ahead gathering: the layer at sequence position p is
 * gathered (as zero_gather_layer, from the current parameter set) into
 * bufs[p % nbufs] on the communication stream, up to `depth` positions
 * ahead of the layer in use. A slot is refilled only after the layer it held
 * has been released. All gathers of the pass come after the work queued on
 * `stream` before this call (for example the optimizer step).
 * Defines: [legal] ZeRO-3 "Prefetching Scheduler" (a look-ahead scheduler
 * fetches the next parameters while the current layer computes) and
 * [genomic] "Bucketed All-Gather" / "Prefetch Scheduling".
 * bufs: nbufs device pointers (host array, copied), each 16-byte aligned and
 * large enough for the largest layer; 1 <= nbufs <= 64; 0 <= depth < nbufs.
 * state: param[0] (and param[1] for ping-pong) as for zero_gather_layer.
 */
zero_status zero_prefetch_begin(zero_ctx_t* ctx, const zero_state* state, void* const* bufs,
                                int32_t nbufs, int32_t depth, int32_t direction, void* stream);

/*
 * zero_layer_acquire -- *buf receives the buffer that holds `layer`; work
 * queued on `stream` after this call sees the gathered layer. Also queues the
 * gathers of the next `depth` layers of the pass whose slots are free.
 * Errors: ZERO_ERR_STATE when no pass is active or the layer's slot is still
 * held by an unreleased layer (acquire in pass order, release after use).
 */
zero_status zero_layer_acquire(zero_ctx_t* ctx, int64_t layer, void** buf, void* stream);

/*
 * zero_layer_release -- the work queued on `stream` so far is done with
 * `layer`'s buffer; its slot may be refilled after that work.
 */
zero_status zero_layer_release(zero_ctx_t* ctx, int64_t layer, void* stream);

/* ------------------------------------------------------------------------ */
/* ZeRO-Offload: the optimizer step on CPU cores (host only, no GPU).       */
/* ------------------------------------------------------------------------ */

/*
 * zero_cpu_step -- the optimizer step of zero_step_ex on host memory, for
 * training with the fp32 master weights and Adam moments offloaded to CPU
 * RAM: acc holds the R reduced fp32 gradient shards (for example copied
 * from the GPU accumulators after zero_reduce_scatter_bucket), master / m /
 * v are updated in place, and param receives the half parameters to copy
 * back to the GPU. The overflow check, loss-scale state machine, grad
 * divisor and clipping follow zero_step_ex exactly, and the element
 * arithmetic is the same IEEE fp32 sequence, so results equal the GPU step
 * bit for bit. inout (host) holds the loss-scale state before the step and
 * receives it after; cur must be 0.
 * Defines: [legal] "CPU Offload" (Adam on the CPU while the GPU runs forward
 * and backward) and [genomic] "CPU Offload" (fp32 master weights and
 * optimizer states in CPU RAM); [legal] / [genomic] "One-Step Delayed
 * Parameter Update" is the caller overlapping this call with the next
 * forward pass (it releases no lock and touches no GPU state).
 * All pointers are HOST memory: R pointers each, S elements per shard
 * (pinned memory makes the surrounding copies asynchronous). nthreads <= 0
 * uses every hardware thread (the calling thread is one of them), and more
 * than 1024 count as 1024; the result
 * does not depend on nthreads except for the summation order of
 * grad_norm_sq. Work under 65,536 elements runs on the calling thread.
 * Without a skip to decide (NONE or STATIC mode) and without clipping, the
 * accumulators are scanned block by block right before each block's update,
 * in one pass (30 bytes per element instead of 34); otherwise every
 * accumulator is scanned first, as zero_cpu_scan does.
 * opts->flags may hold ZERO_STEP_CLEAN (no other flag): the caller vouches
 * that no accumulator element is inf or NaN, for instance because
 * zero_take_overflow read 0 after the reduce-scatters that wrote them. A
 * DYNAMIC-mode step without clipping then has no skip to decide first and
 * runs in one pass too. Should the pass meet an inf or NaN all the same,
 * the update has been applied: the call returns ZERO_ERR_STATE and leaves
 * *inout as it was.
 * Errors: ZERO_ERR_INVALID_ARG, ZERO_ERR_STATE (ZERO_STEP_CLEAN contradicted).
 */
#define ZERO_STEP_CLEAN 8
zero_status zero_cpu_step(const zero_plan_t* plan, const zero_loss_scale_config* cfg,
                          zero_loss_scale_state* inout, const zero_adamw* hp, const zero_step_opts* opts,
                          const float* const* acc, float* const* master, float* const* m, float* const* v,
                          void* const* param, int32_t nthreads);

/*
 * zero_take_overflow -- the overflow flag that this context's reduce-scatters
 * OR-ed since the last step (1 if some value they wrote is inf or NaN, else
 * 0) into *flag, and the flag cleared: for a step taken outside the GPU,
 * such as zero_cpu_step of ZeRO-Offload, which can then skip its scan
 * (ZERO_STEP_CLEAN). A GPU step consumes and clears the flag by itself.
 * Asynchronous on `stream`, after the reduce-scatters queued there.
 * Defines: [legal] "Dynamic Loss Scaling" (the overflow decides the skip)
 * and [legal] "CPU Offload" (the optimizer step runs on the CPU).
 * flag: device memory, one int32, caller-owned, 4-byte aligned.
 * Errors: ZERO_ERR_INVALID_ARG, ZERO_ERR_ALIGN, ZERO_ERR_CUDA.
 */
zero_status zero_take_overflow(zero_ctx_t* ctx, int32_t* flag, void* stream);

/*
 * zero_debug_bounds -- what the bounds-checking debug build recorded. That
 * build (the same sources compiled with ZERO_DEBUG_BOUNDS) checks, in every
 * kernel, each index and pointer it derives before the access that uses it:
 * the vector within the flat range and the shard, the owner within the
 * range given, the owner's buffers present. A failing access is skipped
 * (never trapped) and counted; the first one's site number (the kernel and
 * access) and index are kept. *count receives the number of failing
 * accesses since the last reset, or -1 in the release build, whose kernels
 * carry no checks. reset != 0 clears the record. Synchronizes the device.
 * Errors: ZERO_ERR_INVALID_ARG (NULL output), ZERO_ERR_CUDA.
 */
zero_status zero_debug_bounds(int64_t* count, int64_t* first_site, int64_t* first_index, int32_t reset);

/*
 * The CPU step in three calls, for callers that overlap the update with the
 * upload of the half parameters (ZeRO-Offload with the parameters copied
 * back range by range): zero_cpu_step equals zero_cpu_scan, then
 * zero_cpu_update over [0, S), then zero_cpu_commit.
 *
 * zero_cpu_scan -- the global part of the step: reads every accumulator once
 * and fills *out with the overflow flag, the skip decision, the squared norm
 * and the unscale and clipping coefficients. in is the loss-scale state
 * before the step; it is not changed. Errors: as zero_cpu_step.
 *
 * zero_cpu_update -- the update of elements [lo, hi) of every shard (master,
 * m, v in place, param written), from a decision of zero_cpu_scan on the
 * same accumulators and the same state `in`; nothing is written when the
 * decision skips the step. Ranges may be updated in any order and from
 * different calls; every element must be updated exactly once per step.
 * Errors: ZERO_ERR_INVALID_ARG, ZERO_ERR_RANGE (lo, hi).
 *
 * zero_cpu_commit -- advances the loss-scale state after the updates:
 * skip, backoff, growth and t as in zero_cpu_step. Errors:
 * ZERO_ERR_INVALID_ARG.
 */
typedef struct {
    double grad_norm_sq; /* sum of (float)(acc * inv)^2 over every element, in double */
    float inv;           /* (float)(1 / ((R * grad_divisor) * scale)) */
    float clip;          /* the clipping coefficient; 1 without clipping */
    int32_t overflow;    /* some accumulator is inf or NaN */
    int32_t skip;        /* DYNAMIC mode and overflow: the update writes nothing */
    int32_t clipping;    /* clipping is on (max_grad_norm > 0) */
    int32_t reserved;
} zero_cpu_decision;
zero_status zero_cpu_scan(const zero_plan_t* plan, const zero_loss_scale_config* cfg,
                          const zero_loss_scale_state* in, const zero_step_opts* opts,
                          const float* const* acc, int32_t nthreads, zero_cpu_decision* out);
zero_status zero_cpu_update(const zero_plan_t* plan, const zero_loss_scale_state* in, const zero_adamw* hp,
                            const zero_cpu_decision* decision, const float* const* acc, float* const* master,
                            float* const* m, float* const* v, void* const* param, int64_t lo, int64_t hi,
                            int32_t nthreads);
zero_status zero_cpu_commit(const zero_loss_scale_config* cfg, zero_loss_scale_state* inout,
                            const zero_cpu_decision* decision);

/*
 * The CPU step across processes (ZeRO-Offload with one process per rank,
 * each holding only its own shards in host memory):
 *
 * zero_cpu_scan_shard -- zero_cpu_scan restricted to the owners
 * [owner_lo, owner_hi): partial[0] = their sum of (double)((float)(acc *
 * inv))^2, partial[1] = 1 if one of their accumulators is inf or NaN, else
 * 0. Only acc[o] of the owners is read (other entries may be NULL).
 * partial: host, 2 doubles. The ranks all-reduce partial (sum).
 *
 * zero_cpu_decide -- the step's decision from the all-reduced totals
 * (reduced[0] = the squared norm, reduced[1] = the overflow count): the
 * same decision zero_cpu_scan forms from all accumulators in one process.
 *
 * zero_cpu_update_shard -- zero_cpu_update of every element of the owners'
 * shards; only the owners' pointers are read.
 *
 * Every rank then applies zero_cpu_commit with the same decision, so every
 * rank's loss-scale state stays the same. The norm's summation grouping
 * differs from one process's by rounding only.
 * In one process, the totals may come from the GPU that reduced the
 * gradients: with the context holding the host's loss scale
 * (zero_loss_scale SET) and the step's divisor (zero_ctx_set_grad_divisor),
 * ZERO_RS_NORM reduce-scatters leave the squared norm for
 * zero_grad_norm_shard (NULL grads and acc, every owner) and
 * zero_take_overflow gives the flag; zero_cpu_decide then decides a clipped
 * step without a host scan, and zero_cpu_update reads each host accumulator
 * once.
 * Defines: [legal] "CPU Offload"; [instr] ZeRO-2 "Mechanism" (each process
 * updates its own partition).
 * Errors: ZERO_ERR_INVALID_ARG, ZERO_ERR_RANGE (owner range).
 */
zero_status zero_cpu_scan_shard(const zero_plan_t* plan, const zero_loss_scale_config* cfg,
                                const zero_loss_scale_state* in, const zero_step_opts* opts,
                                const float* const* acc, int32_t owner_lo, int32_t owner_hi, int32_t nthreads,
                                double* partial);
zero_status zero_cpu_decide(const zero_plan_t* plan, const zero_loss_scale_config* cfg,
                            const zero_loss_scale_state* in, const zero_step_opts* opts, const double* reduced,
                            zero_cpu_decision* out);
zero_status zero_cpu_update_shard(const zero_plan_t* plan, const zero_loss_scale_state* in, const zero_adamw* hp,
                                  const zero_cpu_decision* decision, const float* const* acc,
                                  float* const* master, float* const* m, float* const* v, void* const* param,
                                  int32_t owner_lo, int32_t owner_hi, int32_t nthreads);

/*
 * Per-call tracing. zero_trace_start makes every later call of the context
 * that queues GPU work bracket that work with two timing events on its
 * stream, up to `capacity` calls (1 .. 2^20; later ones are counted as
 * dropped); it replaces a trace already started. zero_trace_read waits for
 * the recorded events and copies the records, in call order, into out
 * (host, room for max), sets *count (and *dropped, if not NULL), and empties
 * the trace; zero_trace_stop ends tracing and frees its events. Traced
 * calls: the reduce-scatters (ZERO_TRACE_REDUCE_SCATTER, arg = first bucket
 * or -1), including those the scheduler issues on its stream; zero_step /
 * zero_step_ex (ZERO_TRACE_STEP, the norm pass included) and
 * zero_step_shard(_ex) (ZERO_TRACE_STEP, arg = owner_lo); zero_grad_norm_shard
 * (ZERO_TRACE_NORM); zero_step_commit (ZERO_TRACE_COMMIT); zero_gather_layer
 * and zero_gather_layers (ZERO_TRACE_GATHER, arg = first layer), including
 * the scheduler's prefetches. A call made while its stream is being
 * captured into a CUDA graph is not traced. ms is the device time between
 * the two events: the call's own kernels plus anything the stream ran in
 * between. A record whose end event could not be placed has call 0 and
 * ms -1. Host state: calls on one context must not overlap (as for every
 * call on a context).
 * Errors: ZERO_ERR_INVALID_ARG; zero_trace_read: ZERO_ERR_STATE (not
 * started), ZERO_ERR_RANGE (max smaller than the record count; nothing is
 * consumed), ZERO_ERR_CUDA.
 */
#define ZERO_TRACE_REDUCE_SCATTER 1
#define ZERO_TRACE_STEP 2
#define ZERO_TRACE_GATHER 3
#define ZERO_TRACE_NORM 4
#define ZERO_TRACE_COMMIT 5
typedef struct {
    int32_t call;     /* ZERO_TRACE_* */
    int32_t reserved;
    int64_t arg;      /* bucket, layer or owner index; -1 for the whole range */
    float ms;         /* device time between the call's two events */
    float reserved2;
} zero_trace_record;
zero_status zero_trace_start(zero_ctx_t* ctx, int32_t capacity);
zero_status zero_trace_read(zero_ctx_t* ctx, zero_trace_record* out, int32_t max, int32_t* count,
                            int64_t* dropped);
zero_status zero_trace_stop(zero_ctx_t* ctx);

/* zero_sync -- synchronize `stream` and report any pending CUDA error. */
zero_status zero_sync(zero_ctx_t* ctx, void* stream);

/* Copy the calling thread's last error message into buf (NUL-terminated,
 * truncated to n bytes); returns the message's full length. */
size_t zero_last_error(char* buf, size_t n);

/* Library version string (static storage). */
const char* zero_version(void);

#ifdef __cplusplus
}
#endif
#endif
