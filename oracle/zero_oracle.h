/*
 * zero_oracle.h -- TEST INFRASTRUCTURE, not product code.
 *
 * A plain, slow, single-threaded CPU statement of what the ZeRO partitioned
 * mixed-precision step computes. It exists only so that tests can check the
 * CUDA library against something obviously correct. Only tests/,
 * __graft_entry__.smoke() and bench.py's CPU-baseline / reference legs may
 * load it. It shares no code, header, table or constant with the CUDA
 * library under zero_partitioned_mixed_reduce_b200/ and includes nothing
 * from it.
 *
 * Sources (four web pages on "ZeRO Optimization"):
 *  [inferensys-legal]   inferensys glossary, legal pre-training: stages
 *                       bullets (ZeRO-1/2/3), reduce-scatter / bandwidth
 *                       bullets, mixed-precision bullets.
 *  [inferensys-instr]   inferensys glossary, instruction tuning: ZeRO-1/2/3
 *                       mechanism bullets, "communication operations"
 *                       bullets, mixed-precision bullets.
 *  [mbrenndoerfer]      "ZeRO Optimization: Optimizer, Gradient, and
 *                       Parameter Partitioning", introduction.
 *  [inferensys-genomic] inferensys glossary, genomic MLOps: stages
 *                       bullets, memory-breakdown bullets and 20B example.
 *
 * Where the pages are silent (the Adam formula, the shard layout, the
 * bucket rule, the loss-scale growth/backoff rule), the oracle follows the
 * readings listed in each function's comment.
 */
#ifndef ZERO_ORACLE_H
#define ZERO_ORACLE_H

#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

/* Half-precision storage formats of parameters and gradients. */
#define ORACLE_BF16 0
#define ORACLE_FP16 1

/* Loss-scaling modes. */
#define ORACLE_SCALE_NONE 0
#define ORACLE_SCALE_STATIC 1
#define ORACLE_SCALE_DYNAMIC 2

/* ---- half formats (IEEE binary16 and bfloat16), from their definitions -- */
float oracle_half_to_float(uint16_t h, int32_t dtype);
uint16_t oracle_float_to_half(float x, int32_t dtype);
void oracle_half_to_float_n(const uint16_t* h, float* out, int64_t n, int32_t dtype);
void oracle_float_to_half_n(const float* x, uint16_t* out, int64_t n, int32_t dtype);

/* ---- flat-buffer layout ---------------------------------------------------
 * sizes_out[0..5] = P, L, S, T, n_buckets, n_layers.
 * offsets[n]: flat offset of each tensor. tensor_bucket[n]: bucket of each
 * tensor. bucket_lo/hi: capacity n each. layer_lo/hi: capacity n each.
 * layer_ids may be NULL (every tensor its own layer).
 * Returns 0 on success, a positive code on invalid input. */
int32_t oracle_layout(const int64_t* numels, int64_t n, int32_t R, int32_t align,
                      int64_t bucket_elems, const int32_t* layer_ids,
                      int64_t* offsets, int64_t* sizes_out,
                      int64_t* tensor_bucket, int64_t* bucket_lo, int64_t* bucket_hi,
                      int64_t* layer_lo, int64_t* layer_hi);

/* ---- AdamW hyper-parameters and the loss-scale state machine ------------- */
typedef struct {
    double lr, beta1, beta2, eps, weight_decay;
} oracle_adamw;

typedef struct {
    int32_t mode;            /* ORACLE_SCALE_* */
    float scale;             /* current loss scale */
    int64_t growth_interval; /* clean steps before growth (DYNAMIC) */
    float growth_factor;     /* 2 */
    float backoff_factor;    /* 0.5 */
    float min_scale;         /* 1 */
    int64_t good;            /* consecutive clean steps since last change */
    int64_t t;               /* number of applied optimizer steps */
    int32_t last_overflow;
    int32_t last_skipped;
    double grad_norm_sq;     /* sum of squared unscaled, averaged grads */
} oracle_fsm;

/* Apply the post-step loss-scale update for one step whose overflow flag is
 * `overflow`. Returns 1 when the optimizer step is to be skipped. */
int32_t oracle_fsm_update(oracle_fsm* st, int32_t overflow);

/* acc[e] = f32(g_0[e]) + f32(g_1[e]) + ... + f32(g_{R-1}[e]), summed in
 * rank order in fp32; grads is rank-major (R x P). Returns 1 if any acc
 * element is not finite. */
int32_t oracle_allreduce_sum(int64_t P, int32_t R, int32_t dtype,
                             const uint16_t* grads, float* acc);

/* One unpartitioned data-parallel step: all-reduce (sum) the R gradient
 * replicas, check overflow, run the loss-scale state machine, and (unless
 * skipped) AdamW on master/m/v followed by the cast of master to the half
 * parameter. All arrays are unpadded, length P; grads is R x P rank-major.
 * Returns 1 when the step was skipped. */
int32_t oracle_step(int64_t P, int32_t R, int32_t dtype, const uint16_t* grads,
                    float* master, float* m, float* v, uint16_t* param,
                    const oracle_adamw* hp, oracle_fsm* st);

/* The same step done the ZeRO way over the padded flat layout of length
 * R*S: each owner o reduce-scatters its range [o*S, (o+1)*S) out of the R
 * full replicas, the overflow flags of all owners are OR-ed, each owner
 * updates only its own shard, and the half parameters are all-gathered into
 * `gathered` (length R*S). grads is R x (R*S) rank-major; master, m, v,
 * param hold shard o at [o*S, (o+1)*S). Returns 1 when skipped. */
int32_t oracle_step_sharded(int64_t S, int32_t R, int32_t dtype, const uint16_t* grads,
                            float* master, float* m, float* v, uint16_t* param,
                            uint16_t* gathered, const oracle_adamw* hp, oracle_fsm* st);

/* One step with gradient accumulation and global-norm clipping (not on the
 * pages; the readings are stated in zero_oracle.c). grads holds n_micro
 * micro-batches, each R x P rank-major, in order. grad_divisor k >= 1 joins
 * R and the loss scale in the unscale; max_grad_norm <= 0 turns clipping
 * off. grad_norm_sq records the norm before clipping. Returns 1 when
 * skipped. */
typedef struct {
    double grad_divisor;
    double max_grad_norm;
} oracle_step_opts;

int32_t oracle_step_ex(int64_t P, int32_t R, int32_t dtype, int32_t n_micro, const uint16_t* grads,
                       float* master, float* m, float* v, uint16_t* param,
                       const oracle_adamw* hp, const oracle_step_opts* opts, oracle_fsm* st);

/* oracle_step_ex on a sample of a model's elements: every argument as for
 * oracle_step_ex, except that the clipping coefficient comes from
 * norm_sq_all, the whole model's squared norm (computed elsewhere), which is
 * also what grad_norm_sq records. The overflow flag covers the sample only,
 * so the sample must contain any non-finite element of the model. With
 * norm_sq_all equal to the sample's own norm it is oracle_step_ex. */
int32_t oracle_step_ex_sample(int64_t P, int32_t R, int32_t dtype, int32_t n_micro, const uint16_t* grads,
                              float* master, float* m, float* v, uint16_t* param,
                              const oracle_adamw* hp, const oracle_step_opts* opts, oracle_fsm* st,
                              double norm_sq_all);

/* ---- per-rank model-state memory (bytes) --------------------------------
 * stage 0 = plain data parallel, 1/2/3 = ZeRO stages; psi parameters, N
 * data-parallel ranks; 2 + 2 + 12 bytes per parameter. */
double oracle_model_state_bytes(int32_t stage, double psi, double N);
/* Bytes of the weights alone held in fp32. */
double oracle_fp32_weight_bytes(double psi);

#ifdef __cplusplus
}
#endif
#endif
