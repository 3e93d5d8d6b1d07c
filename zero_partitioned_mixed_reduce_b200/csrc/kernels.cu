// CUDA kernels of the ZeRO data-parallel hot path for B200 (sm_100a).
//
// The path is bound by HBM bandwidth: about 20 floating-point operations per
// parameter against 2R + 26 bytes moved (fused step), so there is no
// contraction to put on tensor cores. Every kernel streams 8-element vectors
// (16 bytes of half, 32 bytes of fp32 moved with one 256-bit access) through
// a persistent grid of a few blocks per SM, keeps many loads in flight per
// thread, and reduces flags and norms with warp shuffles and one shared-memory
// pass per block. Global decisions (overflow, skip, loss-scale update) are
// taken by the last block of the step kernel to finish, found with an atomic
// counter, so no block ever waits on another and no extra launch is needed.
//
// Arithmetic matches include/zero_b200.h exactly: one IEEE fp32 operation per
// step via __f*_rn intrinsics (the file is also built with --fmad=false),
// IEEE division and square root, round-to-nearest-even casts to half that
// keep subnormals and overflow to infinity.
//
// Pages (all titled "ZeRO Optimization"): inferensys legal pre-training and
// instruction-tuning glossaries for the reduce-scatter, ZeRO-1/2/3 mechanism,
// mixed-precision and loss-scaling bullets; inferensys genomic glossary for
// the 2 + 2 + 12 bytes-per-parameter state.
#include <cuda_bf16.h>
#include <cuda_fp16.h>
#include <cuda_runtime.h>

#include <cfloat>
#include <cstdint>
#include <mutex>
#include <string>

#include "debug_bounds.cuh"
#include "device_common.cuh"
#include "internal.h"

namespace zb {

template <typename T, int CAP>
__device__ __forceinline__ bool ptrs_ok(T* const (&p)[CAP], int n) {
    for (int r = 0; r < n; ++r)
        if (!p[r]) return false;
    return true;
}

// Per-step coefficients. scale and t live on the device (the loss-scale
// state machine may skip steps without the host knowing), so the parts that
// depend on them are formed here, in double, with the same IEEE operations
// the host would use; beta^t comes from the host-built power table.
__device__ __forceinline__ Coef make_coef(const StepParams& sp, int R, float scale, int64_t t1) {
    Coef c;
    const double dscale = sp.mode == ZERO_SCALE_NONE ? 1.0 : static_cast<double>(scale);
    c.inv = __double2float_rn(
        __ddiv_rn(1.0, __dmul_rn(__dmul_rn(static_cast<double>(R), sp.divisor), dscale)));
    c.clip = 1.0f;
    c.dec = sp.dec;
    c.b1f = sp.b1f;
    c.omb1 = sp.omb1;
    c.b2f = sp.b2f;
    c.omb2 = sp.omb2;
    c.epsf = sp.epsf;
    const double2 pw = sp.powtab[t1 < sp.powtab_len ? t1 : sp.powtab_len - 1];
    c.ss = __double2float_rn(__ddiv_rn(sp.lr, __dsub_rn(1.0, pw.x)));
    c.bc2s = __double2float_rn(__dsqrt_rn(__dsub_rn(1.0, pw.y)));
    return c;
}

struct Prologue {
    Coef c;
    int src, dst, skip;
};

// Thread 0 of each block reads the device state once; the block shares it.
__device__ __forceinline__ void read_prologue(const StepParams& sp, int R, Prologue* out,
                                              bool skip_on_flag) {
    if (threadIdx.x == 0) {
        const volatile DevState* st = sp.st;
        const float scale = st->scale;
        const int64_t t1 = st->t + 1;
        const int cur = st->cur;
        if (t1 >= sp.powtab_len) sp.st->err = 1;  // host keeps the table ahead of t
        out->c = make_coef(sp, R, scale, t1);
        out->src = cur;
        out->dst = sp.pingpong ? (cur ^ 1) : cur;
        out->skip = skip_on_flag && sp.mode == ZERO_SCALE_DYNAMIC && st->flag != 0u;
        if (sp.clip) out->c.clip = st->clip;
    }
    __syncthreads();
}

// Loss-scale state machine; one thread. Same rules as the header states. A
// step during which some block raised the device error flag (a bounded wait
// that gave up, a power table behind t) is abandoned: t, the scale, the
// clean-step count and cur keep their values, so with ping-pong state the
// current model is the one from before the step.
__device__ void fsm_apply(const StepParams& sp, DevState* st, bool ovf, double norm) {
    int skipped = 0;
    if (*reinterpret_cast<volatile int32_t*>(&st->err) != 0) {
        skipped = 1;
    } else if (sp.mode == ZERO_SCALE_DYNAMIC) {
        if (ovf) {
            const float s = __fmul_rn(st->scale, sp.backoff);
            st->scale = (s < sp.min_scale) ? sp.min_scale : s;
            st->good = 0;
            skipped = 1;
        } else {
            st->t = st->t + 1;
            st->good = st->good + 1;
            if (st->good >= sp.interval) {
                st->scale = __fmul_rn(st->scale, sp.growth);
                st->good = 0;
            }
            if (sp.pingpong) st->cur ^= 1;
        }
    } else {
        st->t = st->t + 1;
        if (sp.pingpong) st->cur ^= 1;
    }
    st->last_overflow = ovf ? 1 : 0;
    st->last_skipped = skipped;
    st->grad_norm_sq = norm;
    st->flag = 0u;
    st->done = 0u;
    __threadfence();
}

__device__ void fsm_update(const StepParams& sp, DevState* st, double norm) {
    fsm_apply(sp, st, *reinterpret_cast<volatile uint32_t*>(&st->flag) != 0u, norm);
}

// Every block publishes its norm partial and flag; the last block to finish
// sums the partials in block order and runs the state machine -- or, for a
// sharded step, hands its local totals to the caller for a cross-rank
// reduction and a later commit. NW: the block's warps.
template <int NW = kWarps>
__device__ void step_epilogue(const StepParams& sp, double nrm, bool bad) {
    __shared__ double red[NW];
    __shared__ int last;
    const double bn = block_sum<NW>(nrm, red);
    const int any_bad = __syncthreads_or(bad ? 1 : 0);
    if (threadIdx.x == 0) {
        sp.partials[blockIdx.x] = bn;
        if (any_bad) atomicOr(&sp.st->flag, 1u);
        __threadfence();
        const unsigned prev = atomicAdd(&sp.st->done, 1u);
        last = (prev == gridDim.x - 1);
    }
    __syncthreads();
    if (!last) return;
    __threadfence();
    double x = 0.0;
    for (unsigned i = threadIdx.x; i < gridDim.x; i += NW * 32)
        x += *reinterpret_cast<volatile double*>(&sp.partials[i]);
    const double total = block_sum<NW>(x, red);
    if (threadIdx.x == 0) {
        if (sp.partial_out) {
            sp.partial_out[0] = total;
            sp.partial_out[1] = *reinterpret_cast<volatile uint32_t*>(&sp.st->flag) != 0u ? 1.0 : 0.0;
            sp.st->flag = 0u;
            sp.st->done = 0u;
            __threadfence();
        } else {
            fsm_update(sp, sp.st, total);
        }
    }
}

__global__ void fsm_commit_kernel(const __grid_constant__ StepParams sp, const double* reduced) {
    if (threadIdx.x == 0 && blockIdx.x == 0) fsm_apply(sp, sp.st, reduced[1] > 0.0, reduced[0]);
}

// ---------------------------------------------------------------------------
// Fused reduce-scatter + unscale + overflow check + AdamW + cast.
// One pass: read R gradient vectors and master/m/v, write master/m/v/param.
// ---------------------------------------------------------------------------

template <int CAP>
struct FusedArgs {
    StepParams sp;
    const uint4* g[CAP];
    const float* acc[CAP];  // ADD_ACC variant: the owners' accumulators
    float* master[2][CAP];
    float* m[2][CAP];
    float* v[2][CAP];
    uint4* param[2][CAP];
    uint4* full[2][CAP];    // PUSH variant: every rank's full-model parameter buffer
};

// PUSH: each updated parameter vector is also stored into every rank's
// full-model buffer of the set written (the ZeRO-1/2 all-gather of the
// parameters, done by the step); with one process per GPU those stores go
// to peer-mapped memory over NVLink while the step streams HBM.
template <typename H, int RC, bool CLIP, bool ACC = false, bool PUSH = false>
__global__ void __launch_bounds__(kThreads)
    fused_step_kernel(const __grid_constant__ FusedArgs<RC == 0 ? ZERO_MAX_RANKS : RC> a) {
    const StepParams& sp = a.sp;
    const int R = RC > 0 ? RC : sp.R;
    __shared__ Prologue pro;
    read_prologue(sp, R, &pro, false);
    const Coef c = pro.c;
    const int src = pro.src, dst = pro.dst;

    double nrm = 0.0;
    bool bad = false;
    const uint32_t stride = gridDim.x * kThreads;
    const uint32_t vend = static_cast<uint32_t>(sp.oend) * sp.S8;
    uint32_t vi = line_start(static_cast<uint32_t>(sp.obeg) * sp.S8, stride);
    OwnerCursor oc(vi, sp.S8);
    for (; vi < vend; vi += stride) {
        oc.seek(vi);
        const uint32_t o = oc.o;
        const size_t j8 = static_cast<size_t>(vi - oc.base) * 8;
        if (!ZB_IN(vi < sp.T8 && o >= static_cast<uint32_t>(sp.obeg) && o < static_cast<uint32_t>(sp.oend) &&
                       vi - oc.base < sp.S8 && ptrs_ok(a.g, R) && a.master[src][o] && a.m[src][o] &&
                       a.v[src][o] && a.master[dst][o] && a.m[dst][o] && a.v[dst][o] && a.param[dst][o] &&
                       (!PUSH || ptrs_ok(a.full[dst], R)),
                   1, vi))
            continue;
        float acc[8];
        F8 p, m, v;
        if constexpr (RC > 0) {
            uint4 gv[RC];
#pragma unroll
            for (int r = 0; r < RC; ++r) gv[r] = ld_grad(a.g[r] + vi);
            p = ld_f8(a.master[src][o] + j8);
            m = ld_f8(a.m[src][o] + j8);
            v = ld_f8(a.v[src][o] + j8);
            unpack8<H>(gv[0], acc);
#pragma unroll
            for (int r = 1; r < RC; ++r) add8<H>(gv[r], acc);
        } else {
            uint4 g0 = ld_grad(a.g[0] + vi);
            p = ld_f8(a.master[src][o] + j8);
            m = ld_f8(a.m[src][o] + j8);
            v = ld_f8(a.v[src][o] + j8);
            unpack8<H>(g0, acc);
#pragma unroll 4
            for (int r = 1; r < R; ++r) add8<H>(ld_grad(a.g[r] + vi), acc);
        }
        if constexpr (ACC) {
            // the earlier micro-batches' sum, then this one's rank-order sum
            if (!ZB_IN(a.acc[o] != nullptr, 2, vi)) continue;
            const F8 prev = ld_f8(a.acc[o] + j8);
#pragma unroll
            for (int e = 0; e < 8; ++e) acc[e] = __fadd_rn(prev.x[e], acc[e]);
        }
        float out[8];
#pragma unroll
        for (int e = 0; e < 8; ++e) {
            bad |= nonfinite(acc[e]);
            const float g = adamw1<CLIP>(c, acc[e], p.x[e], m.x[e], v.x[e]);
            const double gd = static_cast<double>(g);
            nrm = fma(gd, gd, nrm);
            out[e] = p.x[e];
        }
        st_f8(a.master[dst][o] + j8, p);
        st_f8(a.m[dst][o] + j8, m);
        st_f8(a.v[dst][o] + j8, v);
        const uint4 pk = pack8<H>(out);
        st_u4(a.param[dst][o] + (j8 >> 3), pk);
        if constexpr (PUSH) {
            for (int r = 0; r < R; ++r) st_u4(a.full[dst][r] + vi, pk);
        }
    }
    step_epilogue(sp, nrm, bad);
}

// ---------------------------------------------------------------------------
// The same fused step with the read streams staged through shared memory by
// the Tensor Memory Accelerator, for small R: the per-element read (2R + 12
// bytes) then leaves too few bytes in flight per thread on the register
// path. A block is 16 consumer warps and one producer warp, one block per
// SM. The producer's elected lane issues, per 4096-element shard-local tile,
// 1-D bulk copies (cp.async.bulk, no multicast) of the R gradient segments
// and the master/m/v segments into a 2-stage shared-memory ring; each stage
// has a "full" mbarrier (completed by the copies' transaction bytes) and an
// "empty" mbarrier (completed when all 512 consumer threads have read the
// stage into registers). Consumers release a stage before doing the
// arithmetic, so the next tile's copies overlap the current tile's math and
// no block-wide barrier sits in the loop. Tile indices, shard offsets and
// lengths are 64-bit: a shard may hold more than 2^32 elements. Every
// mbarrier wait gives up after 2 s of %globaltimer: the waiting thread
// records ZERO_ERR_TIMEOUT in the device state and leaves its loop, and the
// producer waits (bounded) for its copies still in flight before the block
// finishes; the last block then abandons the step.
// ---------------------------------------------------------------------------

constexpr int kTmaTile = 4096;
static_assert(kTmaTile == kStagedTile, "the host tiling and the kernel's tile agree");
constexpr int kTmaStages = 2;
constexpr int kTmaConsumers = kTmaTile / 8;        // 8 elements per consumer thread
constexpr int kTmaThreads = kTmaConsumers + 32;    // consumers + one producer warp
constexpr int kTmaWarps = kTmaThreads / 32;
constexpr int kErrTimeout = 2;
// One block per SM: the ring takes 2 x (R x 8 KB + 48 KB) of shared memory.
// At R = 2 and 1.37 G elements per shard, measured in the benchmark step:
// 4096-element tiles at one block per SM ran 2-3 % faster than 2048-element
// tiles at two blocks of 288 threads per SM; 5120- and 6144-element tiles,
// a third stage, and 1024-element tiles with 3-4 stages at 3-4 blocks per SM
// were all slower.
constexpr int kTmaBlocksPerSm = 1;

template <int RC>
struct TmaStage {
    static constexpr int kGradBytes = RC * kTmaTile * 2;
    static constexpr int kBytes = kGradBytes + 3 * kTmaTile * 4;
    static constexpr int kSmem = kTmaStages * kBytes;
};

__device__ __forceinline__ uint32_t smem_u32(const void* p) {
    return static_cast<uint32_t>(__cvta_generic_to_shared(p));
}
__device__ __forceinline__ void mbar_init(uint32_t bar, uint32_t count) {
    asm volatile("mbarrier.init.shared::cta.b64 [%0], %1;" ::"r"(bar), "r"(count) : "memory");
}
__device__ __forceinline__ void mbar_expect_tx(uint32_t bar, uint32_t bytes) {
    asm volatile("mbarrier.arrive.expect_tx.shared::cta.b64 _, [%0], %1;" ::"r"(bar), "r"(bytes) : "memory");
}
__device__ __forceinline__ void mbar_arrive(uint32_t bar) {
    asm volatile("{ .reg .b64 st; mbarrier.arrive.shared::cta.b64 st, [%0]; }" ::"r"(bar) : "memory");
}
__device__ __forceinline__ void bulk_g2s(uint32_t dst, const void* src, uint32_t bytes, uint32_t bar) {
    asm volatile(
        "cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1], %2, [%3];" ::"r"(dst),
        "l"(src), "r"(bytes), "r"(bar)
        : "memory");
}
__device__ __forceinline__ uint64_t global_ns() {
    uint64_t t;
    asm volatile("mov.u64 %0, %globaltimer;" : "=l"(t));
    return t;
}
// True once the phase of `parity` has completed; false after 2 s.
__device__ __forceinline__ bool mbar_wait(uint32_t bar, uint32_t parity) {
    uint64_t t0 = 0;
    for (uint32_t it = 0;; ++it) {
        uint32_t done;
        asm volatile(
            "{ .reg .pred p; mbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2; selp.u32 %0, 1, 0, p; }"
            : "=r"(done)
            : "r"(bar), "r"(parity)
            : "memory");
        if (done) return true;
        if ((it & 63) == 0) {
            const uint64_t t = global_ns();
            if (t0 == 0)
                t0 = t;
            else if (t - t0 > 2000000000ull)
                return false;
        }
    }
}
__device__ __forceinline__ uint4 lds16(const void* p) { return *reinterpret_cast<const uint4*>(p); }

template <typename H, int RC, bool CLIP>
__global__ void __launch_bounds__(kTmaThreads, kTmaBlocksPerSm)
    fused_step_tma_kernel(const __grid_constant__ FusedArgs<RC> a, uint64_t tiles_per_shard) {
    using L = TmaStage<RC>;
    extern __shared__ __align__(128) unsigned char smem[];
    __shared__ __align__(8) uint64_t full[kTmaStages], empty[kTmaStages];
    const StepParams& sp = a.sp;
    __shared__ Prologue pro;
    read_prologue(sp, RC, &pro, false);
    const Coef c = pro.c;
    const int src = pro.src, dst = pro.dst;
    const uint64_t S = static_cast<uint64_t>(sp.S8) * 8;
    const uint64_t tps = tiles_per_shard;
    const uint64_t t0 = static_cast<uint64_t>(sp.obeg) * tps, t1 = static_cast<uint64_t>(sp.oend) * tps;
    // this block's tiles: t0 + blockIdx.x + k * gridDim.x, k < count
    const uint64_t G = gridDim.x, first = t0 + blockIdx.x;
    const uint64_t count = first < t1 ? (t1 - first + G - 1) / G : 0;
    if (threadIdx.x == 0) {
        for (int s = 0; s < kTmaStages; ++s) {
            mbar_init(smem_u32(&full[s]), 1);
            mbar_init(smem_u32(&empty[s]), kTmaConsumers);
        }
        asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
    }
    __syncthreads();
    double nrm = 0.0;
    bool bad = false;
    if (threadIdx.x >= kTmaConsumers) {
        // producer warp: one lane issues every copy
        if (threadIdx.x == kTmaConsumers) {
            uint64_t k = 0, dropped = ~0ull;
            for (; k < count; ++k) {
                const int s = static_cast<int>(k % kTmaStages);
                if (k >= kTmaStages &&
                    !mbar_wait(smem_u32(&empty[s]), static_cast<uint32_t>((k / kTmaStages - 1) & 1))) {
                    sp.st->err = kErrTimeout;
                    break;
                }
                const uint64_t tile = first + k * G;
                const uint64_t o = tile / tps;
                const uint64_t j0 = (tile - o * tps) * kTmaTile;
                const uint32_t len = static_cast<uint32_t>(S - j0 < kTmaTile ? S - j0 : kTmaTile);
                // test support (a tile whose copies never come), or a failed
                // check of the debug build: the consumers' wait runs out
                if (tile == sp.drop_tile ||
                    !ZB_IN(o >= static_cast<uint64_t>(sp.obeg) && o < static_cast<uint64_t>(sp.oend) && j0 < S &&
                               len % 8 == 0 && j0 + len <= S && ptrs_ok(a.g, RC) && a.master[src][o] &&
                               a.m[src][o] && a.v[src][o],
                           3, tile)) {
                    dropped = k;
                    continue;
                }
                unsigned char* base = smem + s * L::kBytes;
                const uint32_t bar = smem_u32(&full[s]);
                asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
                mbar_expect_tx(bar, len * (RC * 2 + 12));
#pragma unroll
                for (int r = 0; r < RC; ++r)
                    bulk_g2s(smem_u32(base + r * kTmaTile * 2),
                             reinterpret_cast<const uint16_t*>(a.g[r]) + o * S + j0, len * 2, bar);
                bulk_g2s(smem_u32(base + L::kGradBytes), a.master[src][o] + j0, len * 4, bar);
                bulk_g2s(smem_u32(base + L::kGradBytes + kTmaTile * 4), a.m[src][o] + j0, len * 4, bar);
                bulk_g2s(smem_u32(base + L::kGradBytes + 2 * kTmaTile * 4), a.v[src][o] + j0, len * 4, bar);
            }
            // copies still in flight land before the block's shared memory is released
            for (uint64_t q = k > kTmaStages ? k - kTmaStages : 0; q < k; ++q)
                if (q != dropped)
                    mbar_wait(smem_u32(&full[q % kTmaStages]), static_cast<uint32_t>((q / kTmaStages) & 1));
        }
    } else {
        for (uint64_t k = 0; k < count; ++k) {
            const int s = static_cast<int>(k % kTmaStages);
            if (!mbar_wait(smem_u32(&full[s]), static_cast<uint32_t>((k / kTmaStages) & 1))) {
                sp.st->err = kErrTimeout;
                break;
            }
            const uint64_t tile = first + k * G;
            const uint64_t o = tile / tps;
            const uint64_t j0 = (tile - o * tps) * kTmaTile;
            const uint32_t len = static_cast<uint32_t>(S - j0 < kTmaTile ? S - j0 : kTmaTile);
            const uint32_t e0 = threadIdx.x * 8;
            const bool act = e0 < len;
            uint4 gv[RC];
            F8 p, m, v;
            if (act) {
                const unsigned char* base = smem + s * L::kBytes;
#pragma unroll
                for (int r = 0; r < RC; ++r) gv[r] = lds16(base + r * kTmaTile * 2 + e0 * 2);
                const float* ps = reinterpret_cast<const float*>(base + L::kGradBytes);
                *reinterpret_cast<uint4*>(&p.x[0]) = lds16(ps + e0);
                *reinterpret_cast<uint4*>(&p.x[4]) = lds16(ps + e0 + 4);
                *reinterpret_cast<uint4*>(&m.x[0]) = lds16(ps + kTmaTile + e0);
                *reinterpret_cast<uint4*>(&m.x[4]) = lds16(ps + kTmaTile + e0 + 4);
                *reinterpret_cast<uint4*>(&v.x[0]) = lds16(ps + 2 * kTmaTile + e0);
                *reinterpret_cast<uint4*>(&v.x[4]) = lds16(ps + 2 * kTmaTile + e0 + 4);
            }
            mbar_arrive(smem_u32(&empty[s]));  // this thread is done with stage s
            if (!act) continue;
            float acc[8];
            unpack8<H>(gv[0], acc);
#pragma unroll
            for (int r = 1; r < RC; ++r) add8<H>(gv[r], acc);
            float out[8];
#pragma unroll
            for (int e = 0; e < 8; ++e) {
                bad |= nonfinite(acc[e]);
                const double gd = static_cast<double>(adamw1<CLIP>(c, acc[e], p.x[e], m.x[e], v.x[e]));
                nrm = fma(gd, gd, nrm);
                out[e] = p.x[e];
            }
            const uint64_t jj = j0 + e0;
            if (ZB_IN(jj + 8 <= S && a.master[dst][o] && a.m[dst][o] && a.v[dst][o] && a.param[dst][o], 4, jj)) {
                st_f8(a.master[dst][o] + jj, p);
                st_f8(a.m[dst][o] + jj, m);
                st_f8(a.v[dst][o] + jj, v);
                st_u4(a.param[dst][o] + (jj >> 3), pack8<H>(out));
            }
        }
    }
    step_epilogue<kTmaWarps>(sp, nrm, bad);
}

// ---------------------------------------------------------------------------
// Two-pass step: AdamW from the fp32 accumulators written by the
// reduce-scatter kernel. In place on set cur, or from set cur into set 1-cur
// when both sets are given (ping-pong); skipped (no state written) in
// DYNAMIC mode when the reduce-scatter raised the overflow flag. The norm is
// always formed from the accumulators. This register kernel runs the push
// variant; without the push the staged kernel below runs.
// ---------------------------------------------------------------------------

struct AccArgs {
    StepParams sp;
    const float* acc[ZERO_MAX_RANKS];
    float* master[2][ZERO_MAX_RANKS];
    float* m[2][ZERO_MAX_RANKS];
    float* v[2][ZERO_MAX_RANKS];
    uint4* param[2][ZERO_MAX_RANKS];
    uint4* full[2][ZERO_MAX_RANKS];  // PUSH variant, as for the fused step
};

template <typename H, bool CLIP, bool PUSH = false>
__global__ void __launch_bounds__(kThreads) step_from_acc_kernel(const __grid_constant__ AccArgs a) {
    const StepParams& sp = a.sp;
    __shared__ Prologue pro;
    // a sharded step (partial_out) defers the skip to the cross-rank commit:
    // it always writes set 1-cur, and only the commit decides whether cur flips
    read_prologue(sp, sp.R, &pro, sp.partial_out == nullptr);
    const Coef c = pro.c;
    const int src = pro.src, dst = pro.dst;
    const bool skip = pro.skip != 0;

    double nrm = 0.0;
    const uint32_t stride = gridDim.x * kThreads;
    const uint32_t vend = static_cast<uint32_t>(sp.oend) * sp.S8;
    uint32_t vi = line_start(static_cast<uint32_t>(sp.obeg) * sp.S8, stride);
    OwnerCursor oc(vi, sp.S8);
    for (; vi < vend; vi += stride) {
        oc.seek(vi);
        const uint32_t o = oc.o;
        const size_t j8 = static_cast<size_t>(vi - oc.base) * 8;
        if (!ZB_IN(o >= static_cast<uint32_t>(sp.obeg) && o < static_cast<uint32_t>(sp.oend) && vi - oc.base < sp.S8 &&
                       a.acc[o] && (skip || (a.master[src][o] && a.m[src][o] && a.v[src][o] &&
                                             a.master[dst][o] && a.m[dst][o] && a.v[dst][o] && a.param[dst][o] &&
                                             (!PUSH || ptrs_ok(a.full[dst], sp.R)))),
                   5, vi))
            continue;
        const F8 acc = ld_f8(a.acc[o] + j8);
        if (skip) {
#pragma unroll
            for (int e = 0; e < 8; ++e) {
                const double gd = static_cast<double>(__fmul_rn(acc.x[e], c.inv));
                nrm = fma(gd, gd, nrm);
            }
            continue;
        }
        F8 p = ld_f8(a.master[src][o] + j8);
        F8 m = ld_f8(a.m[src][o] + j8);
        F8 v = ld_f8(a.v[src][o] + j8);
        float out[8];
#pragma unroll
        for (int e = 0; e < 8; ++e) {
            const float g = adamw1<CLIP>(c, acc.x[e], p.x[e], m.x[e], v.x[e]);
            const double gd = static_cast<double>(g);
            nrm = fma(gd, gd, nrm);
            out[e] = p.x[e];
        }
        st_f8(a.master[dst][o] + j8, p);
        st_f8(a.m[dst][o] + j8, m);
        st_f8(a.v[dst][o] + j8, v);
        const uint4 pk = pack8<H>(out);
        st_u4(a.param[dst][o] + (j8 >> 3), pk);
        if constexpr (PUSH) {
            for (int r = 0; r < sp.R; ++r) st_u4(a.full[dst][r] + vi, pk);
        }
    }
    step_epilogue(sp, nrm, false);
}

// ---------------------------------------------------------------------------
// The two-pass step from the fp32 accumulators, staged like the fused step
// at R <= 2: whatever R, it reads one fp32 accumulator and master/m/v (16
// bytes) and writes 14, the R = 2 fused step's mix, where staging wins. Per
// 4096-element shard-local tile the producer warp's elected lane bulk-copies
// the accumulator segment and, unless the step is skipped, the master/m/v
// segments into the 2-stage ring; 16 consumer warps release a stage once read
// and then do the arithmetic. A skipped step (DYNAMIC, the reduce-scatter
// raised the overflow flag) loads only the accumulators and forms the norm.
// Same bounded waits as the fused staged kernel. The push variant runs on the
// register kernel above.
// ---------------------------------------------------------------------------

struct TmaAccStage {
    static constexpr int kBytes = 4 * kTmaTile * 4;  // acc, master, m, v
    static constexpr int kSmem = kTmaStages * kBytes;
};

template <typename H, bool CLIP>
__global__ void __launch_bounds__(kTmaThreads, kTmaBlocksPerSm)
    step_from_acc_tma_kernel(const __grid_constant__ AccArgs a, uint64_t tiles_per_shard) {
    using L = TmaAccStage;
    extern __shared__ __align__(128) unsigned char smem[];
    __shared__ __align__(8) uint64_t full[kTmaStages], empty[kTmaStages];
    const StepParams& sp = a.sp;
    __shared__ Prologue pro;
    read_prologue(sp, sp.R, &pro, sp.partial_out == nullptr);
    const Coef c = pro.c;
    const int src = pro.src, dst = pro.dst;
    const bool skip = pro.skip != 0;
    const uint64_t S = static_cast<uint64_t>(sp.S8) * 8;
    const uint64_t tps = tiles_per_shard;
    const uint64_t t0 = static_cast<uint64_t>(sp.obeg) * tps, t1 = static_cast<uint64_t>(sp.oend) * tps;
    const uint64_t G = gridDim.x, first = t0 + blockIdx.x;
    const uint64_t count = first < t1 ? (t1 - first + G - 1) / G : 0;
    if (threadIdx.x == 0) {
        for (int s = 0; s < kTmaStages; ++s) {
            mbar_init(smem_u32(&full[s]), 1);
            mbar_init(smem_u32(&empty[s]), kTmaConsumers);
        }
        asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
    }
    __syncthreads();
    double nrm = 0.0;
    if (threadIdx.x >= kTmaConsumers) {
        if (threadIdx.x == kTmaConsumers) {
            uint64_t k = 0, dropped = ~0ull;
            for (; k < count; ++k) {
                const int s = static_cast<int>(k % kTmaStages);
                if (k >= kTmaStages &&
                    !mbar_wait(smem_u32(&empty[s]), static_cast<uint32_t>((k / kTmaStages - 1) & 1))) {
                    sp.st->err = kErrTimeout;
                    break;
                }
                const uint64_t tile = first + k * G;
                const uint64_t o = tile / tps;
                const uint64_t j0 = (tile - o * tps) * kTmaTile;
                const uint32_t len = static_cast<uint32_t>(S - j0 < kTmaTile ? S - j0 : kTmaTile);
                if (!ZB_IN(o >= static_cast<uint64_t>(sp.obeg) && o < static_cast<uint64_t>(sp.oend) && j0 < S &&
                               len % 8 == 0 && j0 + len <= S && a.acc[o] &&
                               (skip || (a.master[src][o] && a.m[src][o] && a.v[src][o])),
                           14, tile)) {
                    dropped = k;
                    continue;
                }
                unsigned char* base = smem + s * L::kBytes;
                const uint32_t bar = smem_u32(&full[s]);
                asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
                mbar_expect_tx(bar, len * (skip ? 4 : 16));
                bulk_g2s(smem_u32(base), a.acc[o] + j0, len * 4, bar);
                if (!skip) {
                    bulk_g2s(smem_u32(base + kTmaTile * 4), a.master[src][o] + j0, len * 4, bar);
                    bulk_g2s(smem_u32(base + 2 * kTmaTile * 4), a.m[src][o] + j0, len * 4, bar);
                    bulk_g2s(smem_u32(base + 3 * kTmaTile * 4), a.v[src][o] + j0, len * 4, bar);
                }
            }
            for (uint64_t q = k > kTmaStages ? k - kTmaStages : 0; q < k; ++q)
                if (q != dropped)
                    mbar_wait(smem_u32(&full[q % kTmaStages]), static_cast<uint32_t>((q / kTmaStages) & 1));
        }
    } else {
        for (uint64_t k = 0; k < count; ++k) {
            const int s = static_cast<int>(k % kTmaStages);
            if (!mbar_wait(smem_u32(&full[s]), static_cast<uint32_t>((k / kTmaStages) & 1))) {
                sp.st->err = kErrTimeout;
                break;
            }
            const uint64_t tile = first + k * G;
            const uint64_t o = tile / tps;
            const uint64_t j0 = (tile - o * tps) * kTmaTile;
            const uint32_t len = static_cast<uint32_t>(S - j0 < kTmaTile ? S - j0 : kTmaTile);
            const uint32_t e0 = threadIdx.x * 8;
            const bool act = e0 < len;
            F8 g, p, m, v;
            if (act) {
                const float* ps = reinterpret_cast<const float*>(smem + s * L::kBytes);
                *reinterpret_cast<uint4*>(&g.x[0]) = lds16(ps + e0);
                *reinterpret_cast<uint4*>(&g.x[4]) = lds16(ps + e0 + 4);
                if (!skip) {
                    *reinterpret_cast<uint4*>(&p.x[0]) = lds16(ps + kTmaTile + e0);
                    *reinterpret_cast<uint4*>(&p.x[4]) = lds16(ps + kTmaTile + e0 + 4);
                    *reinterpret_cast<uint4*>(&m.x[0]) = lds16(ps + 2 * kTmaTile + e0);
                    *reinterpret_cast<uint4*>(&m.x[4]) = lds16(ps + 2 * kTmaTile + e0 + 4);
                    *reinterpret_cast<uint4*>(&v.x[0]) = lds16(ps + 3 * kTmaTile + e0);
                    *reinterpret_cast<uint4*>(&v.x[4]) = lds16(ps + 3 * kTmaTile + e0 + 4);
                }
            }
            mbar_arrive(smem_u32(&empty[s]));  // this thread is done with stage s
            if (!act) continue;
            if (skip) {
#pragma unroll
                for (int e = 0; e < 8; ++e) {
                    const double gd = static_cast<double>(__fmul_rn(g.x[e], c.inv));
                    nrm = fma(gd, gd, nrm);
                }
                continue;
            }
            float out[8];
#pragma unroll
            for (int e = 0; e < 8; ++e) {
                const double gd = static_cast<double>(adamw1<CLIP>(c, g.x[e], p.x[e], m.x[e], v.x[e]));
                nrm = fma(gd, gd, nrm);
                out[e] = p.x[e];
            }
            const uint64_t jj = j0 + e0;
            if (ZB_IN(jj + 8 <= S && a.master[dst][o] && a.m[dst][o] && a.v[dst][o] && a.param[dst][o], 15, jj)) {
                st_f8(a.master[dst][o] + jj, p);
                st_f8(a.m[dst][o] + jj, m);
                st_f8(a.v[dst][o] + jj, v);
                st_u4(a.param[dst][o] + (jj >> 3), pack8<H>(out));
            }
        }
    }
    step_epilogue<kTmaWarps>(sp, nrm, false);
}

// ---------------------------------------------------------------------------
// Global gradient norm for clipping, before the step: one read-only pass. The
// two-pass path reads the accumulators (clip_norm_kernel); the fused path
// reads the R gradient replicas and reduces them in rank order exactly as the
// step will (grad_norm_kernel). The last block to finish turns the sum of
// squares of the unscaled gradient into the clipping coefficient
// min(1, max_norm / (||g|| + 1e-6)) (in double) and stores it in the device
// state for the step kernel.
// ---------------------------------------------------------------------------

constexpr int kNormUnroll = 4;

// 1 / ((R * divisor) * scale), rounded once to fp32; shared by the block.
__device__ __forceinline__ float block_unscale(const StepParams& sp) {
    __shared__ float s_inv;
    if (threadIdx.x == 0) {
        const volatile DevState* st = sp.st;
        const double dscale = sp.mode == ZERO_SCALE_NONE ? 1.0 : static_cast<double>(st->scale);
        s_inv = __double2float_rn(
            __ddiv_rn(1.0, __dmul_rn(__dmul_rn(static_cast<double>(sp.R), sp.divisor), dscale)));
    }
    __syncthreads();
    return s_inv;
}

// min(1, max_norm / (sqrt(norm_sq) + 1e-6)), in double, rounded once to fp32.
__device__ __forceinline__ float clip_coefficient(double max_norm, double norm_sq) {
    const double cd = __ddiv_rn(max_norm, __dadd_rn(__dsqrt_rn(norm_sq), 1e-6));
    return __double2float_rn(cd < 1.0 ? cd : 1.0);
}

// Every block publishes its partial; the last one stores the coefficient, or,
// for a shard range (partial_out), the range's sum for a cross-rank reduction.
__device__ void norm_to_clip(const StepParams& sp, double nrm) {
    __shared__ double red[kWarps];
    __shared__ int last;
    const double bn = block_sum(nrm, red);
    if (threadIdx.x == 0) {
        sp.partials[blockIdx.x] = bn;
        __threadfence();
        last = (atomicAdd(&sp.st->done, 1u) == gridDim.x - 1);
    }
    __syncthreads();
    if (!last) return;
    __threadfence();
    double x = 0.0;
    for (unsigned i = threadIdx.x; i < gridDim.x; i += kThreads)
        x += *reinterpret_cast<volatile double*>(&sp.partials[i]);
    const double total = block_sum(x, red);
    if (threadIdx.x == 0) {
        if (sp.partial_out) {
            // a shard range's part of the norm, for a cross-rank sum
            sp.partial_out[0] = total;
            sp.partial_out[1] = 0.0;
        } else {
            sp.st->clip = clip_coefficient(sp.max_norm, total);
        }
        sp.st->done = 0u;
        __threadfence();
    }
}

// The coefficient from a norm already summed across ranks.
__global__ void clip_from_norm_kernel(const __grid_constant__ StepParams sp, const double* norm_sq) {
    if (threadIdx.x == 0 && blockIdx.x == 0) {
        sp.st->clip = clip_coefficient(sp.max_norm, *norm_sq);
        __threadfence();
    }
}

struct NormArgs {
    StepParams sp;
    const float* acc[ZERO_MAX_RANKS];
};

__global__ void __launch_bounds__(kThreads) clip_norm_kernel(const __grid_constant__ NormArgs a) {
    const StepParams& sp = a.sp;
    const float inv = block_unscale(sp);
    double nrm = 0.0;
    const uint32_t stride = gridDim.x * kThreads;
    const uint32_t vend = static_cast<uint32_t>(sp.oend) * sp.S8;
    uint32_t vi = line_start(static_cast<uint32_t>(sp.obeg) * sp.S8, stride);
    OwnerCursor oc(vi, sp.S8);
    // a short read-only pass: keep kNormUnroll vectors per thread in flight
    for (; vi < vend; vi += kNormUnroll * stride) {
        F8 acc[kNormUnroll];
#pragma unroll
        for (int u = 0; u < kNormUnroll; ++u) {
            const uint32_t vu = vi + u * stride;
            bool take = vu < vend;
            if (take) {
                oc.seek(vu);
                take = ZB_IN(oc.o >= static_cast<uint32_t>(sp.obeg) && oc.o < static_cast<uint32_t>(sp.oend) &&
                                 vu - oc.base < sp.S8 && a.acc[oc.o],
                             6, vu);
            }
            if (take) {
                acc[u] = ld_f8(a.acc[oc.o] + static_cast<size_t>(vu - oc.base) * 8);
            } else {
#pragma unroll
                for (int e = 0; e < 8; ++e) acc[u].x[e] = 0.0f;
            }
        }
#pragma unroll
        for (int u = 0; u < kNormUnroll; ++u)
#pragma unroll
            for (int e = 0; e < 8; ++e) {
                const double gd = static_cast<double>(__fmul_rn(acc[u].x[e], inv));
                nrm = fma(gd, gd, nrm);
            }
    }
    norm_to_clip(sp, nrm);
}

template <int CAP>
struct GradNormArgs {
    StepParams sp;
    const uint4* g[CAP];
};

// The norm of the reduced gradient straight from the R half replicas (the
// fused path has no accumulator): per 8-element vector the replicas are
// summed in fp32 in rank order, as in the step, then unscaled and squared in
// double. Gradients only: no state is read.
template <typename H, int RC>
__global__ void __launch_bounds__(kThreads)
    grad_norm_kernel(const __grid_constant__ GradNormArgs<RC == 0 ? ZERO_MAX_RANKS : RC> a) {
    const StepParams& sp = a.sp;
    const int R = RC > 0 ? RC : sp.R;
    const float inv = block_unscale(sp);
    double nrm = 0.0;
    const uint32_t stride = gridDim.x * kThreads;
    const uint32_t vend = static_cast<uint32_t>(sp.oend) * sp.S8;
    for (uint32_t vi = line_start(static_cast<uint32_t>(sp.obeg) * sp.S8, stride); vi < vend; vi += stride) {
        if (!ZB_IN(vi >= static_cast<uint32_t>(sp.obeg) * sp.S8 && vi < sp.T8 && ptrs_ok(a.g, R), 7, vi)) continue;
        float acc[8];
        if constexpr (RC > 0) {
            uint4 gv[RC];
#pragma unroll
            for (int r = 0; r < RC; ++r) gv[r] = ld_grad(a.g[r] + vi);
            unpack8<H>(gv[0], acc);
#pragma unroll
            for (int r = 1; r < RC; ++r) add8<H>(gv[r], acc);
        } else {
            unpack8<H>(ld_grad(a.g[0] + vi), acc);
#pragma unroll 4
            for (int r = 1; r < R; ++r) add8<H>(ld_grad(a.g[r] + vi), acc);
        }
#pragma unroll
        for (int e = 0; e < 8; ++e) {
            const double gd = static_cast<double>(__fmul_rn(acc[e], inv));
            nrm = fma(gd, gd, nrm);
        }
    }
    norm_to_clip(sp, nrm);
}

// ---------------------------------------------------------------------------
// Bucketed reduce-scatter into the owners' fp32 accumulators.
// Flat range [lo, hi): an unaligned head and tail are done element by
// element, the aligned body with 8-element vectors (S is a multiple of 8, so
// an aligned vector never straddles two shards).
// ---------------------------------------------------------------------------

template <int CAP>
struct RsArgs {
    int64_t lo, hi, S;
    uint32_t S8, v0, v1;   // aligned body in vectors: [v0, v1)
    int64_t head_end, tail_begin;
    int32_t R;
    DevState* st;
    RsNorm norm;           // norm.partials == nullptr: no norm share
    const uint4* g[CAP];
    float* acc[CAP];
};

// 1 / ((R * divisor) * scale) rounded once to fp32, as the step computes it;
// shared by the block (every thread of the block must call it).
__device__ __forceinline__ float block_unscale_rs(const RsNorm& n, int32_t R, const DevState* st) {
    __shared__ float s_inv;
    if (threadIdx.x == 0) {
        const volatile DevState* vs = st;
        const double dscale = n.mode == ZERO_SCALE_NONE ? 1.0 : static_cast<double>(vs->scale);
        s_inv = __double2float_rn(
            __ddiv_rn(1.0, __dmul_rn(__dmul_rn(static_cast<double>(R), n.divisor), dscale)));
    }
    __syncthreads();
    return s_inv;
}

// The launch's share of the squared norm: every block publishes its partial,
// the last one sums them in block order into *n.out and re-arms the counter.
__device__ void rs_norm_finish(const RsNorm& n, double nrm) {
    __shared__ double red[kWarps];
    __shared__ int last;
    const double bn = block_sum(nrm, red);
    if (threadIdx.x == 0) {
        if (ZB_IN(blockIdx.x < n.cap, 12, blockIdx.x)) n.partials[blockIdx.x] = bn;
        __threadfence();
        last = (atomicAdd(n.done, 1u) == gridDim.x - 1);
    }
    __syncthreads();
    if (!last) return;
    __threadfence();
    double x = 0.0;
    for (unsigned i = threadIdx.x; i < gridDim.x; i += kThreads)
        if (ZB_IN(i < n.cap, 12, i)) x += *reinterpret_cast<volatile double*>(&n.partials[i]);
    const double total = block_sum(x, red);
    if (threadIdx.x == 0) {
        *n.out = total;
        *n.done = 0u;
        __threadfence();
    }
}

template <typename H, int RC, bool ACCUM>
__global__ void __launch_bounds__(kThreads)
    reduce_scatter_kernel(const __grid_constant__ RsArgs<RC == 0 ? ZERO_MAX_RANKS : RC> a) {
    const int R = RC > 0 ? RC : a.R;
    bool bad = false;
    const bool with_norm = a.norm.partials != nullptr;  // uniform over the grid
    const float inv = with_norm ? block_unscale_rs(a.norm, R, a.st) : 0.0f;
    double nrm = 0.0;
    const uint32_t stride = gridDim.x * kThreads;
    const uint32_t tid = blockIdx.x * kThreads + threadIdx.x;
    uint32_t vi = line_start(a.v0, stride);
    OwnerCursor oc(vi, a.S8);
    for (; vi < a.v1; vi += stride) {
        oc.seek(vi);
        if (!ZB_IN(vi >= a.v0 && oc.o < static_cast<uint32_t>(R) && vi - oc.base < a.S8 && a.acc[oc.o] &&
                       ptrs_ok(a.g, R),
                   8, vi))
            continue;
        float acc[8];
        if constexpr (RC > 0) {
            uint4 gv[RC];
#pragma unroll
            for (int r = 0; r < RC; ++r) gv[r] = ld_grad(a.g[r] + vi);
            unpack8<H>(gv[0], acc);
#pragma unroll
            for (int r = 1; r < RC; ++r) add8<H>(gv[r], acc);
        } else {
            unpack8<H>(ld_grad(a.g[0] + vi), acc);
#pragma unroll 4
            for (int r = 1; r < R; ++r) add8<H>(ld_grad(a.g[r] + vi), acc);
        }
        float* dst = a.acc[oc.o] + static_cast<size_t>(vi - oc.base) * 8;
        F8 out;
        if constexpr (ACCUM) {
            const F8 old = ld_f8(dst);
#pragma unroll
            for (int e = 0; e < 8; ++e) acc[e] = __fadd_rn(old.x[e], acc[e]);
        }
#pragma unroll
        for (int e = 0; e < 8; ++e) {
            bad |= nonfinite(acc[e]);
            out.x[e] = acc[e];
        }
        st_f8(dst, out);
        if (with_norm) {
            // the unscaled gradient as the step will form it, squared in double
#pragma unroll
            for (int e = 0; e < 8; ++e) {
                const double gd = static_cast<double>(__fmul_rn(acc[e], inv));
                nrm = fma(gd, gd, nrm);
            }
        }
    }
    // unaligned edges, element by element
    const int64_t nhead = a.head_end - a.lo;
    const int64_t ntail = a.hi - a.tail_begin;
    if (tid < nhead + ntail) {
        const int64_t i = tid < nhead ? a.lo + tid : a.tail_begin + (tid - nhead);
        const int64_t o = i / a.S;
        // a guarded block, not a return: every thread must reach the barrier below
        if (ZB_IN(i >= a.lo && i < a.hi && o < R && a.acc[o] && ptrs_ok(a.g, R), 9, i)) {
            float s = H::one(ld_grad1(reinterpret_cast<const uint16_t*>(a.g[0]) + i));
            for (int r = 1; r < R; ++r)
                s = __fadd_rn(s, H::one(ld_grad1(reinterpret_cast<const uint16_t*>(a.g[r]) + i)));
            float* dst = a.acc[o] + (i - o * a.S);
            if constexpr (ACCUM) s = __fadd_rn(*dst, s);
            bad |= nonfinite(s);
            *dst = s;
            if (with_norm) {
                const double gd = static_cast<double>(__fmul_rn(s, inv));
                nrm = fma(gd, gd, nrm);
            }
        }
    }
    if (__syncthreads_or(bad ? 1 : 0) && threadIdx.x == 0) atomicOr(&a.st->flag, 1u);
    if (with_norm) rs_norm_finish(a.norm, nrm);
}

// ---------------------------------------------------------------------------
// ZeRO-3 gather of one or more consecutive layers from the current parameter
// set, in one launch. The layers' ranges are cut into 8-element slots
// numbered across the bucket; a thread's slots, and so the flat positions it
// reads, only grow, so layer and owner are tracked incrementally. Slots of a
// layer whose start is 8-aligned move as one 16-byte vector, several per
// thread in flight; partial and unaligned slots go element by element.
// ---------------------------------------------------------------------------

struct GatherManyArgs {
    int32_t nl;
    int32_t R;
    int64_t S;
    uint32_t S8;
    uint32_t total_slots;
    const DevState* st;
    const uint16_t* param[2][ZERO_MAX_RANKS];
    int64_t lo[ZERO_GATHER_MAX_LAYERS];
    int64_t n[ZERO_GATHER_MAX_LAYERS];
    uint16_t* out[ZERO_GATHER_MAX_LAYERS];
    uint32_t slot0[ZERO_GATHER_MAX_LAYERS + 1];  // first slot of each layer; slot0[nl] = total
    int32_t aligned[ZERO_GATHER_MAX_LAYERS];
};

// Vectors in flight per thread: 4 for launches of up to kGatherWideSlots
// slots, 8 above. Inside the benchmark step 8 gathered a 100M-element layer 4 %
// faster (and a 50M-element layer 3 %), but a 32M-element bucket 5 % slower:
// its 90 registers leave 2 blocks per SM instead of 4, and a short launch
// then pays a longer tail.
constexpr uint32_t kGatherWideSlots = 1u << 22;

template <int kGatherUnroll>
__global__ void __launch_bounds__(kThreads) gather_many_kernel(const __grid_constant__ GatherManyArgs a) {
    __shared__ int s_cur;
    if (threadIdx.x == 0) s_cur = reinterpret_cast<const volatile DevState*>(a.st)->cur;
    __syncthreads();
    const int cur = s_cur;
    const uint32_t stride = gridDim.x * kThreads;
    uint32_t s = blockIdx.x * kThreads + threadIdx.x;
    if (s >= a.total_slots) return;
    // the current layer's values live in registers; they are reloaded only
    // when the thread's slot crosses into the next layer
    int l = 0;
    while (s >= a.slot0[l + 1]) ++l;
    uint32_t first = a.slot0[l], end = a.slot0[l + 1];
    int64_t lo = a.lo[l], n = a.n[l];
    uint16_t* out = a.out[l];
    bool al = a.aligned[l] != 0;
    OwnerCursor oc(static_cast<uint32_t>(lo / 8), a.S8);
    for (; s < a.total_slots; s += kGatherUnroll * stride) {
        // pass 1: issue the loads of up to kGatherUnroll whole aligned slots
        // (partial or unaligned slots are copied element by element here)
        uint4 q[kGatherUnroll];
        uint16_t* dst[kGatherUnroll];
#pragma unroll
        for (int u = 0; u < kGatherUnroll; ++u) {
            dst[u] = nullptr;
            const uint32_t su = s + u * stride;
            if (su >= a.total_slots) continue;
            if (su >= end) {
                do ++l; while (su >= a.slot0[l + 1]);
                first = a.slot0[l];
                end = a.slot0[l + 1];
                lo = a.lo[l];
                n = a.n[l];
                out = a.out[l];
                al = a.aligned[l] != 0;
            }
            const int64_t e0 = static_cast<int64_t>(su - first) * 8;  // first element in the layer
            if (al && e0 + 8 <= n) {
                const uint32_t vi = static_cast<uint32_t>((lo + e0) >> 3);
                oc.seek(vi);
                if (!ZB_IN(oc.o < static_cast<uint32_t>(a.R) && vi - oc.base < a.S8 && a.param[cur][oc.o] && out,
                           10, vi))
                    continue;
                q[u] = ld_grad(reinterpret_cast<const uint4*>(a.param[cur][oc.o]) + (vi - oc.base));
                dst[u] = out + e0;
            } else {
                const int64_t e1 = e0 + 8 < n ? e0 + 8 : n;
                for (int64_t e = e0; e < e1; ++e) {
                    const int64_t i = lo + e;
                    const int64_t o = i / a.S;
                    if (!ZB_IN(e >= 0 && o < a.R && i - o * a.S < a.S && a.param[cur][o] && out, 11, i)) continue;
                    out[e] = ld_grad1(a.param[cur][o] + (i - o * a.S));
                }
            }
        }
        // pass 2: the stores
#pragma unroll
        for (int u = 0; u < kGatherUnroll; ++u)
            if (dst[u]) st_u4(dst[u], q[u]);
    }
}

// ---------------------------------------------------------------------------
// Launchers.
// ---------------------------------------------------------------------------

namespace {

struct DeviceInfo {
    int sms = 0;
};

DeviceInfo& device_info(int dev) {
    static DeviceInfo infos[64];
    static std::once_flag flags[64];
    std::call_once(flags[dev & 63], [&] {
        cudaDeviceGetAttribute(&infos[dev & 63].sms, cudaDevAttrMultiProcessorCount, dev);
    });
    return infos[dev & 63];
}

int current_sms() {
    int dev = 0;
    cudaGetDevice(&dev);
    return device_info(dev).sms;
}

template <typename K>
int blocks_per_sm(K kernel) {
    int n = 0;
    cudaOccupancyMaxActiveBlocksPerMultiprocessor(&n, kernel, kThreads, 0);
    return n > 0 ? n : 1;
}

uint32_t grid_for(uint64_t work_items, int per_sm, int cap) {
    const uint64_t need = (work_items + kThreads - 1) / kThreads;
    uint64_t g = static_cast<uint64_t>(current_sms()) * static_cast<uint64_t>(per_sm);
    if (g > need) g = need;
    if (cap > 0 && g > static_cast<uint64_t>(cap)) g = cap;
    return static_cast<uint32_t>(g > 0 ? g : 1);
}

template <typename H, int RC, bool CLIP, bool ACC = false, bool PUSH = false>
cudaError_t fused_t(const StepParams& sp, const RankPtrs& p, cudaStream_t s) {
    constexpr int CAP = RC == 0 ? ZERO_MAX_RANKS : RC;
    FusedArgs<CAP> a;
    a.sp = sp;
    for (int r = 0; r < sp.R; ++r) {
        a.g[r] = static_cast<const uint4*>(p.g[r]);
        a.acc[r] = p.acc[r];
        for (int k = 0; k < 2; ++k) {
            a.master[k][r] = p.master[k][r];
            a.m[k][r] = p.m[k][r];
            a.v[k][r] = p.v[k][r];
            a.param[k][r] = static_cast<uint4*>(p.param[k][r]);
            a.full[k][r] = static_cast<uint4*>(p.full[k][r]);
        }
    }
    static const int per_sm = blocks_per_sm(fused_step_kernel<H, RC, CLIP, ACC, PUSH>);
    const uint32_t grid = grid_for(static_cast<uint64_t>(sp.oend - sp.obeg) * sp.S8, per_sm, sp.grid_cap);
    fused_step_kernel<H, RC, CLIP, ACC, PUSH><<<grid, kThreads, 0, s>>>(a);
    return cudaGetLastError();
}

template <typename H, int RC, bool CLIP>
cudaError_t fused_tma_t(const StepParams& sp, const RankPtrs& p, cudaStream_t s) {
    FusedArgs<RC> a;
    a.sp = sp;
    for (int r = 0; r < RC; ++r) {
        a.g[r] = static_cast<const uint4*>(p.g[r]);
        for (int k = 0; k < 2; ++k) {
            a.master[k][r] = p.master[k][r];
            a.m[k][r] = p.m[k][r];
            a.v[k][r] = p.v[k][r];
            a.param[k][r] = static_cast<uint4*>(p.param[k][r]);
        }
    }
    constexpr int smem = TmaStage<RC>::kSmem;
    static const int per_sm = [] {
        cudaFuncSetAttribute(fused_step_tma_kernel<H, RC, CLIP>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                             smem);
        int n = 0;
        cudaOccupancyMaxActiveBlocksPerMultiprocessor(&n, fused_step_tma_kernel<H, RC, CLIP>, kTmaThreads, smem);
        return n > kTmaBlocksPerSm ? kTmaBlocksPerSm : (n > 0 ? n : 1);
    }();
    const int64_t tiles_per_shard = staged_tiles_per_shard(static_cast<int64_t>(sp.S8) * 8);
    const uint64_t tiles = static_cast<uint64_t>(tiles_per_shard) * static_cast<uint64_t>(sp.oend - sp.obeg);
    const uint32_t grid = grid_for(tiles * kThreads, per_sm, sp.grid_cap);
    fused_step_tma_kernel<H, RC, CLIP><<<grid, kTmaThreads, smem, s>>>(a, static_cast<uint64_t>(tiles_per_shard));
    return cudaGetLastError();
}

// The last micro-batch of an accumulation, fused: the register kernel at
// every R (the staged kernel has no accumulator stream).
template <typename H>
cudaError_t fused_acc_dispatch(const StepParams& sp, const RankPtrs& p, cudaStream_t s) {
    switch (sp.R) {
        case 4: return fused_t<H, 4, false, true>(sp, p, s);
        case 8: return fused_t<H, 8, false, true>(sp, p, s);
        case 16: return fused_t<H, 16, false, true>(sp, p, s);
        default: return fused_t<H, 0, false, true>(sp, p, s);
    }
}

template <typename H, bool CLIP>
cudaError_t fused_dispatch(const StepParams& sp, const RankPtrs& p, cudaStream_t s) {
    switch (sp.R) {
        case 1: return fused_tma_t<H, 1, CLIP>(sp, p, s);
        case 2: return fused_tma_t<H, 2, CLIP>(sp, p, s);
        case 4: return fused_t<H, 4, CLIP>(sp, p, s);
        case 8: return fused_t<H, 8, CLIP>(sp, p, s);
        case 16: return fused_t<H, 16, CLIP>(sp, p, s);
        default: return fused_t<H, 0, CLIP>(sp, p, s);
    }
}

template <typename H, int RC, bool ACCUM>
cudaError_t rs_t(int32_t R, int64_t S, int64_t lo, int64_t hi, DevState* st, const RankPtrs& p,
                 cudaStream_t s, int max_sms, const RsNorm* norm) {
    constexpr int CAP = RC == 0 ? ZERO_MAX_RANKS : RC;
    RsArgs<CAP> a;
    a.lo = lo;
    a.hi = hi;
    a.S = S;
    a.S8 = static_cast<uint32_t>(S / 8);
    a.R = R;
    a.st = st;
    a.norm = norm ? *norm : RsNorm{};
    // aligned body [ceil8(lo), floor8(hi)), if non-empty
    const int64_t vlo = (lo + 7) / 8, vhi = hi / 8;
    if (vlo < vhi) {
        a.v0 = static_cast<uint32_t>(vlo);
        a.v1 = static_cast<uint32_t>(vhi);
        a.head_end = vlo * 8;
        a.tail_begin = vhi * 8;
    } else {
        a.v0 = a.v1 = 0;
        a.head_end = hi;  // everything is "head"
        a.tail_begin = hi;
    }
    for (int r = 0; r < R; ++r) {
        a.g[r] = static_cast<const uint4*>(p.g[r]);
        a.acc[r] = p.acc[r];
    }
    static const int per_sm = blocks_per_sm(reduce_scatter_kernel<H, RC, ACCUM>);
    const uint64_t items = static_cast<uint64_t>(a.v1 - a.v0);
    const uint64_t edges = static_cast<uint64_t>((a.head_end - lo) + (hi - a.tail_begin));
    const uint32_t grid = grid_for(items > edges ? items : edges, per_sm, max_sms * per_sm);
    reduce_scatter_kernel<H, RC, ACCUM><<<grid, kThreads, 0, s>>>(a);
    return cudaGetLastError();
}

template <typename H, bool ACCUM>
cudaError_t rs_dispatch(int32_t R, int64_t S, int64_t lo, int64_t hi, DevState* st,
                        const RankPtrs& p, cudaStream_t s, int max_sms, const RsNorm* norm) {
    switch (R) {
        case 1: return rs_t<H, 1, ACCUM>(R, S, lo, hi, st, p, s, max_sms, norm);
        case 2: return rs_t<H, 2, ACCUM>(R, S, lo, hi, st, p, s, max_sms, norm);
        case 4: return rs_t<H, 4, ACCUM>(R, S, lo, hi, st, p, s, max_sms, norm);
        case 8: return rs_t<H, 8, ACCUM>(R, S, lo, hi, st, p, s, max_sms, norm);
        case 16: return rs_t<H, 16, ACCUM>(R, S, lo, hi, st, p, s, max_sms, norm);
        default: return rs_t<H, 0, ACCUM>(R, S, lo, hi, st, p, s, max_sms, norm);
    }
}

template <typename H, bool CLIP, bool PUSH = false>
cudaError_t acc_t(const StepParams& sp, const RankPtrs& p, cudaStream_t s) {
    AccArgs a;
    a.sp = sp;
    for (int r = 0; r < sp.R; ++r) {
        a.acc[r] = p.acc[r];
        for (int k = 0; k < 2; ++k) {
            a.master[k][r] = p.master[k][r];
            a.m[k][r] = p.m[k][r];
            a.v[k][r] = p.v[k][r];
            a.param[k][r] = static_cast<uint4*>(p.param[k][r]);
            a.full[k][r] = static_cast<uint4*>(p.full[k][r]);
        }
    }
    if constexpr (!PUSH) {
        constexpr int smem = TmaAccStage::kSmem;
        static const int per_sm = [] {
            cudaFuncSetAttribute(step_from_acc_tma_kernel<H, CLIP>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                 smem);
            int n = 0;
            cudaOccupancyMaxActiveBlocksPerMultiprocessor(&n, step_from_acc_tma_kernel<H, CLIP>, kTmaThreads, smem);
            return n > kTmaBlocksPerSm ? kTmaBlocksPerSm : (n > 0 ? n : 1);
        }();
        const int64_t tiles_per_shard = staged_tiles_per_shard(static_cast<int64_t>(sp.S8) * 8);
        const uint64_t tiles = static_cast<uint64_t>(tiles_per_shard) * static_cast<uint64_t>(sp.oend - sp.obeg);
        const uint32_t grid = grid_for(tiles * kThreads, per_sm, sp.grid_cap);
        step_from_acc_tma_kernel<H, CLIP><<<grid, kTmaThreads, smem, s>>>(a, static_cast<uint64_t>(tiles_per_shard));
    } else {
        static const int per_sm = blocks_per_sm(step_from_acc_kernel<H, CLIP, PUSH>);
        const uint32_t grid = grid_for(static_cast<uint64_t>(sp.oend - sp.obeg) * sp.S8, per_sm, sp.grid_cap);
        step_from_acc_kernel<H, CLIP, PUSH><<<grid, kThreads, 0, s>>>(a);
    }
    return cudaGetLastError();
}

// The step with the parameter push: the runtime-R register kernel, whatever R.
template <typename H>
cudaError_t fused_push_dispatch(const StepParams& sp, const RankPtrs& p, cudaStream_t s) {
    if (sp.add_acc) return fused_t<H, 0, false, true, true>(sp, p, s);
    if (sp.clip) return fused_t<H, 0, true, false, true>(sp, p, s);
    return fused_t<H, 0, false, false, true>(sp, p, s);
}

}  // namespace

cudaError_t launch_fused_step(const StepParams& sp, const RankPtrs& p, cudaStream_t s) {
    if (sp.push)
        return sp.dtype == ZERO_FP16 ? fused_push_dispatch<Fp16>(sp, p, s) : fused_push_dispatch<Bf16>(sp, p, s);
    if (sp.add_acc)
        return sp.dtype == ZERO_FP16 ? fused_acc_dispatch<Fp16>(sp, p, s) : fused_acc_dispatch<Bf16>(sp, p, s);
    if (sp.clip)
        return sp.dtype == ZERO_FP16 ? fused_dispatch<Fp16, true>(sp, p, s) : fused_dispatch<Bf16, true>(sp, p, s);
    return sp.dtype == ZERO_FP16 ? fused_dispatch<Fp16, false>(sp, p, s) : fused_dispatch<Bf16, false>(sp, p, s);
}

cudaError_t launch_fsm_commit(const StepParams& sp, const double* reduced, cudaStream_t s) {
    fsm_commit_kernel<<<1, 32, 0, s>>>(sp, reduced);
    return cudaGetLastError();
}

cudaError_t launch_step_from_acc(const StepParams& sp, const RankPtrs& p, cudaStream_t s) {
    if (sp.push) {
        if (sp.clip)
            return sp.dtype == ZERO_FP16 ? acc_t<Fp16, true, true>(sp, p, s) : acc_t<Bf16, true, true>(sp, p, s);
        return sp.dtype == ZERO_FP16 ? acc_t<Fp16, false, true>(sp, p, s) : acc_t<Bf16, false, true>(sp, p, s);
    }
    if (sp.clip) return sp.dtype == ZERO_FP16 ? acc_t<Fp16, true>(sp, p, s) : acc_t<Bf16, true>(sp, p, s);
    return sp.dtype == ZERO_FP16 ? acc_t<Fp16, false>(sp, p, s) : acc_t<Bf16, false>(sp, p, s);
}

cudaError_t launch_reduce_scatter(int32_t R, int32_t dtype, int64_t S, int64_t lo, int64_t hi,
                                  DevState* st, const RankPtrs& p, cudaStream_t s, bool accumulate,
                                  int max_sms, const RsNorm* norm) {
    if (accumulate)
        return dtype == ZERO_FP16 ? rs_dispatch<Fp16, true>(R, S, lo, hi, st, p, s, max_sms, norm)
                                  : rs_dispatch<Bf16, true>(R, S, lo, hi, st, p, s, max_sms, norm);
    return dtype == ZERO_FP16 ? rs_dispatch<Fp16, false>(R, S, lo, hi, st, p, s, max_sms, norm)
                              : rs_dispatch<Bf16, false>(R, S, lo, hi, st, p, s, max_sms, norm);
}

// The clipping coefficient from the reduce-scatters' norm shares slots
// [first, first + count), summed in slot order (strided over the block, then
// the block's fixed reduction tree).
__global__ void __launch_bounds__(kThreads)
    clip_from_rs_norm_kernel(const __grid_constant__ StepParams sp, const double* slots, int64_t first,
                             int64_t count) {
    __shared__ double red[kWarps];
    double x = 0.0;
    for (int64_t i = threadIdx.x; i < count; i += kThreads) x += slots[first + i];
    const double total = block_sum(x, red);
    if (threadIdx.x == 0) {
        sp.st->clip = clip_coefficient(sp.max_norm, total);
        __threadfence();
    }
}

cudaError_t launch_clip_from_rs_norm(const StepParams& sp, const double* slots, int64_t first, int64_t count,
                                     cudaStream_t s) {
    clip_from_rs_norm_kernel<<<1, kThreads, 0, s>>>(sp, slots, first, count);
    return cudaGetLastError();
}

namespace {
template <typename H, int RC>
cudaError_t grad_norm_t(const StepParams& sp, const RankPtrs& p, cudaStream_t s) {
    GradNormArgs<RC == 0 ? ZERO_MAX_RANKS : RC> a;
    a.sp = sp;
    for (int r = 0; r < sp.R; ++r) a.g[r] = static_cast<const uint4*>(p.g[r]);
    static const int per_sm = blocks_per_sm(grad_norm_kernel<H, RC>);
    const uint32_t grid = grid_for(static_cast<uint64_t>(sp.oend - sp.obeg) * sp.S8, per_sm, sp.grid_cap);
    grad_norm_kernel<H, RC><<<grid, kThreads, 0, s>>>(a);
    return cudaGetLastError();
}

template <typename H>
cudaError_t grad_norm_dispatch(const StepParams& sp, const RankPtrs& p, cudaStream_t s) {
    switch (sp.R) {
        case 1: return grad_norm_t<H, 1>(sp, p, s);
        case 2: return grad_norm_t<H, 2>(sp, p, s);
        case 4: return grad_norm_t<H, 4>(sp, p, s);
        case 8: return grad_norm_t<H, 8>(sp, p, s);
        case 16: return grad_norm_t<H, 16>(sp, p, s);
        default: return grad_norm_t<H, 0>(sp, p, s);
    }
}
}  // namespace

cudaError_t launch_clip_from_norm(const StepParams& sp, const double* norm_sq, cudaStream_t s) {
    clip_from_norm_kernel<<<1, 32, 0, s>>>(sp, norm_sq);
    return cudaGetLastError();
}

cudaError_t launch_grad_norm(const StepParams& sp, const RankPtrs& p, cudaStream_t s) {
    return sp.dtype == ZERO_FP16 ? grad_norm_dispatch<Fp16>(sp, p, s) : grad_norm_dispatch<Bf16>(sp, p, s);
}

cudaError_t launch_clip_norm(const StepParams& sp, const RankPtrs& p, cudaStream_t s) {
    NormArgs a;
    a.sp = sp;
    for (int r = 0; r < sp.R; ++r) a.acc[r] = p.acc[r];
    static const int per_sm = blocks_per_sm(clip_norm_kernel);
    const uint32_t grid = grid_for(static_cast<uint64_t>(sp.oend - sp.obeg) * sp.S8, per_sm, sp.grid_cap);
    clip_norm_kernel<<<grid, kThreads, 0, s>>>(a);
    return cudaGetLastError();
}

cudaError_t launch_gather_many(int32_t R, int64_t S, int nl, const int64_t* lo, const int64_t* hi,
                               const DevState* st, const RankPtrs& p, void* const* outs,
                               cudaStream_t s, int max_sms) {
    GatherManyArgs a;
    a.nl = nl;
    a.R = R;
    a.S = S;
    a.S8 = static_cast<uint32_t>(S / 8);
    a.st = st;
    for (int r = 0; r < R; ++r)
        for (int k = 0; k < 2; ++k) a.param[k][r] = static_cast<const uint16_t*>(p.param[k][r]);
    uint64_t slots = 0;
    for (int l = 0; l < nl; ++l) {
        a.lo[l] = lo[l];
        a.n[l] = hi[l] - lo[l];
        a.out[l] = static_cast<uint16_t*>(outs[l]);
        a.aligned[l] = (lo[l] % 8) == 0;
        a.slot0[l] = static_cast<uint32_t>(slots);
        slots += static_cast<uint64_t>((a.n[l] + 7) / 8);
    }
    a.slot0[nl] = static_cast<uint32_t>(slots);
    a.total_slots = static_cast<uint32_t>(slots);
    if (slots == 0) return cudaSuccess;
    if (slots > kGatherWideSlots) {
        static const int per_sm = blocks_per_sm(gather_many_kernel<8>);
        const uint32_t grid = grid_for((slots + 7) / 8, per_sm, max_sms * per_sm);
        gather_many_kernel<8><<<grid, kThreads, 0, s>>>(a);
    } else {
        static const int per_sm = blocks_per_sm(gather_many_kernel<4>);
        const uint32_t grid = grid_for((slots + 3) / 4, per_sm, max_sms * per_sm);
        gather_many_kernel<4><<<grid, kThreads, 0, s>>>(a);
    }
    return cudaGetLastError();
}

cudaError_t launch_gather(int32_t R, int64_t S, int64_t lo, int64_t hi, const DevState* st,
                          const RankPtrs& p, void* out, cudaStream_t s) {
    void* outs[1] = {out};
    return launch_gather_many(R, S, 1, &lo, &hi, st, p, outs, s);
}

int step_grid_cap(int device) {
    // at most 8 blocks of 256 threads fit on an SM
    return device_info(device).sms * 8;
}

}  // namespace zb

extern "C" zero_status zero_debug_bounds(int64_t* count, int64_t* first_site, int64_t* first_index,
                                         int32_t reset) {
    if (!count || !first_site || !first_index)
        return zb_fail(ZERO_ERR_INVALID_ARG, "zero_debug_bounds: NULL output");
#ifdef ZERO_DEBUG_BOUNDS
    unsigned long long c = 0, f = 0, c2 = 0, f2 = 0;
    cudaError_t e = zb::bounds_record(&c, &f, reset != 0);
    if (e == cudaSuccess) e = zb::noalloc_bounds_record(&c2, &f2, reset != 0);
    if (e != cudaSuccess) {
        cudaGetLastError();
        return zb_fail(ZERO_ERR_CUDA, std::string("zero_debug_bounds: ") + cudaGetErrorString(e));
    }
    c += c2;
    if (f == 0) f = f2;
    *count = static_cast<int64_t>(c);
    *first_site = static_cast<int64_t>(f >> 48);
    *first_index = static_cast<int64_t>(f & 0xffffffffffffull);
#else
    (void)reset;
    *count = -1;  // the release build carries no checks
    *first_site = 0;
    *first_index = 0;
#endif
    return ZERO_OK;
}
