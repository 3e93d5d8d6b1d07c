// zero_step_noalloc: the two-pass step (reduce-scatter into fp32
// accumulators, then AdamW in place) for callers that cannot allocate device
// memory. Every byte of scratch it needs -- the R fp32 accumulators, the
// per-block norm partials and a small control word -- lives in one static
// device array in this file, so the call makes no cudaMalloc / cudaFree and
// needs no context. See include/zero_b200.h for the contract.
#include <cuda.h>

#include <atomic>
#include <cmath>
#include <mutex>
#include <string>

#include "debug_bounds.cuh"
#include "device_common.cuh"
#include "internal.h"

namespace zb {
namespace {

constexpr int64_t kNoallocMaxElems = ZERO_NOALLOC_MAX_ELEMS;
constexpr int kNoallocMaxBlocks = 4096;
constexpr size_t kAccBytes = static_cast<size_t>(kNoallocMaxElems) * sizeof(float);
constexpr size_t kPartialBytes = static_cast<size_t>(kNoallocMaxBlocks) * sizeof(double);
constexpr size_t kCtrlBytes = 256;
constexpr size_t kScratchBytes = kAccBytes + kPartialBytes + kCtrlBytes;
static_assert(sizeof(DevState) <= kCtrlBytes, "control word does not fit");

}  // namespace

// The scratch of zero_step_noalloc: [accumulators | norm partials | control].
// One copy per device that loads the library, kept until the process exits.
static __device__ __align__(256) unsigned char g_noalloc_scratch[kScratchBytes];

namespace {

struct NoallocArgs {
    Coef c;
    int32_t R;
    int32_t dynamic;
    uint32_t S8, T8;
    DevState* ctrl;
    double* partials;
    const float* acc[ZERO_MAX_RANKS];
    float* master[ZERO_MAX_RANKS];
    float* m[ZERO_MAX_RANKS];
    float* v[ZERO_MAX_RANKS];
    uint4* param[ZERO_MAX_RANKS];
};

// AdamW from the accumulators, in place; skipped in DYNAMIC mode when the
// reduce-scatter raised the overflow flag. The last block to finish sums the
// norm partials and records the flag; the loss-scale update runs on the host.
template <typename H>
__global__ void __launch_bounds__(kThreads) noalloc_step_kernel(const __grid_constant__ NoallocArgs a) {
    __shared__ int s_skip;
    __shared__ double red[kWarps];
    __shared__ int last;
    if (threadIdx.x == 0)
        s_skip = a.dynamic && *reinterpret_cast<volatile uint32_t*>(&a.ctrl->flag) != 0u;
    __syncthreads();
    const bool skip = s_skip != 0;
    const Coef c = a.c;
    double nrm = 0.0;
    const uint32_t stride = gridDim.x * kThreads;
    uint32_t vi = blockIdx.x * kThreads + threadIdx.x;
    OwnerCursor oc(vi, a.S8);
    for (; vi < a.T8; vi += stride) {
        oc.seek(vi);
        const uint32_t o = oc.o;
        const size_t j8 = static_cast<size_t>(vi - oc.base) * 8;
        if (!ZB_IN(o < static_cast<uint32_t>(a.R) && vi - oc.base < a.S8 && a.acc[o] && a.master[o] && a.m[o] &&
                       a.v[o] && a.param[o],
                   13, vi))
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
        F8 p = ld_f8(a.master[o] + j8);
        F8 m = ld_f8(a.m[o] + j8);
        F8 v = ld_f8(a.v[o] + j8);
        float out[8];
#pragma unroll
        for (int e = 0; e < 8; ++e) {
            const double gd = static_cast<double>(adamw1(c, acc.x[e], p.x[e], m.x[e], v.x[e]));
            nrm = fma(gd, gd, nrm);
            out[e] = p.x[e];
        }
        st_f8(a.master[o] + j8, p);
        st_f8(a.m[o] + j8, m);
        st_f8(a.v[o] + j8, v);
        st_u4(a.param[o] + (j8 >> 3), pack8<H>(out));
    }
    const double bn = block_sum(nrm, red);
    if (threadIdx.x == 0) {
        a.partials[blockIdx.x] = bn;
        __threadfence();
        last = (atomicAdd(&a.ctrl->done, 1u) == gridDim.x - 1);
    }
    __syncthreads();
    if (!last) return;
    __threadfence();
    double x = 0.0;
    for (unsigned i = threadIdx.x; i < gridDim.x; i += kThreads)
        x += *reinterpret_cast<volatile double*>(&a.partials[i]);
    const double total = block_sum(x, red);
    if (threadIdx.x == 0) {
        a.ctrl->grad_norm_sq = total;
        a.ctrl->last_overflow = *reinterpret_cast<volatile uint32_t*>(&a.ctrl->flag) != 0u;
        a.ctrl->done = 0u;
        __threadfence();
    }
}

// Device address of g_noalloc_scratch, looked up once per device and CUDA
// context with that device current (a reset device gets a new context, and
// its array a new address). In host code the array's name only stands in for
// the symbol; it is not a device address.
struct ScratchSlot {
    CUcontext ctx = nullptr;
    unsigned char* addr = nullptr;
};
std::mutex g_scratch_mu;
ScratchSlot g_scratch_slot[64];
std::atomic<bool> g_noalloc_used{false};

using CtxGetCurrent = CUresult (*)(CUcontext*);

// The calling thread's current context through the driver's entry point
// (the library links no driver library); NULL when none is current yet or
// the entry point is unavailable.
CUcontext current_context() {
    static const CtxGetCurrent fn = [] {
        void* p = nullptr;
        cudaDriverEntryPointQueryResult q = cudaDriverEntryPointSymbolNotFound;
        if (cudaGetDriverEntryPoint("cuCtxGetCurrent", &p, cudaEnableDefault, &q) != cudaSuccess ||
            q != cudaDriverEntryPointSuccess) {
            cudaGetLastError();
            p = nullptr;
        }
        return reinterpret_cast<CtxGetCurrent>(p);
    }();
    CUcontext c = nullptr;
    if (fn && fn(&c) != CUDA_SUCCESS) c = nullptr;
    return c;
}

zero_status scratch_for_current_device(unsigned char** out) {
    int dev = -1;
    cudaError_t e = cudaGetDevice(&dev);
    if (e != cudaSuccess)
        return zb_fail(ZERO_ERR_CUDA, std::string("zero_step_noalloc: ") + cudaGetErrorString(e));
    if (dev < 0 || dev >= 64) return zb_fail(ZERO_ERR_RANGE, "zero_step_noalloc: device index >= 64");
    std::lock_guard<std::mutex> lock(g_scratch_mu);
    ScratchSlot& slot = g_scratch_slot[dev];
    const CUcontext ctx = current_context();
    if (ctx == nullptr || slot.ctx != ctx || slot.addr == nullptr) {
        // set-up: under CUDA's lazy module loading this also loads this
        // file's module on the device, which reserves the static array
        void* p = nullptr;
        e = cudaGetSymbolAddress(&p, g_noalloc_scratch);
        if (e != cudaSuccess || p == nullptr) {
            cudaGetLastError();
            return zb_fail(ZERO_ERR_CUDA,
                           std::string("zero_step_noalloc: cannot resolve the static scratch: ") +
                               cudaGetErrorString(e));
        }
        slot.addr = static_cast<unsigned char*>(p);
        slot.ctx = current_context();  // the look-up made the device's context current
    }
    g_noalloc_used.store(true);
    *out = slot.addr;
    return ZERO_OK;
}

bool aligned_to(const void* p, uintptr_t a) { return reinterpret_cast<uintptr_t>(p) % a == 0; }

template <typename Ptr>
zero_status check_list(Ptr const* arr, int R, uintptr_t align, const char* what) {
    if (!arr) return zb_fail(ZERO_ERR_INVALID_ARG, std::string("zero_step_noalloc: ") + what + " is NULL");
    for (int r = 0; r < R; ++r) {
        if (!arr[r])
            return zb_fail(ZERO_ERR_INVALID_ARG, std::string("zero_step_noalloc: ") + what + "[" +
                                                     std::to_string(r) + "] is NULL");
        if (!aligned_to(arr[r], align))
            return zb_fail(ZERO_ERR_ALIGN, std::string("zero_step_noalloc: ") + what + "[" +
                                               std::to_string(r) + "] is misaligned");
    }
    return ZERO_OK;
}

}  // namespace

#ifdef ZERO_DEBUG_BOUNDS
cudaError_t noalloc_bounds_record(unsigned long long* count, unsigned long long* first, bool reset) {
    *count = 0;
    *first = 0;
    // reading the record would load this module, and reserve its array, in a
    // process that never used it
    if (!g_noalloc_used.load()) return cudaSuccess;
    return bounds_record(count, first, reset);
}
#endif

}  // namespace zb

extern "C" zero_status zero_step_noalloc(const zero_plan_t* plan, const zero_loss_scale_config* cfg,
                                         zero_loss_scale_state* inout, const zero_adamw* hp,
                                         const void* const* grads, float* const* master,
                                         float* const* m, float* const* v, void* const* param,
                                         void* stream) {
    return zb_guarded("zero_step_noalloc", [&]() -> zero_status {
        using namespace zb;
        if (!plan || !cfg || !inout || !hp)
            return zb_fail(ZERO_ERR_INVALID_ARG, "zero_step_noalloc: NULL plan, cfg, state or hp");
        if (plan->T > kNoallocMaxElems)
            return zb_fail(ZERO_ERR_RANGE,
                           "zero_step_noalloc: the padded model has " + std::to_string(plan->T) +
                               " elements, more than the static scratch holds (" +
                               std::to_string(kNoallocMaxElems) + "); use zero_step with a context");
        if (cfg->mode < ZERO_SCALE_NONE || cfg->mode > ZERO_SCALE_DYNAMIC ||
            (cfg->mode == ZERO_SCALE_DYNAMIC &&
             (cfg->growth_interval < 1 || !(cfg->growth_factor > 1.0f) ||
              !(cfg->backoff_factor > 0.0f && cfg->backoff_factor < 1.0f) || !(cfg->min_scale > 0.0f))))
            return zb_fail(ZERO_ERR_INVALID_ARG, "zero_step_noalloc: bad loss-scale config");
        const float scale = cfg->mode == ZERO_SCALE_NONE ? 1.0f : inout->scale;
        if (!(scale > 0.0f) || !std::isfinite(scale) || inout->t < 0 || inout->good < 0 || inout->cur != 0)
            return zb_fail(ZERO_ERR_INVALID_ARG,
                           "zero_step_noalloc: need finite scale > 0, t >= 0, good >= 0 and cur == 0");
        if (!(hp->lr >= 0.0) || !(hp->beta1 >= 0.0 && hp->beta1 < 1.0) ||
            !(hp->beta2 >= 0.0 && hp->beta2 < 1.0) || !(hp->eps > 0.0) || !(hp->weight_decay >= 0.0) ||
            !std::isfinite(hp->lr) || !std::isfinite(hp->weight_decay))
            return zb_fail(ZERO_ERR_INVALID_ARG,
                           "zero_step_noalloc: need lr >= 0, 0 <= beta < 1, eps > 0, weight_decay >= 0");
        const int R = plan->R;
        zero_status s;
        if ((s = check_list(grads, R, 16, "grads")) != ZERO_OK) return s;
        if ((s = check_list(master, R, 32, "master")) != ZERO_OK) return s;
        if ((s = check_list(m, R, 32, "m")) != ZERO_OK) return s;
        if ((s = check_list(v, R, 32, "v")) != ZERO_OK) return s;
        if ((s = check_list(param, R, 16, "param")) != ZERO_OK) return s;

        unsigned char* base = nullptr;
        if ((s = scratch_for_current_device(&base)) != ZERO_OK) return s;
        float* acc = reinterpret_cast<float*>(base);
        double* partials = reinterpret_cast<double*>(base + kAccBytes);
        DevState* ctrl = reinterpret_cast<DevState*>(base + kAccBytes + kPartialBytes);
        cudaStream_t cs = static_cast<cudaStream_t>(stream);

        // the control word must start at zero: no overflow, no finished blocks
        cudaError_t e = cudaMemsetAsync(ctrl, 0, sizeof(DevState), cs);
        if (e != cudaSuccess) return zb_fail(ZERO_ERR_CUDA, std::string("zero_step_noalloc: ") + cudaGetErrorString(e));

        RankPtrs p;
        for (int r = 0; r < R; ++r) {
            p.g[r] = grads[r];
            p.acc[r] = acc + static_cast<size_t>(r) * plan->S;
        }
        e = launch_reduce_scatter(R, plan->dtype, plan->S, 0, plan->T, ctrl, p, cs);
        if (e != cudaSuccess) return zb_fail(ZERO_ERR_CUDA, std::string("zero_step_noalloc: ") + cudaGetErrorString(e));

        // coefficients of step t+1, formed on the host in double, rounded once
        NoallocArgs a;
        const double t1 = static_cast<double>(inout->t + 1);
        a.c.inv = static_cast<float>(1.0 / (static_cast<double>(R) * static_cast<double>(scale)));
        a.c.dec = static_cast<float>(1.0 - hp->lr * hp->weight_decay);
        a.c.b1f = static_cast<float>(hp->beta1);
        a.c.omb1 = static_cast<float>(1.0 - hp->beta1);
        a.c.b2f = static_cast<float>(hp->beta2);
        a.c.omb2 = static_cast<float>(1.0 - hp->beta2);
        a.c.epsf = static_cast<float>(hp->eps);
        a.c.ss = static_cast<float>(hp->lr / (1.0 - std::pow(hp->beta1, t1)));
        a.c.bc2s = static_cast<float>(std::sqrt(1.0 - std::pow(hp->beta2, t1)));
        a.c.clip = 1.0f;
        a.R = R;
        a.dynamic = cfg->mode == ZERO_SCALE_DYNAMIC;
        a.S8 = static_cast<uint32_t>(plan->S / 8);
        a.T8 = static_cast<uint32_t>(plan->T / 8);
        a.ctrl = ctrl;
        a.partials = partials;
        for (int r = 0; r < R; ++r) {
            a.acc[r] = p.acc[r];
            a.master[r] = master[r];
            a.m[r] = m[r];
            a.v[r] = v[r];
            a.param[r] = static_cast<uint4*>(param[r]);
        }
        int sms = 0, dev = 0, per_sm = 0;
        cudaGetDevice(&dev);
        cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
        if (plan->dtype == ZERO_FP16)
            cudaOccupancyMaxActiveBlocksPerMultiprocessor(&per_sm, noalloc_step_kernel<Fp16>, kThreads, 0);
        else
            cudaOccupancyMaxActiveBlocksPerMultiprocessor(&per_sm, noalloc_step_kernel<Bf16>, kThreads, 0);
        int64_t grid = static_cast<int64_t>(sms) * (per_sm > 0 ? per_sm : 1);
        const int64_t need = (static_cast<int64_t>(a.T8) + kThreads - 1) / kThreads;
        if (grid > need) grid = need;
        if (grid > kNoallocMaxBlocks) grid = kNoallocMaxBlocks;
        if (grid < 1) grid = 1;
        if (plan->dtype == ZERO_FP16)
            noalloc_step_kernel<Fp16><<<static_cast<unsigned>(grid), kThreads, 0, cs>>>(a);
        else
            noalloc_step_kernel<Bf16><<<static_cast<unsigned>(grid), kThreads, 0, cs>>>(a);
        e = cudaGetLastError();
        if (e != cudaSuccess) return zb_fail(ZERO_ERR_CUDA, std::string("zero_step_noalloc: ") + cudaGetErrorString(e));

        // bring the step's result back and run the loss-scale update on the host
        DevState out{};
        e = cudaMemcpyAsync(&out, ctrl, sizeof(DevState), cudaMemcpyDeviceToHost, cs);
        if (e == cudaSuccess) e = cudaStreamSynchronize(cs);
        if (e != cudaSuccess) return zb_fail(ZERO_ERR_CUDA, std::string("zero_step_noalloc: ") + cudaGetErrorString(e));
        const int overflow = out.last_overflow != 0;
        int skipped = 0;
        if (cfg->mode == ZERO_SCALE_DYNAMIC) {
            if (overflow) {
                const float sc = inout->scale * cfg->backoff_factor;
                inout->scale = (sc < cfg->min_scale) ? cfg->min_scale : sc;
                inout->good = 0;
                skipped = 1;
            } else {
                inout->t += 1;
                inout->good += 1;
                if (inout->good >= cfg->growth_interval) {
                    inout->scale = inout->scale * cfg->growth_factor;
                    inout->good = 0;
                }
            }
        } else {
            inout->t += 1;
        }
        inout->last_overflow = overflow;
        inout->last_skipped = skipped;
        inout->grad_norm_sq = out.grad_norm_sq;
        return ZERO_OK;
    });
}
