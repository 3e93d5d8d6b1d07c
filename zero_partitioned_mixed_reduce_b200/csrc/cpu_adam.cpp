// Host-side AdamW for ZeRO-Offload: the fp32 master weights and the Adam
// moments live in (pinned) host memory and the update runs on CPU cores, while
// the GPU only holds the half parameters and reduces the gradients.
//
// Pages: inferensys legal pre-training glossary, "CPU Offload" (optimizer
// states and gradients offloaded to CPU DRAM; Adam runs on the CPU while the
// GPU runs forward and backward) and "One-Step Delayed Parameter Update"
// (the CPU step overlaps the next forward pass); genomic glossary, "CPU
// Offload" (fp32 master weights and optimizer states in CPU RAM, fp16
// parameters and gradients on the GPU).
//
// The arithmetic is the step of include/zero_b200.h, one IEEE binary32
// operation per line (this file is built with -ffp-contract=off), so results
// equal the GPU step bit for bit. The fp32 update is plain C++ that the
// compiler vectorizes (IEEE division and square root vectorize exactly);
// gcc's target_clones builds AVX-512, AVX2 and baseline versions and picks
// one at load time. bf16 is encoded on the bit pattern, round to nearest
// even, keeping subnormals (the AVX-512 bf16 conversion instruction treats
// subnormal inputs as zero); fp16 uses the IEEE conversion instruction where
// the CPU has it, with a scalar encoder of the same rounding as fallback.
#include <algorithm>
#include <cmath>
#include <condition_variable>
#include <cstring>
#include <functional>
#include <mutex>
#include <string>
#include <thread>
#include <vector>

#include <unistd.h>

#include <immintrin.h>

#include "internal.h"

namespace {

inline uint32_t f2u(float x) {
    uint32_t u;
    std::memcpy(&u, &x, 4);
    return u;
}

// The bf16 encoder is branch-free (both cases computed, one selected) so that
// its loop vectorizes. The fp16 encoder below is the scalar reference (the
// fallback, the tail and the NaN fix-up of the vector conversion).

// fp32 -> bf16, round to nearest even on the bits; NaN -> quiet NaN.
inline uint16_t to_bf16(float x) {
    const uint32_t u = f2u(x);
    const bool nan = (u & 0x7fffffffu) > 0x7f800000u;
    const uint32_t lsb = (u >> 16) & 1u;
    const uint32_t rounded = (u + 0x7fffu + lsb) >> 16;
    return static_cast<uint16_t>(nan ? ((u >> 16) | 0x0040u) : rounded);
}

// fp32 -> IEEE binary16, round to nearest even, subnormals kept, overflow to inf.
inline uint16_t to_fp16(float x) {
    const uint32_t u = f2u(x);
    const uint16_t sign = static_cast<uint16_t>((u >> 16) & 0x8000u);
    const uint32_t a = u & 0x7fffffffu;
    if (a > 0x7f800000u) return static_cast<uint16_t>(sign | 0x7e00u);  // NaN
    if (a >= 0x477ff000u) return static_cast<uint16_t>(sign | 0x7c00u);  // >= 65520: inf
    if (a < 0x38800000u) {  // below 2^-14: fp16 subnormal (or zero)
        // value = mant * 2^(e-150) with the implicit bit; the result counts 2^-24 units
        const uint32_t e = a >> 23;
        if (e < 102) return sign;  // below 2^-25: rounds to zero
        const uint32_t mant = (a & 0x7fffffu) | 0x800000u;
        const uint32_t shift = 126 - e;  // 14..24
        const uint32_t q = mant >> shift;
        const uint32_t rem = mant & ((1u << shift) - 1u);
        const uint32_t half = 1u << (shift - 1);
        const uint32_t r = q + ((rem > half || (rem == half && (q & 1u))) ? 1u : 0u);
        return static_cast<uint16_t>(sign | r);
    }
    // normal: rebias the exponent (127 -> 15) and round the 13 dropped bits
    const uint32_t v = a - 0x38000000u;  // exponent -= 112, still in fp32 bit layout
    const uint32_t lsb = (v >> 13) & 1u;
    return static_cast<uint16_t>(sign | ((v + 0x0fffu + lsb) >> 13));
}

struct Coeffs {
    float inv, dec, b1f, omb1, b2f, omb2, epsf, ss, bc2s, clip;
};

// The fp32 AdamW update of n elements, vectorized (IEEE division and square
// root vectorize exactly).
template <bool CLIP>
__attribute__((target_clones("avx512f", "avx2", "default"))) void adam_range(
    const Coeffs c, const float* __restrict acc, float* __restrict p, float* __restrict m,
    float* __restrict v, int64_t n) {
    for (int64_t i = 0; i < n; ++i) {
        const float g0 = acc[i] * c.inv;
        const float g = CLIP ? g0 * c.clip : g0;
        float pp = p[i] * c.dec;
        const float mm = c.b1f * m[i] + c.omb1 * g;
        const float vv = c.b2f * v[i] + c.omb2 * (g * g);
        const float den = std::sqrt(vv) / c.bc2s + c.epsf;
        pp = pp - c.ss * (mm / den);
        p[i] = pp;
        m[i] = mm;
        v[i] = vv;
    }
}

__attribute__((target_clones("avx512f", "avx2", "default"))) void encode_bf16_range(
    const float* __restrict p, uint16_t* __restrict out, int64_t n) {
    for (int64_t i = 0; i < n; ++i) out[i] = to_bf16(p[i]);
}

// fp32 -> fp16 with the conversion instruction (vcvtps2ph, round to nearest
// even: IEEE conversion, subnormal results kept, overflow to infinity, so it
// equals to_fp16 for every non-NaN input); NaN lanes are re-encoded by
// to_fp16, which gives the canonical quiet NaN.
__attribute__((target("avx512f"))) void encode_fp16_avx512(const float* __restrict p, uint16_t* __restrict out,
                                                           int64_t n) {
    int64_t i = 0;
    for (; i + 16 <= n; i += 16) {
        const __m512 x = _mm512_loadu_ps(p + i);
        const __m256i h = _mm512_cvtps_ph(x, _MM_FROUND_TO_NEAREST_INT | _MM_FROUND_NO_EXC);
        _mm256_storeu_si256(reinterpret_cast<__m256i*>(out + i), h);
        const __mmask16 nan = _mm512_cmp_ps_mask(x, x, _CMP_UNORD_Q);
        if (nan)
            for (int j = 0; j < 16; ++j)
                if (nan & (1u << j)) out[i + j] = to_fp16(p[i + j]);
    }
    for (; i < n; ++i) out[i] = to_fp16(p[i]);
}

__attribute__((target("avx2,f16c"))) void encode_fp16_avx2(const float* __restrict p, uint16_t* __restrict out,
                                                           int64_t n) {
    int64_t i = 0;
    for (; i + 8 <= n; i += 8) {
        const __m256 x = _mm256_loadu_ps(p + i);
        const __m128i h = _mm256_cvtps_ph(x, _MM_FROUND_TO_NEAREST_INT | _MM_FROUND_NO_EXC);
        _mm_storeu_si128(reinterpret_cast<__m128i*>(out + i), h);
        const int nan = _mm256_movemask_ps(_mm256_cmp_ps(x, x, _CMP_UNORD_Q));
        if (nan)
            for (int j = 0; j < 8; ++j)
                if (nan & (1 << j)) out[i + j] = to_fp16(p[i + j]);
    }
    for (; i < n; ++i) out[i] = to_fp16(p[i]);
}

void encode_fp16_scalar(const float* __restrict p, uint16_t* __restrict out, int64_t n) {
    for (int64_t i = 0; i < n; ++i) out[i] = to_fp16(p[i]);
}

using EncodeFn = void (*)(const float*, uint16_t*, int64_t);

EncodeFn pick_fp16_encoder() {
    __builtin_cpu_init();
    if (__builtin_cpu_supports("avx512f")) return encode_fp16_avx512;
    if (__builtin_cpu_supports("avx2") && __builtin_cpu_supports("f16c")) return encode_fp16_avx2;
    return encode_fp16_scalar;
}

// Update then encode, block by block, so that the encode re-reads p from cache.
template <bool FP16, bool CLIP>
void update_range(const Coeffs c, const float* __restrict acc, float* __restrict p, float* __restrict m,
                  float* __restrict v, uint16_t* __restrict out, int64_t n) {
    static const EncodeFn enc16 = pick_fp16_encoder();
    constexpr int64_t kBlock = 2048;
    for (int64_t b = 0; b < n; b += kBlock) {
        const int64_t k = n - b < kBlock ? n - b : kBlock;
        adam_range<CLIP>(c, acc + b, p + b, m + b, v + b, k);
        if (FP16)
            enc16(p + b, out + b, k);
        else
            encode_bf16_range(p + b, out + b, k);
    }
}

// Sum of (double)(acc * inv)^2 over [0, n) and whether any acc is non-finite.
// Eight running sums, one per lane of an 8-element block, then added in lane
// order: a fixed summation order that vectorizes without reassociation.
constexpr int kLanes = 8;
__attribute__((target_clones("avx512f", "avx2", "default"))) void scan_range(
    const float* __restrict acc, float inv, int64_t n, double* nrm, int* bad) {
    double lane[kLanes] = {0, 0, 0, 0, 0, 0, 0, 0};
    int flag[kLanes] = {0, 0, 0, 0, 0, 0, 0, 0};
    const int64_t body = n - n % kLanes;
    for (int64_t i = 0; i < body; i += kLanes) {
        for (int j = 0; j < kLanes; ++j) {
            const float a = acc[i + j];
            flag[j] |= !(std::fabs(a) <= 3.4028234663852886e38f);
            const double g = static_cast<double>(a * inv);
            lane[j] += g * g;
        }
    }
    for (int64_t i = body; i < n; ++i) {
        const float a = acc[i];
        flag[0] |= !(std::fabs(a) <= 3.4028234663852886e38f);
        const double g = static_cast<double>(a * inv);
        lane[0] += g * g;
    }
    double s = 0.0;
    int b = 0;
    for (int j = 0; j < kLanes; ++j) {
        s += lane[j];
        b |= flag[j];
    }
    *nrm = s;
    *bad = b;
}

// Scan and update together, block by block: each 2048-element block is
// scanned (overflow, squared norm) right before it is updated, so the
// accumulator block is read from memory once. Only for steps whose update
// needs nothing from the scan: no skip (NONE or STATIC mode) and no clipping.
template <bool FP16>
void scan_update_range(const Coeffs c, const float* __restrict acc, float* __restrict p, float* __restrict m,
                       float* __restrict v, uint16_t* __restrict out, int64_t n, double* nrm, int* bad) {
    constexpr int64_t kBlock = 2048;
    for (int64_t b = 0; b < n; b += kBlock) {
        const int64_t k = n - b < kBlock ? n - b : kBlock;
        double bn = 0.0;
        int bb = 0;
        scan_range(acc + b, c.inv, k, &bn, &bb);
        *nrm += bn;
        *bad |= bb;
        update_range<FP16, false>(c, acc + b, p + b, m + b, v + b, out + b, k);
    }
}

// Worker threads kept between calls: a step on a small model, or an update
// issued in several ranges, would otherwise spend a noticeable part of its
// time starting threads. The caller's thread runs job 0 itself. One job runs
// at a time; a call that finds the pool busy (another host thread is inside a
// CPU step) starts its own threads instead. Workers sleep on a condition
// variable between jobs. The pool is never destroyed (its threads simply end
// with the process), and a forked child builds a fresh one.
class WorkerPool {
public:
    static WorkerPool& get() {
        static std::mutex mu;
        static WorkerPool* pool = nullptr;
        std::lock_guard<std::mutex> lk(mu);
        if (!pool || pool->pid_ != getpid()) pool = new WorkerPool();  // a stale child copy is leaked
        return *pool;
    }

    // fn(t) for t in [0, n), t = 0 on the calling thread; returns when all are done
    bool try_run(int n, const std::function<void(int)>& fn) {
        std::unique_lock<std::mutex> busy(job_mu_, std::try_to_lock);
        if (!busy.owns_lock()) return false;
        {
            std::lock_guard<std::mutex> lk(mu_);
            while (static_cast<int>(workers_.size()) < n - 1) {
                const int id = static_cast<int>(workers_.size()) + 1;
                workers_.emplace_back([this, id, g = gen_] { loop(id, g); });
                workers_.back().detach();
            }
            job_ = &fn;
            njob_ = n;
            pending_ = n - 1;
            ++gen_;
        }
        cv_.notify_all();
        fn(0);
        std::unique_lock<std::mutex> lk(mu_);
        done_cv_.wait(lk, [this] { return pending_ == 0; });
        job_ = nullptr;
        return true;
    }

private:
    WorkerPool() : pid_(getpid()) {}

    // `seen` is the generation before the job that started this worker
    void loop(int id, uint64_t seen) {
        for (;;) {
            const std::function<void(int)>* job;
            {
                std::unique_lock<std::mutex> lk(mu_);
                cv_.wait(lk, [&] { return gen_ != seen; });
                seen = gen_;
                if (id >= njob_) continue;
                job = job_;
            }
            (*job)(id);
            std::lock_guard<std::mutex> lk(mu_);
            if (--pending_ == 0) done_cv_.notify_one();
        }
    }

    const pid_t pid_;
    std::mutex job_mu_, mu_;
    std::condition_variable cv_, done_cv_;
    std::vector<std::thread> workers_;
    const std::function<void(int)>* job_ = nullptr;
    int njob_ = 0, pending_ = 0;
    uint64_t gen_ = 0;
};

// fn(t) for t in [0, n) on n threads
template <typename F>
void run_parallel(int n, F&& fn) {
    if (n <= 1) {
        if (n == 1) fn(0);
        return;
    }
    const std::function<void(int)> job = std::ref(fn);
    if (WorkerPool::get().try_run(n, job)) return;
    std::vector<std::thread> pool;
    for (int t = 1; t < n; ++t) pool.emplace_back([&job, t] { job(t); });
    job(0);
    for (auto& th : pool) th.join();
}

// Elements [lo, hi) of every one of R shards, as one index space of R*(hi-lo)
// elements cut into nthreads equal parts: thread t calls fn(t, r, a, b) for
// each shard piece [a, b) of its part, in shard order. One set of threads
// serves all shards (small work runs on the calling thread).
template <typename F>
void parallel_shards(int R, int64_t lo, int64_t hi, int nthreads, F&& fn) {
    const int64_t len = hi - lo, total = static_cast<int64_t>(R) * len;
    auto part = [&](int t, int64_t q0, int64_t q1) {
        while (q0 < q1) {
            const int r = static_cast<int>(q0 / len);
            const int64_t a = lo + (q0 - static_cast<int64_t>(r) * len);
            const int64_t b = std::min(hi, a + (q1 - q0));
            fn(t, r, a, b);
            q0 += b - a;
        }
    };
    if (len <= 0) return;
    if (nthreads <= 1 || total < (int64_t(1) << 16)) {
        part(0, 0, total);
        return;
    }
    const int64_t chunk = (total + nthreads - 1) / nthreads;
    const int used = static_cast<int>((total + chunk - 1) / chunk);
    run_parallel(used, [&](int t) { part(t, t * chunk, std::min(total, (t + 1) * chunk)); });
}

}  // namespace

namespace {

zero_status check_cfg(const zero_loss_scale_config* cfg, const char* where) {
    if (cfg->mode < ZERO_SCALE_NONE || cfg->mode > ZERO_SCALE_DYNAMIC)
        return zb_fail(ZERO_ERR_INVALID_ARG, std::string(where) + ": bad loss-scale mode");
    if (cfg->mode == ZERO_SCALE_DYNAMIC &&
        (cfg->growth_interval < 1 || !(cfg->growth_factor > 1.0f) ||
         !(cfg->backoff_factor > 0.0f && cfg->backoff_factor < 1.0f) || !(cfg->min_scale > 0.0f)))
        return zb_fail(ZERO_ERR_INVALID_ARG, std::string(where) + ": bad dynamic loss-scale config");
    return ZERO_OK;
}

// at most kMaxThreads: a request for more would only start threads that
// compete for the same memory bandwidth
constexpr int kMaxThreads = 1024;

int thread_count(int32_t nthreads) {
    int n = nthreads >= 1 ? nthreads : static_cast<int>(std::thread::hardware_concurrency());
    return n < 1 ? 1 : (n > kMaxThreads ? kMaxThreads : n);
}

// The AdamW coefficients of step t + 1, formed in double and rounded once,
// exactly as the device step forms them.
Coeffs make_coeffs(float inv, float clip, const zero_adamw& hp, int64_t t) {
    Coeffs c;
    const double t1 = static_cast<double>(t + 1);
    c.inv = inv;
    c.dec = static_cast<float>(1.0 - hp.lr * hp.weight_decay);
    c.b1f = static_cast<float>(hp.beta1);
    c.omb1 = static_cast<float>(1.0 - hp.beta1);
    c.b2f = static_cast<float>(hp.beta2);
    c.omb2 = static_cast<float>(1.0 - hp.beta2);
    c.epsf = static_cast<float>(hp.eps);
    c.ss = static_cast<float>(hp.lr / (1.0 - std::pow(hp.beta1, t1)));
    c.bc2s = static_cast<float>(std::sqrt(1.0 - std::pow(hp.beta2, t1)));
    c.clip = clip;
    return c;
}

bool hp_ok(const zero_adamw* hp) {
    return hp->lr >= 0.0 && hp->beta1 >= 0.0 && hp->beta1 < 1.0 && hp->beta2 >= 0.0 && hp->beta2 < 1.0 &&
           hp->eps > 0.0 && hp->weight_decay >= 0.0;
}

// Everything zero_cpu_scan and zero_cpu_update check, for the one-pass step.
zero_status check_step_args(const zero_plan_t* plan, const zero_loss_scale_config* cfg,
                            const zero_loss_scale_state* in, const zero_adamw* hp, const zero_step_opts& o,
                            const float* const* acc, float* const* master, float* const* m, float* const* v,
                            void* const* param) {
    if (!(o.grad_divisor >= 1.0) || !std::isfinite(o.grad_divisor))
        return zb_fail(ZERO_ERR_INVALID_ARG, "zero_cpu_step: need grad_divisor >= 1, finite max_grad_norm >= 0, "
                                             "no flags");
    zero_status st = check_cfg(cfg, "zero_cpu_step");
    if (st != ZERO_OK) return st;
    const float scale = cfg->mode == ZERO_SCALE_NONE ? 1.0f : in->scale;
    if (!(scale > 0.0f) || !std::isfinite(scale) || in->t < 0)
        return zb_fail(ZERO_ERR_INVALID_ARG, "zero_cpu_step: need a finite scale > 0 and t >= 0");
    if (!hp_ok(hp)) return zb_fail(ZERO_ERR_INVALID_ARG, "zero_cpu_step: bad hyper-parameters");
    for (int r = 0; r < plan->R; ++r)
        if (!acc[r] || !master[r] || !m[r] || !v[r] || !param[r])
            return zb_fail(ZERO_ERR_INVALID_ARG, "zero_cpu_step: NULL rank pointer");
    return ZERO_OK;
}

}  // namespace

namespace {

// Options of the CPU step, validated; the fp32 unscale factor into *inv.
zero_status scan_args(const zero_plan_t* plan, const zero_loss_scale_config* cfg, const zero_loss_scale_state* in,
                      const zero_step_opts* opts, zero_step_opts* o, float* inv) {
    *o = zero_step_opts{1.0, 0.0, 0, 0};
    if (opts) *o = *opts;
    if (!(o->grad_divisor >= 1.0) || !std::isfinite(o->grad_divisor) || !(o->max_grad_norm >= 0.0) ||
        !std::isfinite(o->max_grad_norm) || o->flags != 0 || o->reserved != 0)
        return zb_fail(ZERO_ERR_INVALID_ARG, "zero_cpu_step: need grad_divisor >= 1, finite max_grad_norm >= 0, no flags");
    zero_status st = check_cfg(cfg, "zero_cpu_step");
    if (st != ZERO_OK) return st;
    const float scale = cfg->mode == ZERO_SCALE_NONE ? 1.0f : in->scale;
    if (!(scale > 0.0f) || !std::isfinite(scale) || in->t < 0)
        return zb_fail(ZERO_ERR_INVALID_ARG, "zero_cpu_step: need a finite scale > 0 and t >= 0");
    *inv = static_cast<float>(1.0 / ((static_cast<double>(plan->R) * o->grad_divisor) * static_cast<double>(scale)));
    return ZERO_OK;
}

zero_status check_owners(const zero_plan_t* plan, int32_t owner_lo, int32_t owner_hi, const char* where) {
    if (owner_lo < 0 || owner_lo >= owner_hi || owner_hi > plan->R)
        return zb_fail(ZERO_ERR_RANGE, std::string(where) + ": need 0 <= owner_lo < owner_hi <= R");
    return ZERO_OK;
}

// Overflow and squared norm over shards [r0, r1): each thread sums its
// pieces in order, and the per-thread partials are summed in thread order.
void scan_shards(const zero_plan_t* plan, const float* const* acc, float inv, int32_t r0, int32_t r1, int nt,
                 double* nrm, int* overflow) {
    std::vector<double> part(static_cast<size_t>(nt), 0.0);
    std::vector<int> bad(static_cast<size_t>(nt), 0);
    parallel_shards(r1 - r0, 0, plan->S, nt, [&](int t, int i, int64_t a, int64_t b) {
        double pn = 0.0;
        int pb = 0;
        scan_range(acc[r0 + i] + a, inv, b - a, &pn, &pb);
        part[t] += pn;
        bad[t] |= pb;
    });
    double s = 0.0;
    int o = 0;
    for (size_t k = 0; k < part.size(); ++k) {
        s += part[k];
        o |= bad[k];
    }
    *nrm = s;
    *overflow = o;
}

// The step's decision from the (global) squared norm and overflow.
zero_cpu_decision decide(const zero_loss_scale_config* cfg, const zero_step_opts& o, float inv, double nrm,
                         int overflow) {
    zero_cpu_decision d;
    d.grad_norm_sq = nrm;
    d.inv = inv;
    d.clip = 1.0f;
    if (o.max_grad_norm > 0.0) {
        const double cd = o.max_grad_norm / (std::sqrt(nrm) + 1e-6);
        d.clip = static_cast<float>(cd < 1.0 ? cd : 1.0);
    }
    d.overflow = overflow ? 1 : 0;
    d.skip = (cfg->mode == ZERO_SCALE_DYNAMIC && overflow) ? 1 : 0;
    d.clipping = o.max_grad_norm > 0.0 ? 1 : 0;
    d.reserved = 0;
    return d;
}

// Elements [lo, hi) of shards [r0, r1) from a decision.
zero_status update_shards(const zero_plan_t* plan, const zero_loss_scale_state* in, const zero_adamw* hp,
                          const zero_cpu_decision* d, const float* const* acc, float* const* master, float* const* m,
                          float* const* v, void* const* param, int32_t r0, int32_t r1, int64_t lo, int64_t hi,
                          int32_t nthreads) {
    if (!hp_ok(hp)) return zb_fail(ZERO_ERR_INVALID_ARG, "zero_cpu_step: bad hyper-parameters");
    if (in->t < 0) return zb_fail(ZERO_ERR_INVALID_ARG, "zero_cpu_update: need t >= 0");
    for (int r = r0; r < r1; ++r)
        if (!acc[r] || !master[r] || !m[r] || !v[r] || !param[r])
            return zb_fail(ZERO_ERR_INVALID_ARG, "zero_cpu_step: NULL rank pointer");
    if (d->skip || lo == hi) return ZERO_OK;  // a skipped step writes nothing
    const int nt = thread_count(nthreads);
    const Coeffs c = make_coeffs(d->inv, d->clip, *hp, in->t);
    const bool fp16 = plan->dtype == ZERO_FP16, clip = d->clipping != 0;
    parallel_shards(r1 - r0, lo, hi, nt, [&](int, int i, int64_t a, int64_t b) {
        const int r = r0 + i;
        const int64_t n = b - a;
        uint16_t* out = static_cast<uint16_t*>(param[r]) + a;
        if (fp16 && clip) update_range<true, true>(c, acc[r] + a, master[r] + a, m[r] + a, v[r] + a, out, n);
        else if (fp16) update_range<true, false>(c, acc[r] + a, master[r] + a, m[r] + a, v[r] + a, out, n);
        else if (clip) update_range<false, true>(c, acc[r] + a, master[r] + a, m[r] + a, v[r] + a, out, n);
        else update_range<false, false>(c, acc[r] + a, master[r] + a, m[r] + a, v[r] + a, out, n);
    });
    return ZERO_OK;
}

}  // namespace

extern "C" zero_status zero_cpu_scan(const zero_plan_t* plan, const zero_loss_scale_config* cfg,
                                     const zero_loss_scale_state* in, const zero_step_opts* opts,
                                     const float* const* acc, int32_t nthreads, zero_cpu_decision* out) {
    return zb_guarded("zero_cpu_scan", [&]() -> zero_status {
        if (!plan || !cfg || !in || !acc || !out) return zb_fail(ZERO_ERR_INVALID_ARG, "zero_cpu_scan: NULL argument");
        zero_step_opts o;
        float inv = 0.0f;
        zero_status st = scan_args(plan, cfg, in, opts, &o, &inv);
        if (st != ZERO_OK) return st;
        for (int r = 0; r < plan->R; ++r)
            if (!acc[r]) return zb_fail(ZERO_ERR_INVALID_ARG, "zero_cpu_step: NULL rank pointer");
        double nrm = 0.0;
        int overflow = 0;
        scan_shards(plan, acc, inv, 0, plan->R, thread_count(nthreads), &nrm, &overflow);
        *out = decide(cfg, o, inv, nrm, overflow);
        return ZERO_OK;
    });
}

extern "C" zero_status zero_cpu_scan_shard(const zero_plan_t* plan, const zero_loss_scale_config* cfg,
                                           const zero_loss_scale_state* in, const zero_step_opts* opts,
                                           const float* const* acc, int32_t owner_lo, int32_t owner_hi,
                                           int32_t nthreads, double* partial) {
    return zb_guarded("zero_cpu_scan_shard", [&]() -> zero_status {
        if (!plan || !cfg || !in || !acc || !partial)
            return zb_fail(ZERO_ERR_INVALID_ARG, "zero_cpu_scan_shard: NULL argument");
        zero_status st = check_owners(plan, owner_lo, owner_hi, "zero_cpu_scan_shard");
        if (st != ZERO_OK) return st;
        zero_step_opts o;
        float inv = 0.0f;
        if ((st = scan_args(plan, cfg, in, opts, &o, &inv)) != ZERO_OK) return st;
        for (int r = owner_lo; r < owner_hi; ++r)
            if (!acc[r]) return zb_fail(ZERO_ERR_INVALID_ARG, "zero_cpu_scan_shard: NULL owned accumulator");
        double nrm = 0.0;
        int overflow = 0;
        scan_shards(plan, acc, inv, owner_lo, owner_hi, thread_count(nthreads), &nrm, &overflow);
        partial[0] = nrm;
        partial[1] = overflow ? 1.0 : 0.0;
        return ZERO_OK;
    });
}

extern "C" zero_status zero_cpu_decide(const zero_plan_t* plan, const zero_loss_scale_config* cfg,
                                       const zero_loss_scale_state* in, const zero_step_opts* opts,
                                       const double* reduced, zero_cpu_decision* out) {
    return zb_guarded("zero_cpu_decide", [&]() -> zero_status {
        if (!plan || !cfg || !in || !reduced || !out)
            return zb_fail(ZERO_ERR_INVALID_ARG, "zero_cpu_decide: NULL argument");
        zero_step_opts o;
        float inv = 0.0f;
        zero_status st = scan_args(plan, cfg, in, opts, &o, &inv);
        if (st != ZERO_OK) return st;
        if (!(reduced[1] >= 0.0) || !(reduced[0] >= 0.0 || std::isnan(reduced[0])))
            return zb_fail(ZERO_ERR_INVALID_ARG, "zero_cpu_decide: need a norm sum and an overflow count >= 0");
        *out = decide(cfg, o, inv, reduced[0], reduced[1] > 0.0 ? 1 : 0);
        return ZERO_OK;
    });
}

extern "C" zero_status zero_cpu_update(const zero_plan_t* plan, const zero_loss_scale_state* in,
                                       const zero_adamw* hp, const zero_cpu_decision* d,
                                       const float* const* acc, float* const* master, float* const* m,
                                       float* const* v, void* const* param, int64_t lo, int64_t hi,
                                       int32_t nthreads) {
    return zb_guarded("zero_cpu_update", [&]() -> zero_status {
        if (!plan || !in || !hp || !d || !acc || !master || !m || !v || !param)
            return zb_fail(ZERO_ERR_INVALID_ARG, "zero_cpu_update: NULL argument");
        if (lo < 0 || lo > hi || hi > plan->S)
            return zb_fail(ZERO_ERR_RANGE, "zero_cpu_update: need 0 <= lo <= hi <= S");
        return update_shards(plan, in, hp, d, acc, master, m, v, param, 0, plan->R, lo, hi, nthreads);
    });
}

extern "C" zero_status zero_cpu_update_shard(const zero_plan_t* plan, const zero_loss_scale_state* in,
                                             const zero_adamw* hp, const zero_cpu_decision* d,
                                             const float* const* acc, float* const* master, float* const* m,
                                             float* const* v, void* const* param, int32_t owner_lo,
                                             int32_t owner_hi, int32_t nthreads) {
    return zb_guarded("zero_cpu_update_shard", [&]() -> zero_status {
        if (!plan || !in || !hp || !d || !acc || !master || !m || !v || !param)
            return zb_fail(ZERO_ERR_INVALID_ARG, "zero_cpu_update_shard: NULL argument");
        zero_status st = check_owners(plan, owner_lo, owner_hi, "zero_cpu_update_shard");
        if (st != ZERO_OK) return st;
        return update_shards(plan, in, hp, d, acc, master, m, v, param, owner_lo, owner_hi, 0, plan->S, nthreads);
    });
}

extern "C" zero_status zero_cpu_commit(const zero_loss_scale_config* cfg, zero_loss_scale_state* inout,
                                       const zero_cpu_decision* d) {
    return zb_guarded("zero_cpu_commit", [&]() -> zero_status {
        if (!cfg || !inout || !d) return zb_fail(ZERO_ERR_INVALID_ARG, "zero_cpu_commit: NULL argument");
        zero_status st = check_cfg(cfg, "zero_cpu_commit");
        if (st != ZERO_OK) return st;
        // the loss-scale state machine, the same rules as the device step
        int skipped = 0;
        if (cfg->mode == ZERO_SCALE_DYNAMIC) {
            if (d->overflow) {
                const float s = inout->scale * cfg->backoff_factor;
                inout->scale = (s < cfg->min_scale) ? cfg->min_scale : s;
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
        inout->last_overflow = d->overflow;
        inout->last_skipped = skipped;
        inout->grad_norm_sq = d->grad_norm_sq;
        return ZERO_OK;
    });
}

extern "C" zero_status zero_cpu_step(const zero_plan_t* plan, const zero_loss_scale_config* cfg,
                                     zero_loss_scale_state* inout, const zero_adamw* hp,
                                     const zero_step_opts* opts, const float* const* acc, float* const* master,
                                     float* const* m, float* const* v, void* const* param, int32_t nthreads) {
    return zb_guarded("zero_cpu_step", [&]() -> zero_status {
        if (!plan || !cfg || !inout || !hp || !acc || !master || !m || !v || !param)
            return zb_fail(ZERO_ERR_INVALID_ARG, "zero_cpu_step: NULL argument");
        zero_step_opts o{1.0, 0.0, 0, 0};
        if (opts) o = *opts;
        if (o.flags & ~static_cast<int64_t>(ZERO_STEP_CLEAN))
            return zb_fail(ZERO_ERR_INVALID_ARG, "zero_cpu_step: the only flag is ZERO_STEP_CLEAN");
        const bool clean = (o.flags & ZERO_STEP_CLEAN) != 0;
        o.flags = 0;  // the scan and update below take no flags
        const bool one_pass = (cfg->mode != ZERO_SCALE_DYNAMIC || clean) && o.max_grad_norm == 0.0 &&
                              o.reserved == 0;
        if (!one_pass) {
            // the update depends on the whole scan (a skip, or the clipping
            // coefficient): scan every accumulator first
            zero_cpu_decision d;
            zero_status st = zero_cpu_scan(plan, cfg, inout, &o, acc, nthreads, &d);
            if (st == ZERO_OK)
                st = zero_cpu_update(plan, inout, hp, &d, acc, master, m, v, param, 0, plan->S, nthreads);
            if (st == ZERO_OK) st = zero_cpu_commit(cfg, inout, &d);
            return st;
        }
        // NONE / STATIC, or DYNAMIC known clean, without clipping: one pass
        // (scan and update per block)
        zero_cpu_decision d;
        zero_status st = check_step_args(plan, cfg, inout, hp, o, acc, master, m, v, param);
        if (st != ZERO_OK) return st;
        const int R = plan->R;
        const int nt = thread_count(nthreads);
        const float scale = cfg->mode == ZERO_SCALE_NONE ? 1.0f : inout->scale;
        const float inv =
            static_cast<float>(1.0 / ((static_cast<double>(R) * o.grad_divisor) * static_cast<double>(scale)));
        const Coeffs c = make_coeffs(inv, 1.0f, *hp, inout->t);
        const bool fp16 = plan->dtype == ZERO_FP16;
        std::vector<double> part(static_cast<size_t>(nt), 0.0);
        std::vector<int> bad(static_cast<size_t>(nt), 0);
        parallel_shards(R, 0, plan->S, nt, [&](int t, int r, int64_t a, int64_t b) {
            uint16_t* out = static_cast<uint16_t*>(param[r]) + a;
            if (fp16)
                scan_update_range<true>(c, acc[r] + a, master[r] + a, m[r] + a, v[r] + a, out, b - a, &part[t],
                                        &bad[t]);
            else
                scan_update_range<false>(c, acc[r] + a, master[r] + a, m[r] + a, v[r] + a, out, b - a, &part[t],
                                         &bad[t]);
        });
        double nrm = 0.0;
        int overflow = 0;
        for (size_t i = 0; i < part.size(); ++i) {
            nrm += part[i];
            overflow |= bad[i];
        }
        if (overflow && clean && cfg->mode == ZERO_SCALE_DYNAMIC)
            return zb_fail(ZERO_ERR_STATE,
                           "zero_cpu_step: ZERO_STEP_CLEAN, but an accumulator is inf or NaN; the update was "
                           "applied and the loss-scale state left as it was");
        d.grad_norm_sq = nrm;
        d.inv = inv;
        d.clip = 1.0f;
        d.overflow = overflow;
        d.skip = 0;
        d.clipping = 0;
        d.reserved = 0;
        return zero_cpu_commit(cfg, inout, &d);
    });
}
