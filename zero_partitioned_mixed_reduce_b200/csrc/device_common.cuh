// Device-side helpers shared by the kernels of libzero_b200.so: 8-element
// vector memory access, half-format packing, the one-element AdamW update
// (one rounded fp32 operation per line), block reductions, and the owner of a
// flat index. Included by kernels.cu and noalloc.cu only.
#pragma once

#include <cuda_bf16.h>
#include <cuda_fp16.h>
#include <cuda_runtime.h>

#include <cfloat>
#include <cstdint>
#include <cstring>

#include "internal.h"

namespace zb {

constexpr int kThreads = 256;
constexpr int kWarps = kThreads / 32;

// ---------------------------------------------------------------------------
// Memory access helpers.
// ---------------------------------------------------------------------------

struct F8 {
    float x[8];
};

// Gradients are read exactly once per step and never written by the step:
// read-only path, no L1 allocation.
__device__ __forceinline__ uint4 ld_grad(const uint4* p) {
    uint4 r;
    asm volatile("ld.global.nc.L1::no_allocate.v4.u32 {%0,%1,%2,%3}, [%4];"
                 : "=r"(r.x), "=r"(r.y), "=r"(r.z), "=r"(r.w)
                 : "l"(p));
    return r;
}

__device__ __forceinline__ uint16_t ld_grad1(const uint16_t* p) {
    uint16_t r;
    asm volatile("ld.global.nc.L1::no_allocate.u16 %0, [%1];" : "=h"(r) : "l"(p));
    return r;
}

// 8 fp32 values with one 256-bit access (sm_100); p is 32-byte aligned.
__device__ __forceinline__ F8 ld_f8(const float* p) {
    F8 r;
    asm volatile("ld.global.L1::no_allocate.v8.f32 {%0,%1,%2,%3,%4,%5,%6,%7}, [%8];"
                 : "=f"(r.x[0]), "=f"(r.x[1]), "=f"(r.x[2]), "=f"(r.x[3]), "=f"(r.x[4]),
                   "=f"(r.x[5]), "=f"(r.x[6]), "=f"(r.x[7])
                 : "l"(p));
    return r;
}

__device__ __forceinline__ void st_f8(float* p, const F8& v) {
    asm volatile("st.global.v8.f32 [%0], {%1,%2,%3,%4,%5,%6,%7,%8};" ::"l"(p), "f"(v.x[0]),
                 "f"(v.x[1]), "f"(v.x[2]), "f"(v.x[3]), "f"(v.x[4]), "f"(v.x[5]), "f"(v.x[6]),
                 "f"(v.x[7])
                 : "memory");
}

__device__ __forceinline__ void st_u4(void* p, const uint4& v) {
    asm volatile("st.global.v4.u32 [%0], {%1,%2,%3,%4};" ::"l"(p), "r"(v.x), "r"(v.y), "r"(v.z),
                 "r"(v.w)
                 : "memory");
}

// ---------------------------------------------------------------------------
// Half formats: two values per 32-bit word, element 0 in the low half.
// ---------------------------------------------------------------------------

struct Bf16 {
    static __device__ __forceinline__ float2 unpack(uint32_t w) {
        // a bf16 is the top half of the fp32 with the same value
        return make_float2(__uint_as_float(w << 16), __uint_as_float(w & 0xffff0000u));
    }
    static __device__ __forceinline__ float one(uint16_t h) {
        return __uint_as_float(static_cast<uint32_t>(h) << 16);
    }
    static __device__ __forceinline__ uint32_t pack(float lo, float hi) {
        __nv_bfloat162 h = __floats2bfloat162_rn(lo, hi);
        uint32_t w;
        memcpy(&w, &h, 4);
        return w;
    }
};

struct Fp16 {
    static __device__ __forceinline__ float2 unpack(uint32_t w) {
        __half2 h;
        memcpy(&h, &w, 4);
        return __half22float2(h);
    }
    static __device__ __forceinline__ float one(uint16_t h) {
        return __half2float(__ushort_as_half(h));
    }
    static __device__ __forceinline__ uint32_t pack(float lo, float hi) {
        __half2 h = __floats2half2_rn(lo, hi);
        uint32_t w;
        memcpy(&w, &h, 4);
        return w;
    }
};

template <typename H>
__device__ __forceinline__ void unpack8(const uint4& q, float* f) {
    float2 a = H::unpack(q.x), b = H::unpack(q.y), c = H::unpack(q.z), d = H::unpack(q.w);
    f[0] = a.x; f[1] = a.y; f[2] = b.x; f[3] = b.y;
    f[4] = c.x; f[5] = c.y; f[6] = d.x; f[7] = d.y;
}

template <typename H>
__device__ __forceinline__ void add8(const uint4& q, float* f) {
    float g[8];
    unpack8<H>(q, g);
#pragma unroll
    for (int e = 0; e < 8; ++e) f[e] = __fadd_rn(f[e], g[e]);
}

template <typename H>
__device__ __forceinline__ uint4 pack8(const float* f) {
    return make_uint4(H::pack(f[0], f[1]), H::pack(f[2], f[3]), H::pack(f[4], f[5]),
                      H::pack(f[6], f[7]));
}

__device__ __forceinline__ bool nonfinite(float x) { return !(fabsf(x) <= FLT_MAX); }

// ---------------------------------------------------------------------------
// AdamW on one element. Every line is one rounded fp32 operation.
// ---------------------------------------------------------------------------

struct Coef {
    float inv, dec, b1f, omb1, b2f, omb2, epsf, ss, bc2s;
    float clip;  // global-norm clipping coefficient; exactly 1 when clipping is off
};

// Returns the unscaled gradient before clipping (for the norm); with CLIP the
// update uses it times the clipping coefficient.
template <bool CLIP = false>
__device__ __forceinline__ float adamw1(const Coef& c, float acc, float& p, float& m, float& v) {
    const float g0 = __fmul_rn(acc, c.inv);
    const float g = CLIP ? __fmul_rn(g0, c.clip) : g0;
    float pp = __fmul_rn(p, c.dec);
    const float mm = __fadd_rn(__fmul_rn(c.b1f, m), __fmul_rn(c.omb1, g));
    const float vv = __fadd_rn(__fmul_rn(c.b2f, v), __fmul_rn(c.omb2, __fmul_rn(g, g)));
    const float den = __fadd_rn(__fdiv_rn(__fsqrt_rn(vv), c.bc2s), c.epsf);
    pp = __fsub_rn(pp, __fmul_rn(c.ss, __fdiv_rn(mm, den)));
    p = pp;
    m = mm;
    v = vv;
    return g0;
}

// ---------------------------------------------------------------------------
// Block reductions.
// ---------------------------------------------------------------------------

__device__ __forceinline__ double warp_sum(double x) {
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) x += __shfl_xor_sync(0xffffffffu, x, o);
    return x;
}

// Deterministic for a fixed grid: fixed per-thread order, fixed tree. NW is
// the block's warp count (smem holds NW entries); every thread calls it.
template <int NW = kWarps>
__device__ __forceinline__ double block_sum(double x, double* smem) {
    static_assert(NW >= 1 && NW <= 32, "one warp sums the warps' partials");
    x = warp_sum(x);
    const int w = threadIdx.x >> 5, l = threadIdx.x & 31;
    __syncthreads();
    if (l == 0) smem[w] = x;
    __syncthreads();
    double r = 0.0;
    if (w == 0) {
        r = l < NW ? smem[l] : 0.0;
        r = warp_sum(r);
    }
    return r;  // valid in thread 0
}

// First vector of this thread's grid-stride sequence over [v0, ...): the
// sequence is laid on 128-byte lines of the half-precision gradients (8
// vectors of 16 bytes) starting at or below v0, so every warp reads whole
// lines; a thread whose first vector falls below v0 starts one stride later.
// A start that is not on a line boundary made each warp straddle one more
// line per gradient stream, about 15 % slower at R = 16.
__device__ __forceinline__ uint32_t line_start(uint32_t v0, uint32_t stride) {
    const uint32_t v = (v0 & ~7u) + blockIdx.x * blockDim.x + threadIdx.x;
    return v < v0 ? v + stride : v;
}

// Owner of a flat vector index, tracked incrementally along a grid-stride loop.
struct OwnerCursor {
    uint32_t o, base, S8;
    __device__ __forceinline__ OwnerCursor(uint32_t v, uint32_t s8) : S8(s8) {
        o = v / s8;
        base = o * s8;
    }
    __device__ __forceinline__ void seek(uint32_t v) {
        while (v - base >= S8) {
            base += S8;
            ++o;
        }
    }
};

}  // namespace zb
