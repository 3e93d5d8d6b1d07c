// Bounds checks of the debug build (ZERO_DEBUG_BOUNDS). ZB_IN(cond, site,
// index) guards an access: in the debug build a false cond is counted, the
// first failing site and index are kept, and the caller skips the access; in
// the release build it is the constant true and cond is not evaluated.
// Every .cu file of the library is its own CUDA module and keeps its own
// record (the counters have internal linkage); zero_debug_bounds sums them.
// Sites: 1 fused vector, 2 fused accumulator, 3 staged tile issue, 4 staged
// tile store, 5 two-pass vector, 6 accumulator norm, 7 replica norm,
// 8 reduce-scatter vector, 9 reduce-scatter element, 10 gather vector,
// 11 gather element, 12 reduce-scatter norm partial, 13 static-scratch step
// vector.
#pragma once

#include <cuda_runtime.h>

#ifdef ZERO_DEBUG_BOUNDS
namespace zb {
static __device__ unsigned long long g_bounds_count = 0;
static __device__ unsigned long long g_bounds_first = 0;

static __device__ __noinline__ bool bounds_fail(unsigned site, unsigned long long index) {
    atomicAdd(&g_bounds_count, 1ull);
    atomicCAS(&g_bounds_first, 0ull, (static_cast<unsigned long long>(site) << 48) | (index & 0xffffffffffffull));
    return false;
}

// This module's record (after the device's work so far), optionally cleared.
static inline cudaError_t bounds_record(unsigned long long* count, unsigned long long* first, bool reset) {
    cudaError_t e = cudaDeviceSynchronize();
    if (e == cudaSuccess) e = cudaMemcpyFromSymbol(count, g_bounds_count, sizeof *count);
    if (e == cudaSuccess) e = cudaMemcpyFromSymbol(first, g_bounds_first, sizeof *first);
    if (e == cudaSuccess && reset) {
        const unsigned long long zero = 0;
        e = cudaMemcpyToSymbol(g_bounds_count, &zero, sizeof zero);
        if (e == cudaSuccess) e = cudaMemcpyToSymbol(g_bounds_first, &zero, sizeof zero);
    }
    return e;
}
}  // namespace zb
#define ZB_IN(cond, site, index) ((cond) ? true : ::zb::bounds_fail((site), (index)))
#else
#define ZB_IN(cond, site, index) true
#endif
