// Small single-block kernels around the reduce-scatters: the sum of their
// norm shares (ZERO_RS_NORM slots) for a sharded step -- a rank's part of the
// global squared gradient norm, which the ranks then all-reduce, without
// reading the accumulator again -- and the hand-over of their overflow flag
// to a step taken elsewhere (the CPU step of ZeRO-Offload).
#include "device_common.cuh"
#include "internal.h"

namespace zb {

// slots [first, first + count) summed in slot order (strided over the block,
// then the block's fixed reduction tree) into out[0]; out[1] = 0.
__global__ void __launch_bounds__(kThreads)
    sum_norm_slots_kernel(const double* slots, int64_t first, int64_t count, double* out) {
    __shared__ double red[kWarps];
    double x = 0.0;
    for (int64_t i = threadIdx.x; i < count; i += kThreads) x += slots[first + i];
    const double total = block_sum(x, red);
    if (threadIdx.x == 0) {
        out[0] = total;
        out[1] = 0.0;
    }
}

cudaError_t launch_sum_norm_slots(const double* slots, int64_t first, int64_t count, double* out,
                                  cudaStream_t s) {
    sum_norm_slots_kernel<<<1, kThreads, 0, s>>>(slots, first, count, out);
    return cudaGetLastError();
}

// *out = 1 if the reduce-scatters since the last step raised the overflow
// flag, else 0; the flag is cleared for the next step.
__global__ void take_overflow_kernel(DevState* st, int32_t* out) {
    if (threadIdx.x == 0 && blockIdx.x == 0) {
        volatile uint32_t* f = &st->flag;
        *out = *f != 0u ? 1 : 0;
        *f = 0u;
        __threadfence();
    }
}

cudaError_t launch_take_overflow(DevState* st, int32_t* out, cudaStream_t s) {
    take_overflow_kernel<<<1, 32, 0, s>>>(st, out);
    return cudaGetLastError();
}

}  // namespace zb
