// The sum of the reduce-scatters' norm shares (ZERO_RS_NORM slots) for a
// sharded step: a rank's part of the global squared gradient norm, which
// the ranks then all-reduce, without reading the accumulator again.
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

}  // namespace zb
