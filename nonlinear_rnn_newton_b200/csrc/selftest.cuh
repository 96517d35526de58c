// Self tests of the bounded device-side waits: each kernel runs one wait
// against a condition that nothing satisfies, so the wait must give up after
// its limit, raise PARARNN_ERR_TIMEOUT in the workspace header and return.
#pragma once

#include "scan_common.cuh"

namespace pararnn {

// The walking look-back of tile 1 whose predecessor (tile 0) never
// publishes.  One warp.
__global__ void selftest_lookback_kernel(unsigned long long* desc, int* err, unsigned long long limit_ns)
{
    const int lane = threadIdx.x & 31;
    Aff<1> ta[kV];
#pragma unroll
    for (int j = 0; j < kV; ++j) ta[j] = Aff<1>::identity();
    publish_aggregate<Aff<1>, 1>(desc, 1, 0, ta, lane);
    LookbackProbe<Aff<1>, 1> pr;
    lookback_probe(pr, 0, desc, lane);
    float carry[1][kV];
    (void)lookback_resolve<Aff<1>, 1, true>(1, 1, 0, carry, desc, lane, err, limit_ns, pr);
}

// The grid barrier with one CTA that never arrives.
__global__ void selftest_barrier_kernel(unsigned* counter, int* err, unsigned long long limit_ns)
{
    __shared__ int s_flag;
    if (blockIdx.x == gridDim.x - 1) return;
    (void)grid_barrier(counter, 0u, err, limit_ns, &s_flag);
}

}  // namespace pararnn
