// The weight gradient of the adjoint, da[g][d] = sum over (b, l) of
// (d pre / d a) du, from the per-tile partial sums the adjoint scan writes
// (partial[r][s][g][kDc], one row r per (b, chunk)), in a fixed order so
// that every run gives the same bits.
//
// Two kernels.  da_slab_kernel splits the rows into `slabs` fixed ranges;
// each block sums one range for one (slab of 128 channels, gate) pair, one
// channel a thread, with eight running sums (row i of the range goes to sum
// i % 8, added pairwise at the end) so that enough loads are in flight to
// stream the partials at HBM speed.  da_final_kernel adds the slab sums in
// slab order.
#pragma once

#include "pararnn_internal.h"

namespace pararnn {

// grid (S*G, slabs), kDc threads
__global__ void __launch_bounds__(kDc) da_slab_kernel(const float* __restrict__ partial, float* __restrict__ sums,
                                                      int rows, int slabs, int SG)
{
    const int sg = blockIdx.x, y = blockIdx.y, dd = threadIdx.x;
    const int r0 = int((long long)rows * y / slabs), r1 = int((long long)rows * (y + 1) / slabs);
    const size_t stride = size_t(SG) * kDc;
    const float* src = partial + (size_t(r0) * SG + sg) * kDc + dd;
    float acc[8] = {0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f};
    int i = 0;
    for (; i + 8 <= r1 - r0; i += 8) {
#pragma unroll
        for (int j = 0; j < 8; ++j) acc[j] += __ldcs(src + size_t(i + j) * stride);
    }
#pragma unroll
    for (int j = 0; j < 7; ++j)
        if (i + j < r1 - r0) acc[j] += __ldcs(src + size_t(i + j) * stride);
    sums[(size_t(y) * SG + sg) * kDc + dd] = ((acc[0] + acc[1]) + (acc[2] + acc[3])) + ((acc[4] + acc[5]) + (acc[6] + acc[7]));
}

// one thread per da entry (g, d); 256 threads a block
__global__ void __launch_bounds__(256) da_final_kernel(const float* __restrict__ sums, float* __restrict__ da,
                                                       int slabs, int S, int G, long long D)
{
    const long long col = blockIdx.x * 256LL + threadIdx.x;
    if (col >= (long long)G * D) return;
    const int g = int(col / D);
    const long long d = col - (long long)g * D;
    const int s = int(d / kDc), dd = int(d - (long long)s * kDc);
    const size_t SG = size_t(S) * G;
    float t = 0.f;
    for (int y = 0; y < slabs; ++y) t += sums[(y * SG + size_t(s) * G + g) * kDc + dd];
    da[col] = t;
}

}  // namespace pararnn
