// One recurrence step for a batch of sequences: the decode step of inference.
//
// Page: "ParaRNN: Apple destrava treino paralelo de RNNs não-lineares e escala
// pra 7B parâmetros" -- "Por que RNN ainda importa": at inference an RNN
// generates each token at a cost that does not grow with the context, since
// the next state depends only on the current state and the new input.  This
// is that step, s_next = f(s_prev, u), for every (b, d) channel at once.
//
// One thread owns four adjacent channels of one batch row: 16-byte state and
// weight loads, 8-byte (bf16) or 16-byte (fp32) gate loads, one 16-byte store
// per state component.  Each thread reads all of its inputs before it writes,
// so the next state may overwrite the previous one in place.
#pragma once

#include "cells.cuh"

namespace pararnn {

__device__ __forceinline__ void load_gates4(const uint16_t* p, float (&v)[4])
{
    const uint2 x = *reinterpret_cast<const uint2*>(p);
    v[0] = __uint_as_float(x.x << 16);
    v[1] = __uint_as_float(x.x & 0xffff0000u);
    v[2] = __uint_as_float(x.y << 16);
    v[3] = __uint_as_float(x.y & 0xffff0000u);
}

__device__ __forceinline__ void load_gates4(const float* p, float (&v)[4])
{
    const float4 x = *reinterpret_cast<const float4*>(p);
    v[0] = x.x;
    v[1] = x.y;
    v[2] = x.z;
    v[3] = x.w;
}

// u [B][G][D], a [G][D], prev[q] [B][D] (nullptr = zeros), next[q] [B][D];
// D a multiple of 4, every row 16-byte aligned.
template <class Cell, class UT>
__global__ void __launch_bounds__(256) decode_step_kernel(const UT* __restrict__ u, const float* __restrict__ a,
                                                          const float* prev0, const float* prev1, float* next0,
                                                          float* next1, long long B, long long D)
{
    constexpr int G = Cell::G, NS = Cell::NS;
    const long long i = (long long)blockIdx.x * blockDim.x + threadIdx.x;
    const long long D4 = D >> 2;
    if (i >= B * D4) return;
    const long long b = i / D4, d = (i - b * D4) << 2;
    const float* prev[2] = {prev0, prev1};
    float* next[2] = {next0, next1};
    float s[NS][4], ug[G][4], ag[G][4];
#pragma unroll
    for (int q = 0; q < NS; ++q) {
        float4 x = make_float4(0.f, 0.f, 0.f, 0.f);
        if (prev[q]) x = *reinterpret_cast<const float4*>(prev[q] + b * D + d);
        s[q][0] = x.x;
        s[q][1] = x.y;
        s[q][2] = x.z;
        s[q][3] = x.w;
    }
#pragma unroll
    for (int g = 0; g < G; ++g) {
        load_gates4(u + (b * G + g) * D + d, ug[g]);
        const float4 x = __ldg(reinterpret_cast<const float4*>(a + g * D + d));
        ag[g][0] = x.x;
        ag[g][1] = x.y;
        ag[g][2] = x.z;
        ag[g][3] = x.w;
    }
    float f[NS][4];
#pragma unroll
    for (int j = 0; j < 4; ++j) {
        float sj[NS], uj[G], aj[G], fj[NS];
#pragma unroll
        for (int q = 0; q < NS; ++q) sj[q] = s[q][j];
#pragma unroll
        for (int g = 0; g < G; ++g) {
            uj[g] = ug[g][j];
            aj[g] = ag[g][j];
        }
        Cell::value(sj, uj, aj, fj);
#pragma unroll
        for (int q = 0; q < NS; ++q) f[q][j] = fj[q];
    }
#pragma unroll
    for (int q = 0; q < NS; ++q)
        *reinterpret_cast<float4*>(next[q] + b * D + d) = make_float4(f[q][0], f[q][1], f[q][2], f[q][3]);
}

}  // namespace pararnn
