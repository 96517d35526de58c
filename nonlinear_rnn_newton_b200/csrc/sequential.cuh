// Naive sequential application on the GPU: one thread per (b, d) channel
// walks l = 1..L, the "traditional sequential application" the page
// "ParaRNN: Apple destrava treino paralelo de RNNs não-lineares e escala pra
// 7B parâmetros" compares against (section "O compromisso que SSMs fizeram":
// h_l = sigma(h_{l-1}, x_l) one step at a time).  A baseline, not the method.
#pragma once

#include "cells.cuh"

namespace pararnn {

__device__ __forceinline__ float load_gate(const uint16_t* p) { return __uint_as_float(uint32_t(*p) << 16); }
__device__ __forceinline__ float load_gate(const float* p) { return *p; }

template <class Cell, class UT>
__global__ void __launch_bounds__(64) sequential_kernel(const UT* __restrict__ u, const float* __restrict__ a,
                                                        const float* s00, const float* s01, float* st0,
                                                        float* st1, long long B, long long L, long long D)
{
    constexpr int G = Cell::G, NS = Cell::NS;
    constexpr int P = 8;  // rows of u loaded ahead of the dependency chain
    const long long idx = (long long)blockIdx.x * blockDim.x + threadIdx.x;
    if (idx >= B * D) return;
    const long long b = idx / D, d = idx - (idx / D) * D;
    const float* s0[2] = {s00, s01};
    float* st[2] = {st0, st1};
    float s[NS], aa[G];
#pragma unroll
    for (int q = 0; q < NS; ++q) s[q] = s0[q] ? s0[q][b * D + d] : 0.0f;
#pragma unroll
    for (int g = 0; g < G; ++g) aa[g] = a[g * D + d];
    const UT* ub = u + (b * L) * G * D + d;
    float buf[P][G];
#pragma unroll
    for (int t = 0; t < P; ++t)
#pragma unroll
        for (int g = 0; g < G; ++g) buf[t][g] = t < L ? load_gate(ub + ((long long)t * G + g) * D) : 0.f;
    for (long long l0 = 0; l0 < L; l0 += P) {
        float nxt[P][G];
#pragma unroll
        for (int t = 0; t < P; ++t) {
            const long long l = l0 + P + t;
#pragma unroll
            for (int g = 0; g < G; ++g) nxt[t][g] = l < L ? load_gate(ub + (l * G + g) * D) : 0.f;
        }
#pragma unroll
        for (int t = 0; t < P; ++t) {
            const long long l = l0 + t;
            if (l < L) {
                float f[NS];
                Cell::value(s, buf[t], aa, f);
#pragma unroll
                for (int q = 0; q < NS; ++q) {
                    s[q] = f[q];
                    st[q][(b * L + l) * D + d] = f[q];
                }
            }
        }
#pragma unroll
        for (int t = 0; t < P; ++t)
#pragma unroll
            for (int g = 0; g < G; ++g) buf[t][g] = nxt[t][g];
    }
}

}  // namespace pararnn
