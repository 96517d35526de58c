// Pieces of the Newton solve with the sequence split into segments (one per
// GPU), beside the fused pass (newton_solve_ws_kernel in segment mode).
//
// Page: "ParaRNN: Apple destrava treino paralelo de RNNs não-lineares e escala
// pra 7B parâmetros" -- "A sacada: método de Newton": each iteration solves a
// linear recurrence s^{k+1}_l = J_l s^{k+1}_{l-1} + o_l.  Over a segment that
// starts after step l0 - 1 its solution is affine in the state entering the
// segment, c = s^{k+1}_{l0-1}:  s^{k+1}_l = beta_l + A_l c.  One pass with
// c = 0 gives beta, one pass with c = e_j per state component gives
// beta + A e_j; the maps of the segments' last steps, gathered from every
// GPU and composed in order, give each segment its c (a scan over segments),
// and a fix-up writes s^{k+1} = beta + A c and the residual of the result.
#pragma once

#include "cells.cuh"

namespace pararnn {

// Ring slot 0 of the chunk-boundary rows [NS][B][n_chunks][Dpad] from a given
// iterate [NS][B][L][D]: row c holds the state at the end of chunk c, step
// (c+1)*Lc - 1 (c < n_chunks - 1), which is where a pass reads the state
// entering chunk c + 1; a warm-started first pass then finds it where a later
// pass would.  One thread per 4 channels.
__global__ void __launch_bounds__(256) bnd_gather_kernel(const float* __restrict__ in0, const float* __restrict__ in1,
                                                         float* __restrict__ bnd, int NS, long long B, long long L,
                                                         long long D, int n_chunks, int Lc, int Dpad)
{
    const long long D4 = D >> 2;
    const long long per_q = B * (n_chunks - 1) * D4;
    const long long i = (long long)blockIdx.x * blockDim.x + threadIdx.x;
    if (n_chunks < 2 || i >= NS * per_q) return;
    const int q = int(i / per_q);
    long long r = i - q * per_q;
    const long long d = (r % D4) << 2;
    r /= D4;
    const int c = int(r % (n_chunks - 1)) + 1;
    const long long b = r / (n_chunks - 1);
    const float* src = (q == 0 ? in0 : in1) + (b * L + (long long)c * Lc - 1) * D + d;  // end of chunk c - 1
    float* dst = bnd + (((long long)q * B + b) * n_chunks + (c - 1)) * Dpad + d;
    *reinterpret_cast<float4*>(dst) = *reinterpret_cast<const float4*>(src);
}

__device__ __forceinline__ float gate_value(const uint16_t* p) { return __uint_as_float(uint32_t(*p) << 16); }
__device__ __forceinline__ float gate_value(const float* p) { return *p; }

// s = beta + sum_j (unit_j - beta) c_j over the segment, and max |F| of the
// result, F_l = s_l - f(s_{l-1}, u_l) with s_{-1} = c.
//   beta [NS][B][L][D], unit [NS (j)][NS][B][L][D] (the pass with c = e_j),
//   carry [NS][B][D], out [NS][B][L][D], res: max |F| as float bits
//   (non-negative floats order like their bits; NaN kept).
// One thread per (b, l, d).
template <class Cell, class UT>
__global__ void __launch_bounds__(256) segment_update_kernel(const UT* __restrict__ u, const float* __restrict__ a,
                                                             const float* __restrict__ beta,
                                                             const float* __restrict__ unit,
                                                             const float* __restrict__ carry, float* __restrict__ out,
                                                             unsigned* res, long long B, long long L, long long D)
{
    constexpr int G = Cell::G, NS = Cell::NS;
    const long long per = B * L * D;
    const long long i = (long long)blockIdx.x * blockDim.x + threadIdx.x;
    float emax = 0.f;
    if (i < per) {
        const long long d = i % D, bl = i / D, b = bl / L, l = bl - b * L;
        float c[NS];
#pragma unroll
        for (int q = 0; q < NS; ++q) c[q] = carry[(q * B + b) * D + d];
        auto fix = [&](long long idx, int q) {
            const float be = beta[q * per + idx];
            float v = be;
#pragma unroll
            for (int j = 0; j < NS; ++j) v = fmaf(unit[(j * NS + q) * per + idx] - be, c[j], v);
            return v;
        };
        float cur[NS], prv[NS], uu[G], aa[G], f[NS];
#pragma unroll
        for (int q = 0; q < NS; ++q) {
            cur[q] = fix(i, q);
            prv[q] = l > 0 ? fix(i - D, q) : c[q];
            out[q * per + i] = cur[q];
        }
#pragma unroll
        for (int g = 0; g < G; ++g) {
            uu[g] = gate_value(u + (bl * G + g) * D + d);
            aa[g] = a[g * D + d];
        }
        Cell::value(prv, uu, aa, f);
#pragma unroll
        for (int q = 0; q < NS; ++q) {
            const float e = fabsf(cur[q] - f[q]);
            emax = (e > emax || e != e) ? e : emax;
        }
    }
    // block maximum, NaN kept
#pragma unroll
    for (int off = 16; off > 0; off >>= 1) {
        const float o = __shfl_xor_sync(0xffffffffu, emax, off);
        emax = (o > emax || o != o) ? o : emax;
    }
    __shared__ float wmax[8];
    if ((threadIdx.x & 31) == 0) wmax[threadIdx.x >> 5] = emax;
    __syncthreads();
    if (threadIdx.x == 0) {
        float m = 0.f;
        for (int w = 0; w < int(blockDim.x >> 5); ++w) m = (wmax[w] > m || wmax[w] != wmax[w]) ? wmax[w] : m;
        atomicMax(res, __float_as_uint(m) & 0x7fffffffu);
    }
}

// The state entering every segment, from the segments' last-step values:
//   ends [R][1 + NS][NS][B][D]: per segment, its last step's state in the
//   pass with c = 0 (beta) and in the passes with c = e_j;
//   s0 [NS][B][D] (NULL = zeros) enters segment 0;
//   carries [R][NS][B][D]: c_0 = s0, c_{r+1} = beta_r + sum_j (unit_rj - beta_r) c_r[j].
template <int NS>
__global__ void __launch_bounds__(256) segment_carries_kernel(const float* __restrict__ ends,
                                                              const float* __restrict__ s0,
                                                              float* __restrict__ carries, int R, long long BD)
{
    const long long i = (long long)blockIdx.x * blockDim.x + threadIdx.x;
    if (i >= BD) return;
    float c[NS];
#pragma unroll
    for (int q = 0; q < NS; ++q) c[q] = s0 ? s0[q * BD + i] : 0.f;
    for (int r = 0; r < R; ++r) {
        float nc[NS];
#pragma unroll
        for (int q = 0; q < NS; ++q) {
            carries[((long long)r * NS + q) * BD + i] = c[q];
            const float be = ends[((long long)r * (1 + NS) * NS + q) * BD + i];
            float v = be;
#pragma unroll
            for (int j = 0; j < NS; ++j)
                v = fmaf(ends[(((long long)r * (1 + NS) + 1 + j) * NS + q) * BD + i] - be, c[j], v);
            nc[q] = v;
        }
#pragma unroll
        for (int q = 0; q < NS; ++q) c[q] = nc[q];
    }
}

}  // namespace pararnn
