// Pieces of the Newton solve with the sequence split into segments (one per
// GPU), beside the fused pass (newton_solve_ws_kernel in segment mode).
//
// Page: "ParaRNN: Apple destrava treino paralelo de RNNs não-lineares e escala
// pra 7B parâmetros" -- "A sacada: método de Newton": each iteration solves a
// linear recurrence s^{k+1}_l = J_l s^{k+1}_{l-1} + o_l whose step maps
// depend only on the iterate H^k.  Over a segment their composition is one
// affine map of the state entering the segment.  Per iteration each GPU folds
// its segment's step maps (segment_fold_kernel, segment_record_kernel), the
// segments' records are gathered from every GPU (the one data exchange), and
// every GPU composes them in order into the state entering its own segment
// (segment_combine_kernel); one fused pass in segment mode then writes the
// segment's next iterate and its residual.
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

__device__ __forceinline__ float max_nan(float a, float b) { return (b > a || b != b) ? b : a; }

// Block-wide maximum (NaN kept) folded into *res as float bits
// (non-negative floats order like their bits).
__device__ __forceinline__ void block_max_into(float v, unsigned* res)
{
#pragma unroll
    for (int off = 16; off > 0; off >>= 1) v = max_nan(v, __shfl_xor_sync(0xffffffffu, v, off));
    __shared__ float wmax[32];
    if ((threadIdx.x & 31) == 0) wmax[threadIdx.x >> 5] = v;
    __syncthreads();
    if (threadIdx.x == 0) {
        float m = 0.f;
        for (int w = 0; w < int((blockDim.x + 31) >> 5); ++w) m = max_nan(m, wmax[w]);
        atomicMax(res, __float_as_uint(m) & 0x7fffffffu);
    }
}

// Record a segment contributes to an iteration of the split solve, per
// channel, fields [F][B][D] with F = NC + 2 NS + G, then one float:
//   fold  [NC]: the composition of the step maps s -> J_l s + o_l of steps
//               1..Ls-1 of the segment (identity if Ls = 1), linearised at
//               the iterate H^k;
//   last  [NS]: H^k at the segment's last step (the next segment's first
//               step is linearised there);
//   first [NS]: H^k at the segment's first step;
//   gates [G]:  the first step's gate pre-activations (fp32);
//   then max |F_l(H^k)| over steps 1..Ls-1 (float, NaN kept).
template <class Cell>
struct SegRecord {
    static constexpr int NC = Cell::Map::kFloats, NS = Cell::NS, G = Cell::G;
    static constexpr int F = NC + 2 * NS + G;
    static constexpr int fold = 0, last = NC, first = NC + NS, gates = NC + 2 * NS;
    static __host__ __device__ long long floats(long long BD) { return F * BD + 4; }
};

// Steps folded per thread in segment_fold_kernel: the fewest of 64, 128,
// 256, ... that leave at most kFoldParts parts to compose in order (so that
// short segments still give every SM several warps, and the parts of a long
// one stay few for segment_record_kernel's serial composition).
constexpr int kFoldParts = 256;
__host__ __device__ inline long long fold_steps(long long Ls)
{
    long long steps = 64;
    while ((Ls - 1 + steps - 1) / steps > kFoldParts) steps *= 2;
    return steps;
}

// Fold of steps [1 + f*steps, 1 + (f+1)*steps) of a segment (f =
// blockIdx.y) for 4 channels a thread: the step maps at H^k (s_in, NULL = the
// zero guess) composed in order into part [nf][NC][B][D], and max |F| of the
// steps into *res.  Page: "A sacada: método de Newton" (the Newton step is the
// linear recurrence s^{k+1}_l = J_l s^{k+1}_{l-1} + o_l, o_l = f_l - J_l s^k_{l-1}).
// A step's map needs only H^k, so two consecutive steps are evaluated
// together in the packed two-row form of the cell (channel pairs in float2,
// reciprocals shared between the rows), as in the fused pass.
template <class Cell, class UT>
__global__ void __launch_bounds__(128) segment_fold_kernel(const UT* __restrict__ u, const float* __restrict__ a,
                                                           const float* __restrict__ s_in, float* __restrict__ part,
                                                           unsigned* res, long long B, long long Ls, long long D,
                                                           int steps)
{
    using Packed = typename Cell::Packed;
    using Map2 = typename Packed::Map2;
    using Rows2 = typename Packed::Rows2;
    constexpr int G = Cell::G, NS = Cell::NS, NC = Cell::Map::kFloats, NP = kV / 2;
    const long long D4 = D >> 2, BD = B * D, per = B * Ls * D;
    const long long i = (long long)blockIdx.x * blockDim.x + threadIdx.x;
    float rmax = 0.f;
    if (i < B * D4) {
        const long long b = i / D4, d = (i - b * D4) << 2;
        const long long l0 = 1 + (long long)blockIdx.y * steps;
        const long long l1 = l0 + steps < Ls ? l0 + steps : Ls;
        float2 av[G][NP];
#pragma unroll
        for (int g = 0; g < G; ++g) {
            const F4 x = load4(a + g * D + d);
#pragma unroll
            for (int jp = 0; jp < NP; ++jp) av[g][jp] = make_float2(x.v[2 * jp], x.v[2 * jp + 1]);
        }
        // gates and H^k of step l, as channel pairs
        auto load_step = [&](long long l, float2 (&ug)[G][NP], float2 (&hk)[NS][NP]) {
#pragma unroll
            for (int g = 0; g < G; ++g) {
                const F4 x = load4(u + ((b * Ls + l) * G + g) * D + d);
#pragma unroll
                for (int jp = 0; jp < NP; ++jp) ug[g][jp] = make_float2(x.v[2 * jp], x.v[2 * jp + 1]);
            }
#pragma unroll
            for (int q = 0; q < NS; ++q) {
                F4 x{{0.f, 0.f, 0.f, 0.f}};
                if (s_in) x = load4(s_in + q * per + (b * Ls + l) * D + d);
#pragma unroll
                for (int jp = 0; jp < NP; ++jp) hk[q][jp] = make_float2(x.v[2 * jp], x.v[2 * jp + 1]);
            }
        };
        auto keep_max = [&](float2 h, float2 f) {
            rmax = max_nan(rmax, fabsf(h.x - f.x));
            rmax = max_nan(rmax, fabsf(h.y - f.y));
        };
        // H^k before the first step
        float2 prev[NS][NP];
#pragma unroll
        for (int q = 0; q < NS; ++q) {
            F4 x{{0.f, 0.f, 0.f, 0.f}};
            if (s_in) x = load4(s_in + q * per + (b * Ls + l0 - 1) * D + d);
#pragma unroll
            for (int jp = 0; jp < NP; ++jp) prev[q][jp] = make_float2(x.v[2 * jp], x.v[2 * jp + 1]);
        }
        Map2 acc[NP];
#pragma unroll
        for (int jp = 0; jp < NP; ++jp) acc[jp] = Map2::identity();
        long long l = l0;
        // (both steps' loads are in flight together; unrolling further measured
        // slower, from the registers it takes)
#pragma unroll 1
        for (; l + 1 < l1; l += 2) {
            float2 ua[G][NP], ub[G][NP], ha[NS][NP], hb[NS][NP];
            load_step(l, ua, ha);
            load_step(l + 1, ub, hb);
#pragma unroll
            for (int jp = 0; jp < NP; ++jp) {
                float2 sa[NS], sb[NS], u_a[G], u_b[G], aa[G], fa[NS], fb[NS], ja[NS], jb[NS], oa[NS], ob[NS];
#pragma unroll
                for (int q = 0; q < NS; ++q) {
                    sa[q] = prev[q][jp];
                    sb[q] = ha[q][jp];
                }
#pragma unroll
                for (int g = 0; g < G; ++g) {
                    u_a[g] = ua[g][jp];
                    u_b[g] = ub[g][jp];
                    aa[g] = av[g][jp];
                }
                Map2 ea, eb;
                Rows2::eval(sa, u_a, sb, u_b, aa, fa, fb, ea, eb);
                apply_matrix2(ea, sa, ja);
                apply_matrix2(eb, sb, jb);
#pragma unroll
                for (int q = 0; q < NS; ++q) {
                    oa[q] = fma2(ja[q], bc2(-1.0f), fa[q]);
                    ob[q] = fma2(jb[q], bc2(-1.0f), fb[q]);
                    keep_max(ha[q][jp], fa[q]);
                    keep_max(hb[q][jp], fb[q]);
                    prev[q][jp] = hb[q][jp];
                }
                set_offset2(ea, oa);
                set_offset2(eb, ob);
                acc[jp] = compose(eb, compose(ea, acc[jp]));
            }
        }
        if (l < l1) {  // an odd step left
            float2 ua[G][NP], ha[NS][NP];
            load_step(l, ua, ha);
#pragma unroll
            for (int jp = 0; jp < NP; ++jp) {
                float2 sa[NS], u_a[G], aa[G], fa[NS], ja[NS], oa[NS];
#pragma unroll
                for (int q = 0; q < NS; ++q) sa[q] = prev[q][jp];
#pragma unroll
                for (int g = 0; g < G; ++g) {
                    u_a[g] = ua[g][jp];
                    aa[g] = av[g][jp];
                }
                Map2 ea;
                Packed::eval(sa, u_a, aa, fa, ea);
                apply_matrix2(ea, sa, ja);
#pragma unroll
                for (int q = 0; q < NS; ++q) {
                    oa[q] = fma2(ja[q], bc2(-1.0f), fa[q]);
                    keep_max(ha[q][jp], fa[q]);
                }
                set_offset2(ea, oa);
                acc[jp] = compose(ea, acc[jp]);
            }
        }
#pragma unroll
        for (int c = 0; c < NC; ++c) {
            float v[kV];
#pragma unroll
            for (int jp = 0; jp < NP; ++jp) {
                v[2 * jp] = acc[jp].lane(0).get(c);
                v[2 * jp + 1] = acc[jp].lane(1).get(c);
            }
            store4(part + ((long long)blockIdx.y * NC + c) * BD + b * D + d, v);
        }
    }
    block_max_into(rmax, res);
}

// The segment's record (SegRecord) from the fold parts: the parts composed in
// order, H^k at the first and last steps, the first step's gates.  One
// thread per channel.
template <class Cell, class UT>
__global__ void __launch_bounds__(256) segment_record_kernel(const UT* __restrict__ u, const float* __restrict__ s_in,
                                                             const float* __restrict__ part, int nf,
                                                             float* __restrict__ rec, long long B, long long Ls,
                                                             long long D)
{
    using Map = typename Cell::Map;
    using R = SegRecord<Cell>;
    constexpr int G = Cell::G, NS = Cell::NS, NC = Map::kFloats;
    const long long BD = B * D, per = B * Ls * D;
    const long long i = (long long)blockIdx.x * blockDim.x + threadIdx.x;
    if (i >= BD) return;
    const long long b = i / D, d = i - b * D;
    Map acc = Map::identity();
    // (unrolled, so that the reads of several parts are in flight while the
    // compositions form the chain)
#pragma unroll 8
    for (int f = 0; f < nf; ++f) {
        Map m;
#pragma unroll
        for (int c = 0; c < NC; ++c) m.set(c, part[((long long)f * NC + c) * BD + i]);
        acc = compose(m, acc);
    }
#pragma unroll
    for (int c = 0; c < NC; ++c) rec[(R::fold + c) * BD + i] = acc.get(c);
#pragma unroll
    for (int q = 0; q < NS; ++q) {
        rec[(R::last + q) * BD + i] = s_in ? s_in[q * per + (b * Ls + Ls - 1) * D + d] : 0.f;
        rec[(R::first + q) * BD + i] = s_in ? s_in[q * per + (b * Ls) * D + d] : 0.f;
    }
#pragma unroll
    for (int g = 0; g < G; ++g) rec[(R::gates + g) * BD + i] = gate_value(u + (b * Ls * G + g) * D + d);
}

// Every segment's record gathered, in segment order (R records of
// SegRecord::floats(B*D) floats each) -> for segment `me`: the state entering
// it at iterate k+1 (carry) and the iterate's state before it (lin, where its
// first step is linearised), both [NS][B][D]; and max |F(H^k)| over all
// segments into *res.  Page: "A sacada: método de Newton" -- the Newton
// linear recurrence composed segment by segment: segment j maps the state c
// entering it to fold_j(J (c - lin_j) + f(lin_j, u_j1)), with J = df/ds at
// lin_j, the previous segment's last iterate state (s0 for segment 0).
template <class Cell>
__global__ void __launch_bounds__(256) segment_combine_kernel(const float* __restrict__ recs, int n_seg, int me,
                                                              const float* __restrict__ s0, const float* __restrict__ a,
                                                              float* __restrict__ carry, float* __restrict__ lin_out,
                                                              unsigned* res, long long B, long long D)
{
    using Map = typename Cell::Map;
    using R = SegRecord<Cell>;
    constexpr int G = Cell::G, NS = Cell::NS, NC = Map::kFloats;
    const long long BD = B * D, RF = R::floats(BD);
    const long long i = (long long)blockIdx.x * blockDim.x + threadIdx.x;
    float rmax = 0.f;
    if (i < BD) {
        const long long d = i % D;
        float aa[G];
#pragma unroll
        for (int g = 0; g < G; ++g) aa[g] = a[g * D + d];
        float c[NS], lin[NS];
#pragma unroll
        for (int q = 0; q < NS; ++q) c[q] = lin[q] = s0 ? s0[q * BD + i] : 0.f;
        for (int j = 0; j < n_seg; ++j) {
            const float* rj = recs + j * RF;
            float uu[G], f[NS], x[NS], dl[NS], jx[NS];
#pragma unroll
            for (int g = 0; g < G; ++g) uu[g] = rj[(R::gates + g) * BD + i];
            Map m;
            Cell::eval(lin, uu, aa, f, m);
#pragma unroll
            for (int q = 0; q < NS; ++q) {
                rmax = max_nan(rmax, fabsf(rj[(R::first + q) * BD + i] - f[q]));
                if (j == me) {
                    carry[q * BD + i] = c[q];
                    lin_out[q * BD + i] = lin[q];
                }
                dl[q] = c[q] - lin[q];
            }
            apply_matrix(m, dl, jx);
#pragma unroll
            for (int q = 0; q < NS; ++q) x[q] = jx[q] + f[q];
            Map fold;
#pragma unroll
            for (int k = 0; k < NC; ++k) fold.set(k, rj[(R::fold + k) * BD + i]);
            apply(fold, x, c);
#pragma unroll
            for (int q = 0; q < NS; ++q) lin[q] = rj[(R::last + q) * BD + i];
        }
    }
    if (i == 0) {  // the segments' own maxima over their steps 1..Ls-1
        for (int j = 0; j < n_seg; ++j) rmax = max_nan(rmax, recs[j * RF + R::F * BD]);
    }
    block_max_into(rmax, res);
}

// The outcome of the last fused pass on a workspace as device floats:
// out[0] = the residual it published, out[1] = 1 if a device-side error was
// raised, else 0 (so that a host loop can reduce both across GPUs without
// reading the header first).
__global__ void result_outcome_kernel(const WsHeader* hdr, float* out)
{
    out[0] = hdr->result.residual;
    out[1] = hdr->error != 0 ? 1.f : 0.f;
}

}  // namespace pararnn
