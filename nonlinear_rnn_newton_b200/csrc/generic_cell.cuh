// A user-written recurrence step as a cell of the fused Newton solve.
//
// Page: "ParaRNN: Apple destrava treino paralelo de RNNs não-lineares e escala
// pra 7B parâmetros" -- "Como usar": the user supplies only the recurrence
// step; Newton, the Jacobian assembly and the parallel reduction are the
// framework's.  Of the three tiers named there this is the fully fused one
// (a single kernel built from a CUDA version of the step), for steps whose
// Jacobian is diagonal (NS = 1) or one 2x2 block per channel (NS = 2).
//
// Included after the user's source, which defines, inside namespace
// pararnn_user,
//     template <class T, class U>
//     __device__ void recurrence_step(const T* s, const U* u, const U* a,
//                                     T* out);
// (s: the NS state components of one channel at step l-1; u: its G gate
// pre-activations at step l; a: its G recurrence weights; out: the NS
// components at step l; T is the number type of the state, U that of the
// inputs).  Three instantiations serve the solve and the adjoint:
//   * value: T = U = float;
//   * Jacobian block J[q][r] = d out_q / d s_r: T = Dual<NS>, U = float,
//     the state components seeded with unit tangents;
//   * vector-Jacobian products for the adjoint: T = U = Dual<NS + 2G>, with
//     the state, the gates and the weights seeded, so that one evaluation
//     gives d out / d (s, u, a) and lam^T times it.
// The packed two-channel, two-row forms the solve kernel calls evaluate the
// four (row, channel) pairs one after another.
#pragma once

#include "cell_math.cuh"
#include "cells.cuh"

namespace pararnn {

template <int NS>
struct GenericJac2;
template <>
struct GenericJac2<1> {
    using type = Jac2_1;
};
template <>
struct GenericJac2<2> {
    using type = Jac2_2;
};

// lane i of a packed map's matrix part from a scalar block
__device__ __forceinline__ void set_matrix_lane(Aff2<1>& m, int i, const float (&J)[1][1])
{
    if (i == 0) m.m.x = J[0][0];
    else m.m.y = J[0][0];
}

__device__ __forceinline__ void set_matrix_lane(Aff2<2>& m, int i, const float (&J)[2][2])
{
    if (i == 0) {
        m.m00.x = J[0][0];
        m.m01.x = J[0][1];
        m.m10.x = J[1][0];
        m.m11.x = J[1][1];
    } else {
        m.m00.y = J[0][0];
        m.m01.y = J[0][1];
        m.m10.y = J[1][0];
        m.m11.y = J[1][1];
    }
}

__device__ __forceinline__ void set_matrix(Aff<1>& m, const float (&J)[1][1]) { m.m = J[0][0]; }

__device__ __forceinline__ void set_matrix(Aff<2>& m, const float (&J)[2][2])
{
    m.m00 = J[0][0];
    m.m01 = J[0][1];
    m.m10 = J[1][0];
    m.m11 = J[1][1];
}

__device__ __forceinline__ float lane_of(float2 x, int i) { return i == 0 ? x.x : x.y; }
__device__ __forceinline__ void set_lane(float2& x, int i, float v)
{
    if (i == 0) x.x = v;
    else x.y = v;
}

template <int G_, int NS_>
struct GenericCell {
    static constexpr int G = G_;
    static constexpr int NS = NS_;
    using Map = Aff<NS>;
    struct Packed;

    __device__ __forceinline__ static void value(const float* s, const float* u, const float* a, float* f)
    {
        pararnn_user::recurrence_step<float, float>(s, u, a, f);
    }

    // f = step(s) and J[q][r] = d f_q / d s_r
    __device__ __forceinline__ static void value_jac(const float* s, const float* u, const float* a, float* f,
                                                     float (&J)[NS][NS])
    {
        pararnn_user::Dual<NS> x[NS], y[NS];
#pragma unroll
        for (int q = 0; q < NS; ++q) {
            x[q] = pararnn_user::Dual<NS>(s[q]);
            x[q].d[q] = 1.0f;
        }
        pararnn_user::recurrence_step<pararnn_user::Dual<NS>, float>(x, u, a, y);
#pragma unroll
        for (int q = 0; q < NS; ++q) {
            f[q] = y[q].v;
#pragma unroll
            for (int r = 0; r < NS; ++r) J[q][r] = y[q].d[r];
        }
    }

    // f and its Jacobian in the matrix part of an affine map (the adjoint's form)
    __device__ __forceinline__ static void eval(const float* s, const float* u, const float* a, float* f, Map& J)
    {
        float m[NS][NS];
        value_jac(s, u, a, f, m);
        set_matrix(J, m);
    }

    // Reverse mode at one step, lam = dLoss/d out: du_g = lam . d out/d u_g,
    // dacc_g += lam . d out/d a_g, mu_r = lam . d out/d s_r.
    __device__ __forceinline__ static void vjp(const float* s, const float* u, const float* a, const float* lam,
                                               float* du, float* dacc, float* mu)
    {
        constexpr int K = NS + 2 * G;
        using D = pararnn_user::Dual<K>;
        D x[NS], uu[G], aa[G], y[NS];
#pragma unroll
        for (int q = 0; q < NS; ++q) {
            x[q] = D(s[q]);
            x[q].d[q] = 1.0f;
        }
#pragma unroll
        for (int g = 0; g < G; ++g) {
            uu[g] = D(u[g]);
            uu[g].d[NS + g] = 1.0f;
            aa[g] = D(a[g]);
            aa[g].d[NS + G + g] = 1.0f;
        }
        pararnn_user::recurrence_step<D, D>(x, uu, aa, y);
        float t[K];
#pragma unroll
        for (int k = 0; k < K; ++k) {
            t[k] = 0.0f;
#pragma unroll
            for (int q = 0; q < NS; ++q) t[k] = fmaf(lam[q], y[q].d[k], t[k]);
        }
#pragma unroll
        for (int q = 0; q < NS; ++q) mu[q] = t[q];
#pragma unroll
        for (int g = 0; g < G; ++g) {
            du[g] = t[NS + g];
            dacc[g] += t[NS + G + g];
        }
    }

    struct Rows2 {
        // one (row, channel) pair of the packed inputs
        __device__ __forceinline__ static void unpack(const float2* s, const float2* u, const float2* a, int i,
                                                      float* ss, float* uu, float* aa)
        {
#pragma unroll
            for (int q = 0; q < NS; ++q) ss[q] = lane_of(s[q], i);
#pragma unroll
            for (int g = 0; g < G; ++g) {
                uu[g] = lane_of(u[g], i);
                aa[g] = lane_of(a[g], i);
            }
        }

        __device__ __forceinline__ static void eval(const float2* sa, const float2* ua, const float2* sb,
                                                    const float2* ub, const float2* a, float2* fa, float2* fb,
                                                    Aff2<NS>& Ja, Aff2<NS>& Jb)
        {
#pragma unroll
            for (int i = 0; i < 2; ++i) {
                float ss[NS], uu[G], aa[G], f[NS], J[NS][NS];
                unpack(sa, ua, a, i, ss, uu, aa);
                value_jac(ss, uu, aa, f, J);
#pragma unroll
                for (int q = 0; q < NS; ++q) set_lane(fa[q], i, f[q]);
                set_matrix_lane(Ja, i, J);
                unpack(sb, ub, a, i, ss, uu, aa);
                value_jac(ss, uu, aa, f, J);
#pragma unroll
                for (int q = 0; q < NS; ++q) set_lane(fb[q], i, f[q]);
                set_matrix_lane(Jb, i, J);
            }
        }

        __device__ __forceinline__ static void value(const float2* sa, const float2* ua, const float2* sb,
                                                     const float2* ub, const float2* a, float2* fa, float2* fb)
        {
#pragma unroll
            for (int i = 0; i < 2; ++i) {
                float ss[NS], uu[G], aa[G], f[NS];
                unpack(sa, ua, a, i, ss, uu, aa);
                GenericCell::value(ss, uu, aa, f);
#pragma unroll
                for (int q = 0; q < NS; ++q) set_lane(fa[q], i, f[q]);
                unpack(sb, ub, a, i, ss, uu, aa);
                GenericCell::value(ss, uu, aa, f);
#pragma unroll
                for (int q = 0; q < NS; ++q) set_lane(fb[q], i, f[q]);
            }
        }
    };

    struct Packed {
        using Map2 = Aff2<NS>;
        using Jac2 = typename GenericJac2<NS>::type;
        using Rows2 = typename GenericCell::Rows2;
    };
};

// A two-component user cell in accurate math leaves residuals out in the
// passes that continue (its residual evaluation, with the library's accurate
// functions, is a large share of a pass); with the fast functions it keeps
// the full evaluation, as the built-in ParaLSTM does.
template <int G_>
struct PartialResiduals<GenericCell<G_, 2>> {
#ifdef PARARNN_USER_FAST_MATH
    static constexpr bool value = false;
#else
    static constexpr bool value = true;
#endif
};

}  // namespace pararnn
