// Diagonal GRU / LSTM cells, their Jacobians with respect to the previous
// state, and the affine-map monoid the Newton linear systems are scanned in.
//
// Page: "ParaRNN: Apple destrava treino paralelo de RNNs não-lineares e escala
// pra 7B parâmetros", section "Engenharia pra escalar": with diagonal matrices
// in the cell the Jacobian is diagonal (ParaGRU, one scalar per channel) or
// 2x2 block-diagonal over (c, h) (ParaLSTM).  Section "A sacada: método de
// Newton": each Newton iteration is a linear SSM whose state matrices are the
// Jacobians; section "O compromisso que SSMs fizeram": a linear recurrence is
// an associative combination, here of affine maps x -> M x + v.
#pragma once

#include "device_common.cuh"

namespace pararnn {

// ------------------------------------------------------- affine-map monoid
// An element maps the Newton correction at step l-1 to the one at step l:
// delta_l = M delta_{l-1} + v.  compose(later, earlier) applies `earlier`
// first.

template <int NS>
struct Aff;

template <>
struct Aff<1> {
    float m, v;
    static constexpr int kFloats = 2;
    __device__ __forceinline__ static Aff identity() { return {1.0f, 0.0f}; }
    __device__ __forceinline__ float get(int i) const { return i == 0 ? m : v; }
    __device__ __forceinline__ void set(int i, float x)
    {
        if (i == 0) m = x;
        else v = x;
    }
};

template <>
struct Aff<2> {
    float m00, m01, m10, m11, v0, v1;
    static constexpr int kFloats = 6;
    __device__ __forceinline__ static Aff identity() { return {1.0f, 0.0f, 0.0f, 1.0f, 0.0f, 0.0f}; }
    __device__ __forceinline__ float get(int i) const
    {
        switch (i) {
        case 0: return m00;
        case 1: return m01;
        case 2: return m10;
        case 3: return m11;
        case 4: return v0;
        default: return v1;
        }
    }
    __device__ __forceinline__ void set(int i, float x)
    {
        switch (i) {
        case 0: m00 = x; break;
        case 1: m01 = x; break;
        case 2: m10 = x; break;
        case 3: m11 = x; break;
        case 4: v0 = x; break;
        default: v1 = x; break;
        }
    }
};

__device__ __forceinline__ Aff<1> compose(const Aff<1>& later, const Aff<1>& earlier)
{
    return {later.m * earlier.m, fmaf(later.m, earlier.v, later.v)};
}

__device__ __forceinline__ Aff<2> compose(const Aff<2>& L, const Aff<2>& E)
{
    Aff<2> r;
    r.m00 = fmaf(L.m00, E.m00, L.m01 * E.m10);
    r.m01 = fmaf(L.m00, E.m01, L.m01 * E.m11);
    r.m10 = fmaf(L.m10, E.m00, L.m11 * E.m10);
    r.m11 = fmaf(L.m10, E.m01, L.m11 * E.m11);
    r.v0 = fmaf(L.m00, E.v0, fmaf(L.m01, E.v1, L.v0));
    r.v1 = fmaf(L.m10, E.v0, fmaf(L.m11, E.v1, L.v1));
    return r;
}

__device__ __forceinline__ void apply(const Aff<1>& a, const float* x, float* y)
{
    y[0] = fmaf(a.m, x[0], a.v);
}

__device__ __forceinline__ void apply(const Aff<2>& a, const float* x, float* y)
{
    const float x0 = x[0], x1 = x[1];
    y[0] = fmaf(a.m00, x0, fmaf(a.m01, x1, a.v0));
    y[1] = fmaf(a.m10, x0, fmaf(a.m11, x1, a.v1));
}

// Matrix part only: y = M x.
__device__ __forceinline__ void apply_matrix(const Aff<1>& a, const float* x, float* y) { y[0] = a.m * x[0]; }

__device__ __forceinline__ void apply_matrix(const Aff<2>& a, const float* x, float* y)
{
    y[0] = fmaf(a.m00, x[0], a.m01 * x[1]);
    y[1] = fmaf(a.m10, x[0], a.m11 * x[1]);
}

// Row-major NSxNS matrix times vector (matrix held as plain floats).
__device__ __forceinline__ void matrix_times(const float (&m)[1], const float* x, float* y) { y[0] = m[0] * x[0]; }

__device__ __forceinline__ void matrix_times(const float (&m)[4], const float* x, float* y)
{
    y[0] = fmaf(m[0], x[0], m[1] * x[1]);
    y[1] = fmaf(m[2], x[0], m[3] * x[1]);
}

// Set the offset part of a map from column j of off[NS][kV].
template <int V>
__device__ __forceinline__ void set_offset(Aff<1>& a, const float (&off)[1][V], int j) { a.v = off[0][j]; }

template <int V>
__device__ __forceinline__ void set_offset(Aff<2>& a, const float (&off)[2][V], int j)
{
    a.v0 = off[0][j];
    a.v1 = off[1][j];
}

// Set the offset part of a map from o[NS].
__device__ __forceinline__ void set_map_offset(Aff<1>& a, const float* o) { a.v = o[0]; }
__device__ __forceinline__ void set_map_offset(Aff<2>& a, const float* o)
{
    a.v0 = o[0];
    a.v1 = o[1];
}

// Transposed map for the reverse (adjoint) recurrence mu = J^T (g + mu'):
// matrix J^T, offset J^T g.
__device__ __forceinline__ Aff<1> transpose_map(const Aff<1>& J, const float* g)
{
    return {J.m, J.m * g[0]};
}

__device__ __forceinline__ Aff<2> transpose_map(const Aff<2>& J, const float* g)
{
    Aff<2> r;
    r.m00 = J.m00;
    r.m01 = J.m10;
    r.m10 = J.m01;
    r.m11 = J.m11;
    r.v0 = fmaf(J.m00, g[0], J.m10 * g[1]);
    r.v1 = fmaf(J.m01, g[0], J.m11 * g[1]);
    return r;
}

// ------------------------------------------------------------------- cells
// State vector s: GRU (h); LSTM (c, h).  eval() returns the cell output f and
// its Jacobian J = d f / d s (in the matrix part of an Aff; v left to caller).

struct GruPacked;
struct LstmPacked;

struct GruCell {
    static constexpr int G = 3;   // gates z, r, c
    static constexpr int NS = 1;  // state components
    using Map = Aff<1>;
    using Packed = GruPacked;

    __device__ __forceinline__ static void value(const float* s, const float* u, const float* a,
                                                 float* f)
    {
        const float h = s[0];
        float z, r;
        sigmoid2(fmaf(a[0], h, u[0]), fmaf(a[1], h, u[1]), z, r);
        const float c = tanh_fast(fmaf(a[2], r * h, u[2]));
        f[0] = fmaf(z, c - h, h);  // (1-z) h + z c
    }

    // d/dh[(1-z)h + z c] = (1-z) + z'(c-h) + z c',
    // z' = z(1-z) a_z, c' = (1-c^2) a_c (r + h r(1-r) a_r).
    __device__ __forceinline__ static void eval(const float* s, const float* u, const float* a,
                                                float* f, Map& J)
    {
        const float h = s[0];
        float z, r;
        sigmoid2(fmaf(a[0], h, u[0]), fmaf(a[1], h, u[1]), z, r);
        const float c = tanh_fast(fmaf(a[2], r * h, u[2]));
        const float cmh = c - h;
        f[0] = fmaf(z, cmh, h);
        const float zz = z - z * z;                                   // z(1-z)
        const float dr = fmaf(h * a[1], r - r * r, r);                // r + h r(1-r) a_r
        const float dc = (1.0f - c * c) * a[2] * dr;                  // dc/dh
        J.m = fmaf(z, dc, fmaf(zz * a[0], cmh, 1.0f - z));
    }

    // Reverse mode: given lam = dLoss/df, accumulate dLoss/du (du), the
    // contributions to dLoss/da (dacc += d pre / d a * du) and return
    // mu = dLoss/dh_prev = lam * df/dh.
    //   du_z = lam (c-h) z(1-z), du_c = lam z (1-c^2), du_r = du_c a_c h r(1-r),
    //   mu = lam (1-z) + a_z du_z + a_r du_r + a_c r du_c,
    //   d pre/d a = (h, h, r h).
    __device__ __forceinline__ static void vjp(const float* s, const float* u, const float* a, const float* lam,
                                               float* du, float* dacc, float* mu)
    {
        const float h = s[0];
        float z, r;
        sigmoid2(fmaf(a[0], h, u[0]), fmaf(a[1], h, u[1]), z, r);
        const float rh = r * h;
        const float c = tanh_fast(fmaf(a[2], rh, u[2]));
        const float l = lam[0];
        const float gz = l * (c - h) * (z - z * z);
        const float gc = l * z * (1.0f - c * c);
        const float gr = gc * a[2] * h * (r - r * r);
        du[0] = gz;
        du[1] = gr;
        du[2] = gc;
        dacc[0] = fmaf(h, gz, dacc[0]);
        dacc[1] = fmaf(h, gr, dacc[1]);
        dacc[2] = fmaf(rh, gc, dacc[2]);
        mu[0] = fmaf(l, 1.0f - z, fmaf(a[0], gz, fmaf(a[1], gr, a[2] * r * gc)));
    }
};

struct LstmCell {
    static constexpr int G = 4;   // gates i, f, o, g
    static constexpr int NS = 2;  // state (c, h)
    using Map = Aff<2>;
    using Packed = LstmPacked;

    __device__ __forceinline__ static void value(const float* s, const float* u, const float* a,
                                                 float* out)
    {
        const float c = s[0], h = s[1];
        float i, f, o, g;
        sigmoid2(fmaf(a[0], h, u[0]), fmaf(a[1], h, u[1]), i, f);
        sigmoid_tanh(fmaf(a[2], h, u[2]), fmaf(a[3], h, u[3]), o, g);
        const float cn = fmaf(f, c, i * g);
        out[0] = cn;
        out[1] = o * tanh_fast(cn);
    }

    // J = [[dc'/dc, dc'/dh], [dh'/dc, dh'/dh]] with
    // dc'/dh = c f(1-f) a_f + g i(1-i) a_i + i (1-g^2) a_g,
    // dh'/dc = o (1-t^2) f, dh'/dh = o(1-o) a_o t + o (1-t^2) dc'/dh, t = tanh(c').
    __device__ __forceinline__ static void eval(const float* s, const float* u, const float* a,
                                                float* out, Map& J)
    {
        const float c = s[0], h = s[1];
        float i, f, o, g;
        sigmoid2(fmaf(a[0], h, u[0]), fmaf(a[1], h, u[1]), i, f);
        sigmoid_tanh(fmaf(a[2], h, u[2]), fmaf(a[3], h, u[3]), o, g);
        const float cn = fmaf(f, c, i * g);
        const float t = tanh_fast(cn);
        out[0] = cn;
        out[1] = o * t;
        const float dcdh = fmaf(c * a[1], f - f * f, fmaf(g * a[0], i - i * i, i * (1.0f - g * g) * a[3]));
        const float ot = o * (1.0f - t * t);
        J.m00 = f;
        J.m01 = dcdh;
        J.m10 = ot * f;
        J.m11 = fmaf((o - o * o) * a[2], t, ot * dcdh);
    }

    // Reverse mode with lam = (dLoss/dc', dLoss/dh'):
    //   gamma = lam_c + lam_h o (1-t^2)           (total dLoss/dc')
    //   du_i = gamma g i(1-i), du_f = gamma c f(1-f), du_g = gamma i (1-g^2),
    //   du_o = lam_h t o(1-o); mu_c = gamma f, mu_h = sum_x a_x du_x;
    //   d pre/d a = h for every gate.
    __device__ __forceinline__ static void vjp(const float* s, const float* u, const float* a, const float* lam,
                                               float* du, float* dacc, float* mu)
    {
        const float c = s[0], h = s[1];
        float i, f, o, g;
        sigmoid2(fmaf(a[0], h, u[0]), fmaf(a[1], h, u[1]), i, f);
        sigmoid_tanh(fmaf(a[2], h, u[2]), fmaf(a[3], h, u[3]), o, g);
        const float t = tanh_fast(fmaf(f, c, i * g));
        const float gam = fmaf(lam[1] * o, 1.0f - t * t, lam[0]);
        const float gi = gam * g * (i - i * i);
        const float gf = gam * c * (f - f * f);
        const float go = lam[1] * t * (o - o * o);
        const float gg = gam * i * (1.0f - g * g);
        du[0] = gi;
        du[1] = gf;
        du[2] = go;
        du[3] = gg;
        dacc[0] = fmaf(h, gi, dacc[0]);
        dacc[1] = fmaf(h, gf, dacc[1]);
        dacc[2] = fmaf(h, go, dacc[2]);
        dacc[3] = fmaf(h, gg, dacc[3]);
        mu[0] = gam * f;
        mu[1] = fmaf(a[0], gi, fmaf(a[1], gf, fmaf(a[2], go, a[3] * gg)));
    }
};


// ------------------------------------------------- packed (two channels)
// Blackwell issues fp32 add / multiply / fma on register pairs as one
// instruction (__fadd2_rn, __fmul2_rn, __ffma2_rn).  The forms below evaluate
// two adjacent channels at once; the special functions stay per component.

__device__ __forceinline__ float2 bc2(float a) { return make_float2(a, a); }
__device__ __forceinline__ float2 neg2(float2 a) { return make_float2(-a.x, -a.y); }
__device__ __forceinline__ float2 fma2(float2 a, float2 b, float2 c) { return __ffma2_rn(a, b, c); }
__device__ __forceinline__ float2 mul2(float2 a, float2 b) { return __fmul2_rn(a, b); }
__device__ __forceinline__ float2 add2(float2 a, float2 b) { return __fadd2_rn(a, b); }
__device__ __forceinline__ float2 ex2_2(float2 t) { return make_float2(ex2_approx(t.x), ex2_approx(t.y)); }
__device__ __forceinline__ float2 rcp_2(float2 x) { return make_float2(rcp_approx(x.x), rcp_approx(x.y)); }
__device__ __forceinline__ float2 clamp_t2(float2 t)
{
    return make_float2(min_keep_nan(t.x, kMaxT), min_keep_nan(t.y, kMaxT));
}

// s(x), s(y) with one reciprocal per channel (see sigmoid2)
__device__ __forceinline__ void sigmoid2_2(float2 x, float2 y, float2& sx, float2& sy)
{
    const float2 one = bc2(1.0f);
    const float2 dx = add2(ex2_2(clamp_t2(mul2(bc2(-kLog2e), x))), one);
    const float2 dy = add2(ex2_2(clamp_t2(mul2(bc2(-kLog2e), y))), one);
    const float2 inv = rcp_2(mul2(dx, dy));
    sx = mul2(dy, inv);
    sy = mul2(dx, inv);
}

// s(x), tanh(y) with one reciprocal per channel (see sigmoid_tanh)
__device__ __forceinline__ void sigmoid_tanh_2(float2 x, float2 y, float2& sx, float2& ty)
{
    const float2 one = bc2(1.0f);
    const float2 dx = add2(ex2_2(clamp_t2(mul2(bc2(-kLog2e), x))), one);
    const float2 dy = add2(ex2_2(clamp_t2(mul2(bc2(2.0f * kLog2e), y))), one);
    const float2 inv = rcp_2(mul2(dx, dy));
    sx = mul2(dy, inv);
    ty = fma2(mul2(bc2(-2.0f), dx), inv, one);
}

__device__ __forceinline__ float2 tanh_2(float2 x)
{
    const float2 one = bc2(1.0f);
    return fma2(bc2(-2.0f), rcp_2(add2(ex2_2(mul2(bc2(2.0f * kLog2e), x)), one)), one);
}

// Packed affine maps: the same monoid, two channels per component.
template <int NS>
struct Aff2;

template <>
struct Aff2<1> {
    float2 m, v;
    __device__ __forceinline__ static Aff2 identity() { return {bc2(1.0f), bc2(0.0f)}; }
    __device__ __forceinline__ Aff<1> lane(int i) const
    {
        return i == 0 ? Aff<1>{m.x, v.x} : Aff<1>{m.y, v.y};
    }
    // entry i in the order of Aff<1>::get
    __device__ __forceinline__ void set(int i, float2 x)
    {
        if (i == 0) m = x;
        else v = x;
    }
};

template <>
struct Aff2<2> {
    float2 m00, m01, m10, m11, v0, v1;
    __device__ __forceinline__ static Aff2 identity()
    {
        return {bc2(1.0f), bc2(0.0f), bc2(0.0f), bc2(1.0f), bc2(0.0f), bc2(0.0f)};
    }
    __device__ __forceinline__ Aff<2> lane(int i) const
    {
        return i == 0 ? Aff<2>{m00.x, m01.x, m10.x, m11.x, v0.x, v1.x}
                      : Aff<2>{m00.y, m01.y, m10.y, m11.y, v0.y, v1.y};
    }
    // entry i in the order of Aff<2>::get
    __device__ __forceinline__ void set(int i, float2 x)
    {
        switch (i) {
        case 0: m00 = x; break;
        case 1: m01 = x; break;
        case 2: m10 = x; break;
        case 3: m11 = x; break;
        case 4: v0 = x; break;
        default: v1 = x; break;
        }
    }
};

__device__ __forceinline__ Aff2<1> compose(const Aff2<1>& L, const Aff2<1>& E)
{
    return {mul2(L.m, E.m), fma2(L.m, E.v, L.v)};
}

__device__ __forceinline__ Aff2<2> compose(const Aff2<2>& L, const Aff2<2>& E)
{
    Aff2<2> r;
    r.m00 = fma2(L.m00, E.m00, mul2(L.m01, E.m10));
    r.m01 = fma2(L.m00, E.m01, mul2(L.m01, E.m11));
    r.m10 = fma2(L.m10, E.m00, mul2(L.m11, E.m10));
    r.m11 = fma2(L.m10, E.m01, mul2(L.m11, E.m11));
    r.v0 = fma2(L.m00, E.v0, fma2(L.m01, E.v1, L.v0));
    r.v1 = fma2(L.m10, E.v0, fma2(L.m11, E.v1, L.v1));
    return r;
}

// y = M x (matrix part only) and y = M x + v
__device__ __forceinline__ void apply_matrix2(const Aff2<1>& a, const float2* x, float2* y) { y[0] = mul2(a.m, x[0]); }

__device__ __forceinline__ void apply_matrix2(const Aff2<2>& a, const float2* x, float2* y)
{
    y[0] = fma2(a.m00, x[0], mul2(a.m01, x[1]));
    y[1] = fma2(a.m10, x[0], mul2(a.m11, x[1]));
}

__device__ __forceinline__ void apply2(const Aff2<1>& a, const float2* x, float2* y) { y[0] = fma2(a.m, x[0], a.v); }

__device__ __forceinline__ void apply2(const Aff2<2>& a, const float2* x, float2* y)
{
    y[0] = fma2(a.m00, x[0], fma2(a.m01, x[1], a.v0));
    y[1] = fma2(a.m10, x[0], fma2(a.m11, x[1], a.v1));
}

__device__ __forceinline__ void set_offset2(Aff2<1>& a, const float2* off) { a.v = off[0]; }

// The Jacobian part of a packed map, kept between the two sweeps.
struct Jac2_1 {
    float2 m;
};
struct Jac2_2 {
    float2 m00, m01, m10, m11;
};
__device__ __forceinline__ Jac2_1 jacobian_of(const Aff2<1>& a) { return {a.m}; }
__device__ __forceinline__ Jac2_2 jacobian_of(const Aff2<2>& a) { return {a.m00, a.m01, a.m10, a.m11}; }
__device__ __forceinline__ void apply_matrix2(const Jac2_1& a, const float2* x, float2* y) { y[0] = mul2(a.m, x[0]); }
__device__ __forceinline__ void apply_matrix2(const Jac2_2& a, const float2* x, float2* y)
{
    y[0] = fma2(a.m00, x[0], mul2(a.m01, x[1]));
    y[1] = fma2(a.m10, x[0], mul2(a.m11, x[1]));
}

__device__ __forceinline__ void set_offset2(Aff2<2>& a, const float2* off)
{
    a.v0 = off[0];
    a.v1 = off[1];
}

// Jacobian pairs as plain arrays jm[entry][pair] (for shared-memory staging).
template <int NJ>
__device__ __forceinline__ void store_jacobian(const Jac2_1& a, float2 (&jm)[NJ][2], int jp) { jm[0][jp] = a.m; }

template <int NJ>
__device__ __forceinline__ void store_jacobian(const Jac2_2& a, float2 (&jm)[NJ][2], int jp)
{
    jm[0][jp] = a.m00;
    jm[1][jp] = a.m01;
    jm[2][jp] = a.m10;
    jm[3][jp] = a.m11;
}

__device__ __forceinline__ void matrix_times2(const float2 (&jm)[1][2], int jp, const float2* x, float2* y)
{
    y[0] = mul2(jm[0][jp], x[0]);
}

__device__ __forceinline__ void matrix_times2(const float2 (&jm)[4][2], int jp, const float2* x, float2* y)
{
    y[0] = fma2(jm[0][jp], x[0], mul2(jm[1][jp], x[1]));
    y[1] = fma2(jm[2][jp], x[0], mul2(jm[3][jp], x[1]));
}

// Packed diagonal GRU: f and J = df/dh for two channels.
struct GruPacked2;
struct LstmPacked2;

struct GruPacked {
    using Map2 = Aff2<1>;
    using Jac2 = Jac2_1;
    using Rows2 = GruPacked2;
    static constexpr int NJ = 1;  // Jacobian entries kept per channel pair

    __device__ __forceinline__ static void value(const float2* s, const float2* u, const float2* a, float2* f)
    {
        const float2 h = s[0];
        float2 z, r;
        sigmoid2_2(fma2(a[0], h, u[0]), fma2(a[1], h, u[1]), z, r);
        const float2 c = tanh_2(fma2(a[2], mul2(r, h), u[2]));
        f[0] = fma2(z, fma2(h, bc2(-1.0f), c), h);
    }

    __device__ __forceinline__ static void eval(const float2* s, const float2* u, const float2* a, float2* f,
                                                Map2& J)
    {
        const float2 h = s[0], one = bc2(1.0f);
        float2 z, r;
        sigmoid2_2(fma2(a[0], h, u[0]), fma2(a[1], h, u[1]), z, r);
        const float2 c = tanh_2(fma2(a[2], mul2(r, h), u[2]));
        const float2 cmh = fma2(h, bc2(-1.0f), c);
        f[0] = fma2(z, cmh, h);
        const float2 omz = fma2(z, bc2(-1.0f), one);                 // 1 - z
        const float2 dr = fma2(mul2(h, a[1]), fma2(neg2(r), r, r), r);  // r + h r(1-r) a_r
        const float2 dc = mul2(mul2(fma2(neg2(c), c, one), a[2]), dr);  // (1-c^2) a_c dr
        J.m = fma2(z, dc, fma2(mul2(mul2(z, omz), a[0]), cmh, omz));
    }
};

// Packed diagonal LSTM over (c, h): outputs and the 2x2 Jacobian for two channels.
struct LstmPacked {
    using Map2 = Aff2<2>;
    using Jac2 = Jac2_2;
    using Rows2 = LstmPacked2;

    __device__ __forceinline__ static void value(const float2* s, const float2* u, const float2* a, float2* out)
    {
        const float2 c = s[0], h = s[1];
        float2 i, f, o, g;
        sigmoid2_2(fma2(a[0], h, u[0]), fma2(a[1], h, u[1]), i, f);
        sigmoid_tanh_2(fma2(a[2], h, u[2]), fma2(a[3], h, u[3]), o, g);
        const float2 cn = fma2(f, c, mul2(i, g));
        out[0] = cn;
        out[1] = mul2(o, tanh_2(cn));
    }

    __device__ __forceinline__ static void eval(const float2* s, const float2* u, const float2* a, float2* out,
                                                Map2& J)
    {
        const float2 c = s[0], h = s[1], one = bc2(1.0f);
        float2 i, f, o, g;
        sigmoid2_2(fma2(a[0], h, u[0]), fma2(a[1], h, u[1]), i, f);
        sigmoid_tanh_2(fma2(a[2], h, u[2]), fma2(a[3], h, u[3]), o, g);
        const float2 cn = fma2(f, c, mul2(i, g));
        const float2 t = tanh_2(cn);
        out[0] = cn;
        out[1] = mul2(o, t);
        // dc'/dh = c f(1-f) a_f + g i(1-i) a_i + i (1-g^2) a_g
        const float2 dcdh = fma2(mul2(c, a[1]), fma2(neg2(f), f, f),
                                 fma2(mul2(g, a[0]), fma2(neg2(i), i, i), mul2(mul2(i, fma2(neg2(g), g, one)), a[3])));
        const float2 ot = mul2(o, fma2(neg2(t), t, one));  // o (1-t^2)
        J.m00 = f;
        J.m01 = dcdh;
        J.m10 = mul2(ot, f);
        J.m11 = fma2(mul2(fma2(neg2(o), o, o), a[2]), t, mul2(ot, dcdh));
    }
};

// ------------------------------------------- two timesteps, shared reciprocals
// Rows of a sweep are independent evaluations, so two of them can share the
// reciprocal of a product of denominators: with P = p_a p_b,
// 1/p_a = p_b / P and 1/p_b = p_a / P.  Exponents are clamped from above at
// kMaxT4 (four denominators) or kMaxT (two) so that P stays below 2^121; the
// clamp changes s(x) only where s(x) < 2^-30.
constexpr float kMaxT4 = 30.0f;

__device__ __forceinline__ float2 clamp_t2_at(float2 t, float hi)
{
    return make_float2(min_keep_nan(t.x, hi), min_keep_nan(t.y, hi));
}

__device__ __forceinline__ float2 logistic_den2(float2 x, float hi)
{
    return add2(ex2_2(clamp_t2_at(mul2(bc2(-kLog2e), x), hi)), bc2(1.0f));
}

__device__ __forceinline__ float2 tanh_den2(float2 x, float hi)
{
    return add2(ex2_2(clamp_t2_at(mul2(bc2(2.0f * kLog2e), x), hi)), bc2(1.0f));
}

// 1/(da db) -> (1/da, 1/db) with one reciprocal per lane
__device__ __forceinline__ void rcp_pair(float2 da, float2 db, float2& ia, float2& ib)
{
    const float2 inv = rcp_2(mul2(da, db));
    ia = mul2(db, inv);
    ib = mul2(da, inv);
}

// s(x_a), s(y_a), s(x_b), s(y_b) with one reciprocal per lane
__device__ __forceinline__ void sigmoid4_2(float2 xa, float2 ya, float2 xb, float2 yb, float2& sxa, float2& sya,
                                           float2& sxb, float2& syb)
{
    const float2 dxa = logistic_den2(xa, kMaxT4), dya = logistic_den2(ya, kMaxT4);
    const float2 dxb = logistic_den2(xb, kMaxT4), dyb = logistic_den2(yb, kMaxT4);
    const float2 pa = mul2(dxa, dya), pb = mul2(dxb, dyb);
    float2 ia, ib;
    rcp_pair(pa, pb, ia, ib);
    sxa = mul2(dya, ia);
    sya = mul2(dxa, ia);
    sxb = mul2(dyb, ib);
    syb = mul2(dxb, ib);
}

// s(x_a), tanh(y_a), s(x_b), tanh(y_b) with one reciprocal per lane
__device__ __forceinline__ void sigmoid_tanh4_2(float2 xa, float2 ya, float2 xb, float2 yb, float2& sxa,
                                                float2& tya, float2& sxb, float2& tyb)
{
    const float2 one = bc2(1.0f);
    const float2 dxa = logistic_den2(xa, kMaxT4), dya = tanh_den2(ya, kMaxT4);
    const float2 dxb = logistic_den2(xb, kMaxT4), dyb = tanh_den2(yb, kMaxT4);
    const float2 pa = mul2(dxa, dya), pb = mul2(dxb, dyb);
    float2 ia, ib;
    rcp_pair(pa, pb, ia, ib);
    sxa = mul2(dya, ia);
    tya = fma2(mul2(bc2(-2.0f), dxa), ia, one);
    sxb = mul2(dyb, ib);
    tyb = fma2(mul2(bc2(-2.0f), dxb), ib, one);
}

// tanh(x_a), tanh(x_b) with one reciprocal per lane
__device__ __forceinline__ void tanh2_2(float2 xa, float2 xb, float2& ta, float2& tb)
{
    const float2 one = bc2(1.0f);
    float2 ia, ib;
    rcp_pair(tanh_den2(xa, kMaxT), tanh_den2(xb, kMaxT), ia, ib);
    ta = fma2(bc2(-2.0f), ia, one);
    tb = fma2(bc2(-2.0f), ib, one);
}

// Two-row forms of the packed cells: rows a and b evaluated together.
struct GruPacked2 {
    // gates z, r, c at state h for rows a, b
    __device__ __forceinline__ static void gates(float2 ha, const float2* ua, float2 hb, const float2* ub,
                                                 const float2* a, float2& za, float2& ra, float2& ca, float2& zb,
                                                 float2& rb, float2& cb)
    {
        sigmoid4_2(fma2(a[0], ha, ua[0]), fma2(a[1], ha, ua[1]), fma2(a[0], hb, ub[0]), fma2(a[1], hb, ub[1]), za,
                   ra, zb, rb);
        tanh2_2(fma2(a[2], mul2(ra, ha), ua[2]), fma2(a[2], mul2(rb, hb), ub[2]), ca, cb);
    }

    __device__ __forceinline__ static float2 jac(float2 h, float2 z, float2 r, float2 c, const float2* a)
    {
        const float2 one = bc2(1.0f);
        const float2 cmh = fma2(h, bc2(-1.0f), c);
        const float2 omz = fma2(z, bc2(-1.0f), one);
        const float2 dr = fma2(mul2(h, a[1]), fma2(neg2(r), r, r), r);
        const float2 dc = mul2(mul2(fma2(neg2(c), c, one), a[2]), dr);
        return fma2(z, dc, fma2(mul2(mul2(z, omz), a[0]), cmh, omz));
    }

    __device__ __forceinline__ static void eval(const float2* sa, const float2* ua, const float2* sb,
                                                const float2* ub, const float2* a, float2* fa, float2* fb,
                                                Aff2<1>& Ja, Aff2<1>& Jb)
    {
        float2 za, ra, ca, zb, rb, cb;
        gates(sa[0], ua, sb[0], ub, a, za, ra, ca, zb, rb, cb);
        fa[0] = fma2(za, fma2(sa[0], bc2(-1.0f), ca), sa[0]);
        fb[0] = fma2(zb, fma2(sb[0], bc2(-1.0f), cb), sb[0]);
        Ja.m = jac(sa[0], za, ra, ca, a);
        Jb.m = jac(sb[0], zb, rb, cb, a);
    }

    __device__ __forceinline__ static void value(const float2* sa, const float2* ua, const float2* sb,
                                                 const float2* ub, const float2* a, float2* fa, float2* fb)
    {
        float2 za, ra, ca, zb, rb, cb;
        gates(sa[0], ua, sb[0], ub, a, za, ra, ca, zb, rb, cb);
        fa[0] = fma2(za, fma2(sa[0], bc2(-1.0f), ca), sa[0]);
        fb[0] = fma2(zb, fma2(sb[0], bc2(-1.0f), cb), sb[0]);
    }
};

struct LstmPacked2 {
    __device__ __forceinline__ static void gates(float2 ha, const float2* ua, float2 hb, const float2* ub,
                                                 const float2* a, float2 (&ga)[4], float2 (&gb)[4])
    {
        sigmoid4_2(fma2(a[0], ha, ua[0]), fma2(a[1], ha, ua[1]), fma2(a[0], hb, ub[0]), fma2(a[1], hb, ub[1]),
                   ga[0], ga[1], gb[0], gb[1]);
        sigmoid_tanh4_2(fma2(a[2], ha, ua[2]), fma2(a[3], ha, ua[3]), fma2(a[2], hb, ub[2]), fma2(a[3], hb, ub[3]),
                        ga[2], ga[3], gb[2], gb[3]);
    }

    __device__ __forceinline__ static void jac(float2 c, const float2 (&g)[4], float2 t, const float2* a, Aff2<2>& J)
    {
        const float2 one = bc2(1.0f);
        const float2 i = g[0], f = g[1], o = g[2], gg = g[3];
        const float2 dcdh = fma2(mul2(c, a[1]), fma2(neg2(f), f, f),
                                 fma2(mul2(gg, a[0]), fma2(neg2(i), i, i), mul2(mul2(i, fma2(neg2(gg), gg, one)), a[3])));
        const float2 ot = mul2(o, fma2(neg2(t), t, one));
        J.m00 = f;
        J.m01 = dcdh;
        J.m10 = mul2(ot, f);
        J.m11 = fma2(mul2(fma2(neg2(o), o, o), a[2]), t, mul2(ot, dcdh));
    }

    __device__ __forceinline__ static void eval(const float2* sa, const float2* ua, const float2* sb,
                                                const float2* ub, const float2* a, float2* fa, float2* fb,
                                                Aff2<2>& Ja, Aff2<2>& Jb)
    {
        float2 ga[4], gb[4], ta, tb;
        gates(sa[1], ua, sb[1], ub, a, ga, gb);
        const float2 cna = fma2(ga[1], sa[0], mul2(ga[0], ga[3]));
        const float2 cnb = fma2(gb[1], sb[0], mul2(gb[0], gb[3]));
        tanh2_2(cna, cnb, ta, tb);
        fa[0] = cna;
        fa[1] = mul2(ga[2], ta);
        fb[0] = cnb;
        fb[1] = mul2(gb[2], tb);
        jac(sa[0], ga, ta, a, Ja);
        jac(sb[0], gb, tb, a, Jb);
    }

    __device__ __forceinline__ static void value(const float2* sa, const float2* ua, const float2* sb,
                                                 const float2* ub, const float2* a, float2* fa, float2* fb)
    {
        float2 ga[4], gb[4], ta, tb;
        gates(sa[1], ua, sb[1], ub, a, ga, gb);
        const float2 cna = fma2(ga[1], sa[0], mul2(ga[0], ga[3]));
        const float2 cnb = fma2(gb[1], sb[0], mul2(gb[0], gb[3]));
        tanh2_2(cna, cnb, ta, tb);
        fa[0] = cna;
        fa[1] = mul2(ga[2], ta);
        fb[0] = cnb;
        fb[1] = mul2(gb[2], tb);
    }
};

}  // namespace pararnn
