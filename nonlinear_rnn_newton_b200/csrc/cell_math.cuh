// Arithmetic for user-written recurrence steps: forward-mode dual numbers and
// the elementary functions, each for float and for duals.
//
// Page: "ParaRNN: Apple destrava treino paralelo de RNNs não-lineares e escala
// pra 7B parâmetros" -- "Como usar": the user writes only the recurrence step
// and the framework assembles the Jacobians.  A step written once as a
// template over its number type T runs with T = float for the cell's value
// and with T = Dual<K> (value plus K tangents) for the value together with
// its derivatives along K input directions.  Seeding the K = NS state
// components with unit tangents gives the step's NS x NS Jacobian block in
// one evaluation.
//
// Derivative rules used (d = tangent): (a b)' = a' b + a b';
// (a / b)' = (a' b - a b') / b^2; exp' = exp; log' = 1/x; tanh' = 1 - tanh^2;
// sigmoid' = s (1 - s); sqrt' = 1 / (2 sqrt); sin' = cos; cos' = -sin.
// The float versions call the CUDA math library's single-precision
// functions (expf, logf, tanhf, sqrtf, sinf, cosf).  Compiled with
// PARARNN_USER_FAST_MATH (defined for the PARARNN_CELL_FAST_MATH flag) they
// use the hardware approximations instead (__expf, __logf, __sinf, __cosf,
// __fdividef; tanh(x) = 1 - 2/(e^{2x}+1)), as the built-in cells do, and the
// duals' divisions use __fdividef.
#pragma once

namespace pararnn_user {

#ifdef PARARNN_USER_FAST_MATH
__device__ __forceinline__ float div_(float a, float b) { return __fdividef(a, b); }
#else
__device__ __forceinline__ float div_(float a, float b) { return a / b; }
#endif

template <int K>
struct Dual {
    float v;     // value
    float d[K];  // tangents
    __device__ Dual() : v(0.f)
    {
#pragma unroll
        for (int i = 0; i < K; ++i) d[i] = 0.f;
    }
    __device__ Dual(float x) : v(x)  // a constant: zero tangents
    {
#pragma unroll
        for (int i = 0; i < K; ++i) d[i] = 0.f;
    }
};

// the value and tangents of f(x) given f(x.v) and f'(x.v)
template <int K>
__device__ __forceinline__ Dual<K> chain(const Dual<K>& x, float f, float df)
{
    Dual<K> r(f);
#pragma unroll
    for (int i = 0; i < K; ++i) r.d[i] = df * x.d[i];
    return r;
}

template <int K>
__device__ __forceinline__ Dual<K> operator+(const Dual<K>& a, const Dual<K>& b)
{
    Dual<K> r(a.v + b.v);
#pragma unroll
    for (int i = 0; i < K; ++i) r.d[i] = a.d[i] + b.d[i];
    return r;
}
template <int K>
__device__ __forceinline__ Dual<K> operator+(const Dual<K>& a, float b)
{
    Dual<K> r = a;
    r.v += b;
    return r;
}
template <int K>
__device__ __forceinline__ Dual<K> operator+(float a, const Dual<K>& b)
{
    return b + a;
}

template <int K>
__device__ __forceinline__ Dual<K> operator-(const Dual<K>& a)
{
    Dual<K> r(-a.v);
#pragma unroll
    for (int i = 0; i < K; ++i) r.d[i] = -a.d[i];
    return r;
}
template <int K>
__device__ __forceinline__ Dual<K> operator-(const Dual<K>& a, const Dual<K>& b)
{
    Dual<K> r(a.v - b.v);
#pragma unroll
    for (int i = 0; i < K; ++i) r.d[i] = a.d[i] - b.d[i];
    return r;
}
template <int K>
__device__ __forceinline__ Dual<K> operator-(const Dual<K>& a, float b)
{
    Dual<K> r = a;
    r.v -= b;
    return r;
}
template <int K>
__device__ __forceinline__ Dual<K> operator-(float a, const Dual<K>& b)
{
    return -b + a;
}

template <int K>
__device__ __forceinline__ Dual<K> operator*(const Dual<K>& a, const Dual<K>& b)
{
    Dual<K> r(a.v * b.v);
#pragma unroll
    for (int i = 0; i < K; ++i) r.d[i] = fmaf(a.d[i], b.v, a.v * b.d[i]);
    return r;
}
template <int K>
__device__ __forceinline__ Dual<K> operator*(const Dual<K>& a, float b)
{
    Dual<K> r(a.v * b);
#pragma unroll
    for (int i = 0; i < K; ++i) r.d[i] = a.d[i] * b;
    return r;
}
template <int K>
__device__ __forceinline__ Dual<K> operator*(float a, const Dual<K>& b)
{
    return b * a;
}

template <int K>
__device__ __forceinline__ Dual<K> operator/(const Dual<K>& a, const Dual<K>& b)
{
    const float ib = div_(1.0f, b.v);
    const float q = a.v * ib;
    Dual<K> r(q);
#pragma unroll
    for (int i = 0; i < K; ++i) r.d[i] = (a.d[i] - q * b.d[i]) * ib;
    return r;
}
template <int K>
__device__ __forceinline__ Dual<K> operator/(const Dual<K>& a, float b)
{
    const float ib = div_(1.0f, b);
    Dual<K> r(a.v * ib);
#pragma unroll
    for (int i = 0; i < K; ++i) r.d[i] = a.d[i] * ib;
    return r;
}
template <int K>
__device__ __forceinline__ Dual<K> operator/(float a, const Dual<K>& b)
{
    const float ib = div_(1.0f, b.v);
    const float q = a * ib;
    return chain(b, q, -q * ib);
}

template <int K, class X>
__device__ __forceinline__ Dual<K>& operator+=(Dual<K>& a, const X& b)
{
    return a = a + b;
}
template <int K, class X>
__device__ __forceinline__ Dual<K>& operator-=(Dual<K>& a, const X& b)
{
    return a = a - b;
}
template <int K, class X>
__device__ __forceinline__ Dual<K>& operator*=(Dual<K>& a, const X& b)
{
    return a = a * b;
}
template <int K, class X>
__device__ __forceinline__ Dual<K>& operator/=(Dual<K>& a, const X& b)
{
    return a = a / b;
}

// ------------------------------------------------------ elementary functions

#ifdef PARARNN_USER_FAST_MATH
__device__ __forceinline__ float exp(float x) { return __expf(x); }
__device__ __forceinline__ float log(float x) { return __logf(x); }
__device__ __forceinline__ float tanh(float x) { return 1.0f - __fdividef(2.0f, __expf(2.0f * x) + 1.0f); }
__device__ __forceinline__ float sin(float x) { return __sinf(x); }
__device__ __forceinline__ float cos(float x) { return __cosf(x); }
__device__ __forceinline__ float sigmoid(float x) { return __fdividef(1.0f, 1.0f + __expf(-x)); }
#else
__device__ __forceinline__ float exp(float x) { return expf(x); }
__device__ __forceinline__ float log(float x) { return logf(x); }
__device__ __forceinline__ float tanh(float x) { return tanhf(x); }
__device__ __forceinline__ float sin(float x) { return sinf(x); }
__device__ __forceinline__ float cos(float x) { return cosf(x); }
__device__ __forceinline__ float sigmoid(float x) { return 1.0f / (1.0f + expf(-x)); }
#endif
__device__ __forceinline__ float sqrt(float x) { return sqrtf(x); }

template <int K>
__device__ __forceinline__ Dual<K> exp(const Dual<K>& x)
{
    const float e = exp(x.v);
    return chain(x, e, e);
}
template <int K>
__device__ __forceinline__ Dual<K> log(const Dual<K>& x)
{
    return chain(x, log(x.v), div_(1.0f, x.v));
}
template <int K>
__device__ __forceinline__ Dual<K> tanh(const Dual<K>& x)
{
    const float t = tanh(x.v);
    return chain(x, t, fmaf(-t, t, 1.0f));
}
template <int K>
__device__ __forceinline__ Dual<K> sigmoid(const Dual<K>& x)
{
    const float s = sigmoid(x.v);
    return chain(x, s, s - s * s);
}
template <int K>
__device__ __forceinline__ Dual<K> sqrt(const Dual<K>& x)
{
    const float r = sqrtf(x.v);
    return chain(x, r, div_(0.5f, r));
}
template <int K>
__device__ __forceinline__ Dual<K> sin(const Dual<K>& x)
{
    return chain(x, sin(x.v), cos(x.v));
}
template <int K>
__device__ __forceinline__ Dual<K> cos(const Dual<K>& x)
{
    return chain(x, cos(x.v), -sin(x.v));
}

// the value part (for branches on a state's value)
__device__ __forceinline__ float value_of(float x) { return x; }
template <int K>
__device__ __forceinline__ float value_of(const Dual<K>& x)
{
    return x.v;
}

}  // namespace pararnn_user
