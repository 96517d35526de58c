"""Example sources for pararnn_cell_create: the diagonal GRU and LSTM of the
built-in solves, written as user cells (one recurrence step, templated on the
number types of the state, T, and of the inputs, U; the library derives the
Jacobians and the adjoint's derivatives).  Gate order and equations
are those of the built-in cells: GRU (z, r, c) with the candidate on r*h,
LSTM (i, f, o, g) over the state (c, h)."""

GRU = r"""
template <class T, class U>
__device__ void recurrence_step(const T* s, const U* u, const U* a, T* out)
{
    const T h = s[0];
    const T z = sigmoid(u[0] + a[0] * h);
    const T r = sigmoid(u[1] + a[1] * h);
    const T c = tanh(u[2] + a[2] * (r * h));
    out[0] = (1.0f - z) * h + z * c;
}
"""

LSTM = r"""
template <class T, class U>
__device__ void recurrence_step(const T* s, const U* u, const U* a, T* out)
{
    const T c = s[0], h = s[1];
    const T i = sigmoid(u[0] + a[0] * h);
    const T f = sigmoid(u[1] + a[1] * h);
    const T o = sigmoid(u[2] + a[2] * h);
    const T g = tanh(u[3] + a[3] * h);
    const T cn = f * c + i * g;
    out[0] = cn;
    out[1] = o * tanh(cn);
}
"""
