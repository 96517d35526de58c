"""User-written cells for the tests of the runtime-compiled solve: each one is
the CUDA source handed to pararnn_cell_create and, for the oracle, the same
step and its Jacobian written in float64 (vectorised over channels:
s [NS, B, D], u [G, B, D], a [G, D]).  The steps take the array module as
`xp` (numpy, or torch for the autograd gradients of the oracle's BPTT)."""
from dataclasses import dataclass
from typing import Callable

import numpy as np

from nonlinear_rnn_newton_b200 import example_cells


def sig(x, xp=np):
    return 1.0 / (1.0 + xp.exp(-x))


@dataclass
class UserCell:
    name: str
    G: int
    NS: int
    source: str
    step: Callable
    jac: Callable


# ----------------------------------------------------------------- GRU

GRU_SRC = example_cells.GRU


def gru_step(s, u, a, xp=np):
    h = s[0]
    z = sig(u[0] + a[0] * h, xp)
    r = sig(u[1] + a[1] * h, xp)
    c = xp.tanh(u[2] + a[2] * r * h)
    return ((1 - z) * h + z * c)[None]


def gru_jac(s, u, a):
    h = s[0]
    z = sig(u[0] + a[0] * h)
    r = sig(u[1] + a[1] * h)
    c = np.tanh(u[2] + a[2] * r * h)
    dr = r + h * r * (1 - r) * a[1]
    return ((1 - z) + (c - h) * z * (1 - z) * a[0] + z * (1 - c * c) * a[2] * dr)[None, None]


# ---------------------------------------------------------------- LSTM

LSTM_SRC = example_cells.LSTM


def lstm_step(s, u, a, xp=np):
    c, h = s[0], s[1]
    i, f, o = sig(u[0] + a[0] * h, xp), sig(u[1] + a[1] * h, xp), sig(u[2] + a[2] * h, xp)
    g = xp.tanh(u[3] + a[3] * h)
    cn = f * c + i * g
    return xp.stack([cn, o * xp.tanh(cn)])


def lstm_jac(s, u, a):
    c, h = s
    i, f, o = sig(u[0] + a[0] * h), sig(u[1] + a[1] * h), sig(u[2] + a[2] * h)
    g = np.tanh(u[3] + a[3] * h)
    cn = f * c + i * g
    t = np.tanh(cn)
    dcdh = c * f * (1 - f) * a[1] + g * i * (1 - i) * a[0] + i * (1 - g * g) * a[3]
    J = np.empty((2, 2) + c.shape)
    J[0, 0], J[0, 1] = f, dcdh
    J[1, 0] = o * (1 - t * t) * f
    J[1, 1] = o * (1 - o) * a[2] * t + o * (1 - t * t) * dcdh
    return J


# -------------------------------------------------- diagonal Elman (tanh)

ELMAN_SRC = r"""
template <class T, class U>
__device__ void recurrence_step(const T* s, const U* u, const U* a, T* out)
{
    out[0] = tanh(u[0] + a[0] * s[0]);
}
"""


def elman_step(s, u, a, xp=np):
    return xp.tanh(u[0] + a[0] * s[0])[None]


def elman_jac(s, u, a):
    t = np.tanh(u[0] + a[0] * s[0])
    return ((1 - t * t) * a[0])[None, None]


# ------------------------------- two coupled components, every rule used

MIXED_SRC = r"""
// x, y coupled both ways; uses +, -, *, /, sin, cos, sqrt, exp, log,
// sigmoid and tanh on duals
template <class T, class U>
__device__ void recurrence_step(const T* s, const U* u, const U* a, T* out)
{
    const T x = s[0], y = s[1];
    const T p = u[0] + a[0] * y;
    const T q = u[1] + a[1] * x;
    out[0] = 0.5f * sin(p) + 0.5f * x / sqrt(1.0f + x * x);
    const T lg = log(1.0f + exp(-(q * q)));
    out[1] = sigmoid(q) * tanh(y) + 0.2f * lg * (1.0f / (1.25f + cos(y)));
}
"""


def mixed_step(s, u, a, xp=np):
    x, y = s[0], s[1]
    p = u[0] + a[0] * y
    q = u[1] + a[1] * x
    o0 = 0.5 * xp.sin(p) + 0.5 * x / xp.sqrt(1 + x * x)
    o1 = sig(q, xp) * xp.tanh(y) + 0.2 * xp.log(1 + xp.exp(-q * q)) / (1.25 + xp.cos(y))
    return xp.stack([o0, o1])


def mixed_jac(s, u, a):
    x, y = s
    p = u[0] + a[0] * y
    q = u[1] + a[1] * x
    S, T, cy = sig(q), np.tanh(y), 1.25 + np.cos(y)
    e = np.exp(-q * q)
    lg = np.log(1 + e)
    J = np.empty((2, 2) + x.shape)
    J[0, 0] = 0.5 * (1 + x * x) ** -1.5
    J[0, 1] = 0.5 * np.cos(p) * a[0]
    J[1, 0] = a[1] * (S * (1 - S) * T + 0.2 * (-2 * q * e / (1 + e)) / cy)
    J[1, 1] = S * (1 - T * T) + 0.2 * lg * np.sin(y) / (cy * cy)
    return J


CELLS = {
    "gru": UserCell("gru", 3, 1, GRU_SRC, gru_step, gru_jac),
    "lstm": UserCell("lstm", 4, 2, LSTM_SRC, lstm_step, lstm_jac),
    "elman": UserCell("elman", 1, 1, ELMAN_SRC, elman_step, elman_jac),
    "mixed": UserCell("mixed", 2, 2, MIXED_SRC, mixed_step, mixed_jac),
}
