"""CPU oracle for the ParaRNN Newton solve (diagonal GRU / LSTM).

TEST INFRASTRUCTURE ONLY.  Only ``tests/``, ``__graft_entry__.smoke()`` and
the CPU-baseline leg of ``bench.py`` may import this package.  The product
library (``nonlinear_rnn_newton_b200``) never imports, links or runs it, and
the two share no code: the oracle is plain C in fp64 (``oracle.c``), called
here through ctypes on numpy float64 arrays.

What each function follows is cited in ``oracle.c`` against the page
"ParaRNN: Apple destrava treino paralelo de RNNs não-lineares e escala pra
7B parâmetros" (sections "O compromisso que SSMs fizeram", "A sacada: método
de Newton", "Engenharia pra escalar").  Pins: torch.nn.GRU / nn.LSTM in
float64, torch autograd, dense solves of the Newton system, finite
differences (see ``tests/test_oracle.py``).
"""
import ctypes
import os

import numpy as np

from . import build as _build

_lib = None

OK = 0
NOT_CONVERGED = 1
NONFINITE = -5


def configure(lib):
    """Declare the C signatures on a loaded oracle library (also used by the
    mutation tests, which load deliberately broken copies of ``oracle.c``)."""
    d = ctypes.POINTER(ctypes.c_double)
    i64 = ctypes.c_int64
    lib.oracle_gru_cell.argtypes = [ctypes.c_double, d, d, d, d]
    lib.oracle_lstm_cell.argtypes = [ctypes.c_double, ctypes.c_double, d, d, d, d, d]
    lib.oracle_gru_seq.argtypes = [i64, i64, i64, d, d, d, d]
    lib.oracle_lstm_seq.argtypes = [i64, i64, i64, d, d, d, d, d, d]
    lib.oracle_gru_newton.argtypes = [i64, i64, i64, d, d, d, ctypes.c_double,
                                      ctypes.c_int, d, ctypes.POINTER(ctypes.c_int), d, d]
    lib.oracle_gru_newton.restype = ctypes.c_int
    lib.oracle_lstm_newton.argtypes = [i64, i64, i64, d, d, d, d, ctypes.c_double,
                                       ctypes.c_int, d, d, ctypes.POINTER(ctypes.c_int), d, d]
    lib.oracle_lstm_newton.restype = ctypes.c_int
    lib.oracle_gru_bptt.argtypes = [i64, i64, i64, d, d, d, d, d, d, d]
    lib.oracle_lstm_bptt.argtypes = [i64, i64, i64, d, d, d, d, d, d, d, d, d, d]
    lib.oracle_set_threads.argtypes = [ctypes.c_int]
    lib.oracle_max_threads.restype = ctypes.c_int
    return lib


def _load():
    global _lib
    if _lib is None:
        _lib = configure(ctypes.CDLL(_build.build()))
    return _lib


def _f64(x):
    if x is None:
        return None
    if hasattr(x, "detach"):  # torch tensor: exact widening to float64
        x = x.detach().to("cpu").double().numpy()
    return np.ascontiguousarray(x, dtype=np.float64)


def _p(x):
    if x is None:
        return None
    return x.ctypes.data_as(ctypes.POINTER(ctypes.c_double))


def set_threads(n: int) -> None:
    _load().oracle_set_threads(int(n))


def max_threads() -> int:
    return int(_load().oracle_max_threads())


def gru_cell(h: float, u3, a3):
    """One GRU step for one channel: returns (f, A = df/dh)."""
    u3, a3 = _f64(u3), _f64(a3)
    f = ctypes.c_double()
    A = ctypes.c_double()
    _load().oracle_gru_cell(float(h), _p(u3), _p(a3), ctypes.byref(f), ctypes.byref(A))
    return f.value, A.value


def lstm_cell(c: float, h: float, u4, a4):
    """One LSTM step for one channel: returns (c', h', J 2x2 row-major)."""
    u4, a4 = _f64(u4), _f64(a4)
    cn = ctypes.c_double()
    hn = ctypes.c_double()
    J = np.zeros(4)
    _load().oracle_lstm_cell(float(c), float(h), _p(u4), _p(a4),
                             ctypes.byref(cn), ctypes.byref(hn), _p(J))
    return cn.value, hn.value, J.reshape(2, 2)


def gru_seq(u, a, h0=None):
    """Sequential application; u [B,L,3,D], a [3,D], h0 [B,D] -> h [B,L,D]."""
    u, a, h0 = _f64(u), _f64(a), _f64(h0)
    B, L, G, D = u.shape
    assert G == 3 and a.shape == (3, D)
    h = np.empty((B, L, D))
    _load().oracle_gru_seq(B, L, D, _p(u), _p(a), _p(h0), _p(h))
    return h


def lstm_seq(u, a, c0=None, h0=None):
    """Sequential application; u [B,L,4,D] (i,f,o,g) -> (c, h) [B,L,D]."""
    u, a, c0, h0 = _f64(u), _f64(a), _f64(c0), _f64(h0)
    B, L, G, D = u.shape
    assert G == 4 and a.shape == (4, D)
    c = np.empty((B, L, D))
    h = np.empty((B, L, D))
    _load().oracle_lstm_seq(B, L, D, _p(u), _p(a), _p(c0), _p(h0), _p(c), _p(h))
    return c, h


def gru_newton(u, a, h0=None, tol=1e-6, max_iters=10):
    """Serial CPU Newton.  Returns (h, iters, residual, status, res_hist)."""
    u, a, h0 = _f64(u), _f64(a), _f64(h0)
    B, L, G, D = u.shape
    h = np.empty((B, L, D))
    it = ctypes.c_int()
    res = ctypes.c_double()
    hist = np.full(max_iters + 1, np.nan)
    st = _load().oracle_gru_newton(B, L, D, _p(u), _p(a), _p(h0), float(tol),
                                   int(max_iters), _p(h), ctypes.byref(it),
                                   ctypes.byref(res), _p(hist))
    if st == -2:
        raise MemoryError("oracle_gru_newton: allocation failed")
    return h, it.value, res.value, st, hist[: it.value + 1]


def lstm_newton(u, a, c0=None, h0=None, tol=1e-6, max_iters=10):
    """Serial CPU Newton over (c,h).  Returns (c, h, iters, residual, status, res_hist)."""
    u, a, c0, h0 = _f64(u), _f64(a), _f64(c0), _f64(h0)
    B, L, G, D = u.shape
    c = np.empty((B, L, D))
    h = np.empty((B, L, D))
    it = ctypes.c_int()
    res = ctypes.c_double()
    hist = np.full(max_iters + 1, np.nan)
    st = _load().oracle_lstm_newton(B, L, D, _p(u), _p(a), _p(c0), _p(h0), float(tol),
                                    int(max_iters), _p(c), _p(h), ctypes.byref(it),
                                    ctypes.byref(res), _p(hist))
    if st == -2:
        raise MemoryError("oracle_lstm_newton: allocation failed")
    return c, h, it.value, res.value, st, hist[: it.value + 1]


def gru_bptt(u, a, h0, gh):
    """BPTT of Loss = sum(gh*h).  Returns (du [B,L,3,D], da [3,D], dh0 [B,D])."""
    u, a, h0, gh = _f64(u), _f64(a), _f64(h0), _f64(gh)
    B, L, G, D = u.shape
    du = np.empty((B, L, 3, D))
    da = np.empty((3, D))
    dh0 = np.empty((B, D))
    _load().oracle_gru_bptt(B, L, D, _p(u), _p(a), _p(h0), _p(gh), _p(du), _p(da), _p(dh0))
    return du, da, dh0


def lstm_bptt(u, a, c0, h0, gh, gc=None):
    """BPTT of Loss = sum(gh*h) + sum(gc*c).  Returns (du, da, dc0, dh0)."""
    u, a, c0, h0, gh, gc = _f64(u), _f64(a), _f64(c0), _f64(h0), _f64(gh), _f64(gc)
    B, L, G, D = u.shape
    du = np.empty((B, L, 4, D))
    da = np.empty((4, D))
    dc0 = np.empty((B, D))
    dh0 = np.empty((B, D))
    _load().oracle_lstm_bptt(B, L, D, _p(u), _p(a), _p(c0), _p(h0), _p(gh), _p(gc),
                             _p(du), _p(da), _p(dc0), _p(dh0))
    return du, da, dc0, dh0


def project(x, w, bias=None):
    """Input projection of the gate pre-activations in float64:
    u[b, l, g, d] = sum_k x[b, l, k] w[g, d, k] + bias[g, d]
    (x [B, L, Din], w [G, D, Din], bias [G, D] or None).  Page "ParaRNN: Apple
    destrava treino paralelo de RNNs não-lineares e escala pra 7B parâmetros",
    section "O compromisso que SSMs fizeram": the input enters the recurrence
    through a projection (B_l x_l).  A library contraction is the step."""
    x, w = _f64(x), _f64(w)
    u = np.einsum("blk,gdk->blgd", x, w)
    if bias is not None:
        u = u + _f64(bias)[None, None]
    return u


def library_path() -> str:
    return os.path.abspath(_build.LIB)
