"""Thin Python binding of libpararnn.so (ctypes).

Argument marshalling only: every step of the solve, adjoint and baselines
runs in the library's CUDA kernels.  PyTorch supplies device memory, streams
and host<->device copies.  There is no CPU fallback: if the library is
missing, importing this module raises ImportError.

Names follow the C ABI in include/pararnn.h.
"""
import ctypes
import os

import torch

_HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_HERE, "libpararnn.so")

OK = 0
NOT_CONVERGED = 1
ERR_INVALID_ARG = -1
ERR_WORKSPACE = -2
ERR_CUDA = -3
ERR_TIMEOUT = -4
ERR_NONFINITE = -5
ERR_UNSUPPORTED = -6

F32 = 0
BF16 = 1


class PararnnError(RuntimeError):
    def __init__(self, status, msg):
        super().__init__(f"pararnn status {status}: {msg}")
        self.status = status


class Result(ctypes.Structure):
    _fields_ = [("status", ctypes.c_int32), ("iters", ctypes.c_int32),
                ("residual", ctypes.c_float), ("residual0", ctypes.c_float)]


_vp = ctypes.c_void_p
_i64 = ctypes.c_int64
_st = ctypes.c_int

# name -> (restype, argtypes)
SIGNATURES = {
    "pararnn_gru_workspace_size": (ctypes.c_size_t, [_i64, _i64, _i64]),
    "pararnn_lstm_workspace_size": (ctypes.c_size_t, [_i64, _i64, _i64]),
    "pararnn_gru_adjoint_workspace_size": (ctypes.c_size_t, [_i64, _i64, _i64]),
    "pararnn_lstm_adjoint_workspace_size": (ctypes.c_size_t, [_i64, _i64, _i64]),
    "pararnn_linear_scan_workspace_size": (ctypes.c_size_t, [_i64, _i64, _i64]),
    "pararnn_gru_solve": (_st, [_vp, _st, _vp, _vp, _vp, _i64, _i64, _i64, ctypes.c_float, ctypes.c_int,
                                _vp, ctypes.c_size_t, _vp, ctypes.POINTER(ctypes.c_int),
                                ctypes.POINTER(ctypes.c_float)]),
    "pararnn_gru_solve_async": (_st, [_vp, _st, _vp, _vp, _vp, _i64, _i64, _i64, ctypes.c_float,
                                      ctypes.c_int, _vp, ctypes.c_size_t, _vp]),
    "pararnn_gru_solve_noalloc": (_st, [_vp, _st, _vp, _vp, _vp, _i64, _i64, _i64, ctypes.c_float,
                                        ctypes.c_int, _vp, ctypes.POINTER(ctypes.c_int),
                                        ctypes.POINTER(ctypes.c_float)]),
    "pararnn_gru_solve_noalloc_max_scratch": (ctypes.c_size_t, []),
    "pararnn_lstm_solve": (_st, [_vp, _st, _vp, _vp, _vp, _vp, _vp, _i64, _i64, _i64, ctypes.c_float,
                                 ctypes.c_int, _vp, ctypes.c_size_t, _vp, ctypes.POINTER(ctypes.c_int),
                                 ctypes.POINTER(ctypes.c_float)]),
    "pararnn_lstm_solve_async": (_st, [_vp, _st, _vp, _vp, _vp, _vp, _vp, _i64, _i64, _i64,
                                       ctypes.c_float, ctypes.c_int, _vp, ctypes.c_size_t, _vp]),
    "pararnn_read_result": (_st, [_vp, _vp, ctypes.POINTER(Result)]),
    "pararnn_read_pass_times": (_st, [_vp, _vp, ctypes.POINTER(ctypes.c_double), ctypes.c_int,
                                      ctypes.POINTER(ctypes.c_int)]),
    "pararnn_gru_adjoint": (_st, [_vp, _st, _vp, _vp, _vp, _vp, _vp, _vp, _vp, _i64, _i64, _i64, _vp,
                                  ctypes.c_size_t, _vp]),
    "pararnn_lstm_adjoint": (_st, [_vp, _st, _vp, _vp, _vp, _vp, _vp, _vp, _vp, _vp, _vp, _vp, _vp,
                                   _i64, _i64, _i64, _vp, ctypes.c_size_t, _vp]),
    "pararnn_gru_sequential": (_st, [_vp, _st, _vp, _vp, _vp, _i64, _i64, _i64, _vp]),
    "pararnn_lstm_sequential": (_st, [_vp, _st, _vp, _vp, _vp, _vp, _vp, _i64, _i64, _i64, _vp]),
    "pararnn_cell_create": (_st, [ctypes.c_char_p, ctypes.c_int, ctypes.c_int, ctypes.c_uint,
                                  ctypes.POINTER(ctypes.c_void_p)]),
    "pararnn_cell_compute_warps": (ctypes.c_int, [_vp, _st]),
    "pararnn_cell_destroy": (None, [_vp]),
    "pararnn_cell_compile_log": (ctypes.c_char_p, []),
    "pararnn_cell_workspace_size": (ctypes.c_size_t, [_vp, _st, _i64, _i64, _i64]),
    "pararnn_cell_solve": (_st, [_vp, _vp, _st, _vp, _vp, _vp, _i64, _i64, _i64, ctypes.c_float, ctypes.c_int, _vp,
                                 ctypes.c_size_t, _vp, ctypes.POINTER(ctypes.c_int), ctypes.POINTER(ctypes.c_float)]),
    "pararnn_cell_adjoint_workspace_size": (ctypes.c_size_t, [_vp, _i64, _i64, _i64]),
    "pararnn_cell_adjoint": (_st, [_vp, _vp, _st, _vp, _vp, _vp, _vp, _vp, _vp, _vp, _i64, _i64, _i64, _vp,
                                   ctypes.c_size_t, _vp]),
    "pararnn_cell_solve_async": (_st, [_vp, _vp, _st, _vp, _vp, _vp, _i64, _i64, _i64, ctypes.c_float, ctypes.c_int,
                                       _vp, ctypes.c_size_t, _vp]),
    "pararnn_gru_segment_pass": (_st, [_vp, _st, _vp, _vp, _vp, _vp, _vp, _vp, _i64, _i64, _i64, _vp,
                                       ctypes.c_size_t, _vp]),
    "pararnn_lstm_segment_pass": (_st, [_vp, _st, _vp, _vp, _vp, _vp, _vp, _vp, _i64, _i64, _i64, _vp,
                                        ctypes.c_size_t, _vp]),
    "pararnn_result_to_device": (_st, [_vp, _vp, _vp]),
    "pararnn_gru_project_workspace_size": (ctypes.c_size_t, [_i64, _i64, _i64, _i64]),
    "pararnn_gru_project_solve": (_st, [_vp, _vp, _vp, _vp, _vp, _vp, _vp, _i64, _i64, _i64, _i64, ctypes.c_float,
                                        ctypes.c_int, _vp, ctypes.c_size_t, _vp, _vp, _vp]),
    "pararnn_gru_project_solve_async": (_st, [_vp, _vp, _vp, _vp, _vp, _vp, _vp, _i64, _i64, _i64, _i64,
                                              ctypes.c_float, ctypes.c_int, _vp, ctypes.c_size_t, _vp]),
    "pararnn_segment_record_floats": (ctypes.c_size_t, [ctypes.c_int, _i64, _i64]),
    "pararnn_segment_fold_workspace_size": (ctypes.c_size_t, [ctypes.c_int, _i64, _i64, _i64]),
    "pararnn_gru_segment_fold": (_st, [_vp, _st, _vp, _vp, _vp, _i64, _i64, _i64, _vp, ctypes.c_size_t, _vp]),
    "pararnn_lstm_segment_fold": (_st, [_vp, _st, _vp, _vp, _vp, _i64, _i64, _i64, _vp, ctypes.c_size_t, _vp]),
    "pararnn_gru_segment_combine": (_st, [_vp, ctypes.c_int, ctypes.c_int, _vp, _vp, _vp, _vp, _vp, _i64, _i64,
                                          _vp]),
    "pararnn_lstm_segment_combine": (_st, [_vp, ctypes.c_int, ctypes.c_int, _vp, _vp, _vp, _vp, _vp, _i64, _i64,
                                           _vp]),
    "pararnn_gru_step": (_st, [_vp, _st, _vp, _vp, _vp, _i64, _i64, _vp]),
    "pararnn_lstm_step": (_st, [_vp, _st, _vp, _vp, _vp, _vp, _vp, _i64, _i64, _vp]),
    "pararnn_linear_scan": (_st, [_vp, _st, _vp, _vp, _i64, _i64, _i64, _vp, ctypes.c_size_t, _vp]),
    "pararnn_status_string": (ctypes.c_char_p, [_st]),
    "pararnn_last_error": (ctypes.c_char_p, []),
    "pararnn_version": (ctypes.c_char_p, []),
    "pararnn_kernel_launch_count": (ctypes.c_uint64, []),
    "pararnn_selftest_wait_timeout": (_st, [ctypes.c_int, _i64, _vp, ctypes.c_size_t, _vp]),
}


def load(path=LIB_PATH):
    """Load a build of the library and declare its signatures."""
    if not os.path.exists(path):
        raise ImportError(f"{path} is not built; run `python -m nonlinear_rnn_newton_b200.build`")
    lib = ctypes.CDLL(path)
    for name, (res, args) in SIGNATURES.items():
        fn = getattr(lib, name)
        fn.restype = res
        fn.argtypes = args
    return lib


lib = load()


def last_error() -> str:
    return lib.pararnn_last_error().decode()


def status_string(s: int) -> str:
    return lib.pararnn_status_string(int(s)).decode()


def version() -> str:
    return lib.pararnn_version().decode()


def kernel_launch_count() -> int:
    return int(lib.pararnn_kernel_launch_count())


def _check(status, allow=(OK, NOT_CONVERGED, ERR_NONFINITE)):
    if status not in allow:
        raise PararnnError(status, f"{status_string(status)}: {last_error()}")
    return status


def _ptr(t):
    return None if t is None else ctypes.c_void_p(t.data_ptr())


def _stream(device, stream=None):
    if stream is None:
        stream = torch.cuda.current_stream(device)
    return ctypes.c_void_p(stream.cuda_stream)


def _dtype_code(u):
    if u.dtype == torch.bfloat16:
        return BF16
    if u.dtype == torch.float32:
        return F32
    raise TypeError(f"u must be bfloat16 or float32, got {u.dtype}")


def _need(t, name, shape, dtype=torch.float32, device=None):
    if t is None:
        return
    if tuple(t.shape) != tuple(shape):
        raise ValueError(f"{name}: expected shape {tuple(shape)}, got {tuple(t.shape)}")
    if t.dtype != dtype:
        raise TypeError(f"{name}: expected {dtype}, got {t.dtype}")
    if not t.is_contiguous():
        raise ValueError(f"{name} must be contiguous")
    if device is not None and t.device != device:
        raise ValueError(f"{name} must be on {device}, is on {t.device}")


def _workspace(nbytes, device, workspace):
    """The caller's workspace as is (the library checks its size), or a new one."""
    if workspace is None:
        return torch.empty(max(int(nbytes), 256), dtype=torch.uint8, device=device)
    return workspace


# ------------------------------------------------------------------ sizes

def pararnn_gru_workspace_size(B, L, D):
    return int(lib.pararnn_gru_workspace_size(B, L, D))


def pararnn_lstm_workspace_size(B, L, D):
    return int(lib.pararnn_lstm_workspace_size(B, L, D))


def pararnn_gru_adjoint_workspace_size(B, L, D):
    return int(lib.pararnn_gru_adjoint_workspace_size(B, L, D))


def pararnn_lstm_adjoint_workspace_size(B, L, D):
    return int(lib.pararnn_lstm_adjoint_workspace_size(B, L, D))


def pararnn_linear_scan_workspace_size(B, L, D):
    return int(lib.pararnn_linear_scan_workspace_size(B, L, D))


# ------------------------------------------------------------------ solves

def _to_device(t, device, stream):
    if t is None or t.device == device:
        return t
    with torch.cuda.stream(stream):
        return t.to(device, non_blocking=True)


def pararnn_gru_solve(u, a, h0=None, tol=1e-6, max_iters=10, h=None, workspace=None, stream=None,
                      device=None):
    """ParaGRU Newton solve.  u [B,L,3,D] (bf16/fp32), a [3,D] fp32, h0 [B,D]
    fp32 or None.  Returns (h [B,L,D], iters, residual, status).

    Device tensors are used in place.  Host (CPU) tensors are copied to
    ``device`` (default cuda:0) and the states copied back to the host."""
    host = u.device.type == "cpu"
    dev = torch.device(device or "cuda:0") if host else u.device
    strm = stream or torch.cuda.current_stream(dev)
    if host:
        u, a, h0 = (_to_device(t, dev, strm) for t in (u, a, h0))
    B, L, G, D = u.shape
    if G != 3:
        raise ValueError("GRU gates must be [B,L,3,D]")
    _need(a, "a", (3, D), device=dev)
    _need(h0, "h0", (B, D), device=dev)
    dh = h if (h is not None and not host) else None
    if dh is None:
        dh = torch.empty((B, L, D), dtype=torch.float32, device=dev)
    _need(dh, "h", (B, L, D), device=dev)
    ws = _workspace(pararnn_gru_workspace_size(B, L, D), dev, workspace)
    it = ctypes.c_int(0)
    res = ctypes.c_float(0.0)
    with torch.cuda.device(dev):
        st = lib.pararnn_gru_solve(_ptr(u), _dtype_code(u), _ptr(a), _ptr(h0), _ptr(dh), B, L, D,
                                   float(tol), int(max_iters), _ptr(ws), ws.numel(), _stream(dev, strm),
                                   ctypes.byref(it), ctypes.byref(res))
    _check(st)
    if host:
        out = h if h is not None else torch.empty((B, L, D), dtype=torch.float32, pin_memory=True)
        out.copy_(dh)
        dh = out
    return dh, it.value, res.value, st


def _gru_device_args(u, a, h0, h):
    """Shape, dtype, layout and device checks of a ParaGRU call on device
    tensors (the library checks pointers and sizes again, but it cannot see
    a tensor's shape or device); returns (B, L, D)."""
    if u.dim() != 4:
        raise ValueError(f"u must be [B,L,3,D], got shape {tuple(u.shape)}")
    B, L, G, D = u.shape
    if G != 3:
        raise ValueError("GRU gates must be [B,L,3,D]")
    _dtype_code(u)
    if not u.is_contiguous():
        raise ValueError("u must be contiguous")
    _need(a, "a", (3, D), device=u.device)
    _need(h0, "h0", (B, D), device=u.device)
    if h is None:
        raise ValueError("h (the output) is required")
    _need(h, "h", (B, L, D), device=u.device)
    return B, L, D


def pararnn_gru_solve_noalloc(u, a, h0, h, tol=1e-6, max_iters=10, stream=None):
    """ParaGRU Newton solve on the library's fixed device scratch (no
    workspace; device tensors only, h is the output).  Returns
    (iters, residual, status)."""
    B, L, D = _gru_device_args(u, a, h0, h)
    it = ctypes.c_int(0)
    res = ctypes.c_float(0.0)
    with torch.cuda.device(u.device):  # the scratch used is the current device's
        st = lib.pararnn_gru_solve_noalloc(_ptr(u), _dtype_code(u), _ptr(a), _ptr(h0), _ptr(h), B, L, D,
                                           float(tol), int(max_iters), _stream(u.device, stream),
                                           ctypes.byref(it), ctypes.byref(res))
    _check(st)
    return it.value, res.value, st


def pararnn_gru_project_workspace_size(B, L, D, Din):
    return int(lib.pararnn_gru_project_workspace_size(B, L, D, Din))


def _project_args(x, w, bias, a, h0, u, h):
    if x.dim() != 3 or w.dim() != 3:
        raise ValueError("x must be [B,L,Din] and w [3,D,Din]")
    B, L, Din = x.shape
    G, D, Din2 = w.shape
    if G != 3 or Din2 != Din:
        raise ValueError(f"w must be [3,D,{Din}], got {tuple(w.shape)}")
    _need(x, "x", (B, L, Din), dtype=torch.bfloat16, device=x.device)
    _need(w, "w", (3, D, Din), dtype=torch.bfloat16, device=x.device)
    _need(bias, "bias", (3, D), device=x.device)
    _need(a, "a", (3, D), device=x.device)
    _need(h0, "h0", (B, D), device=x.device)
    _need(u, "u", (B, L, 3, D), dtype=torch.bfloat16, device=x.device)
    _need(h, "h", (B, L, D), device=x.device)
    return B, L, Din, D


def pararnn_gru_project_solve(x, w, bias, a, h0=None, tol=1e-6, max_iters=10, u=None, h=None, workspace=None,
                              stream=None):
    """ParaGRU solve from the layer input: u = bf16(x w^T + bias) on the tensor
    cores with Newton pass 0 in the same kernel, then the rest of the solve.
    x [B,L,Din] bf16, w [3,D,Din] bf16, bias [3,D] fp32 or None (device
    tensors).  Returns (u [B,L,3,D] bf16, h [B,L,D], iters, residual, status)."""
    B, L, Din = x.shape
    D = w.shape[1]
    dev = x.device
    if u is None:
        u = torch.empty((B, L, 3, D), dtype=torch.bfloat16, device=dev)
    if h is None:
        h = torch.empty((B, L, D), dtype=torch.float32, device=dev)
    _project_args(x, w, bias, a, h0, u, h)
    ws = _workspace(pararnn_gru_project_workspace_size(B, L, D, Din), dev, workspace)
    it = ctypes.c_int(0)
    res = ctypes.c_float(0.0)
    with torch.cuda.device(dev):
        st = lib.pararnn_gru_project_solve(_ptr(x), _ptr(w), _ptr(bias), _ptr(a), _ptr(h0), _ptr(u), _ptr(h), B, L,
                                           Din, D, float(tol), int(max_iters), _ptr(ws),
                                           ws.numel() * ws.element_size(), _stream(dev, stream), ctypes.byref(it),
                                           ctypes.byref(res))
    _check(st)
    return u, h, it.value, res.value, st


def pararnn_gru_project_solve_async(x, w, bias, a, h0, u, h, workspace, tol=1e-6, max_iters=10, stream=None):
    """Queue the fused projection + solve (device tensors only); read the
    outcome with pararnn_read_result(workspace)."""
    B, L, Din, D = _project_args(x, w, bias, a, h0, u, h)
    st = lib.pararnn_gru_project_solve_async(_ptr(x), _ptr(w), _ptr(bias), _ptr(a), _ptr(h0), _ptr(u), _ptr(h), B,
                                             L, Din, D, float(tol), int(max_iters), _ptr(workspace),
                                             workspace.numel() * workspace.element_size(), _stream(x.device, stream))
    return _check(st)


def pararnn_gru_solve_noalloc_max_scratch():
    return lib.pararnn_gru_solve_noalloc_max_scratch()


def pararnn_gru_solve_async(u, a, h0, h, workspace, tol=1e-6, max_iters=10, stream=None):
    """Queue a ParaGRU solve (device tensors only); read the outcome with
    pararnn_read_result(workspace)."""
    B, L, D = _gru_device_args(u, a, h0, h)
    st = lib.pararnn_gru_solve_async(_ptr(u), _dtype_code(u), _ptr(a), _ptr(h0), _ptr(h), B, L, D,
                                     float(tol), int(max_iters), _ptr(workspace),
                                     workspace.numel() * workspace.element_size(),
                                     _stream(u.device, stream))
    return _check(st)


def pararnn_lstm_solve(u, a, c0=None, h0=None, tol=1e-6, max_iters=10, c=None, h=None, workspace=None,
                       stream=None, device=None):
    """ParaLSTM Newton solve.  u [B,L,4,D] gates (i,f,o,g).  Returns
    (c, h, iters, residual, status).  Host tensors are handled as in
    pararnn_gru_solve."""
    host = u.device.type == "cpu"
    dev = torch.device(device or "cuda:0") if host else u.device
    strm = stream or torch.cuda.current_stream(dev)
    if host:
        u, a, c0, h0 = (_to_device(t, dev, strm) for t in (u, a, c0, h0))
    B, L, G, D = u.shape
    if G != 4:
        raise ValueError("LSTM gates must be [B,L,4,D]")
    _need(a, "a", (4, D), device=dev)
    _need(c0, "c0", (B, D), device=dev)
    _need(h0, "h0", (B, D), device=dev)
    dc = c if (c is not None and not host) else torch.empty((B, L, D), dtype=torch.float32, device=dev)
    dh = h if (h is not None and not host) else torch.empty((B, L, D), dtype=torch.float32, device=dev)
    _need(dc, "c", (B, L, D), device=dev)
    _need(dh, "h", (B, L, D), device=dev)
    ws = _workspace(pararnn_lstm_workspace_size(B, L, D), dev, workspace)
    it = ctypes.c_int(0)
    res = ctypes.c_float(0.0)
    with torch.cuda.device(dev):
        st = lib.pararnn_lstm_solve(_ptr(u), _dtype_code(u), _ptr(a), _ptr(c0), _ptr(h0), _ptr(dc), _ptr(dh),
                                    B, L, D, float(tol), int(max_iters), _ptr(ws), ws.numel(),
                                    _stream(dev, strm), ctypes.byref(it), ctypes.byref(res))
    _check(st)
    if host:
        oc = c if c is not None else torch.empty((B, L, D), dtype=torch.float32, pin_memory=True)
        oh = h if h is not None else torch.empty((B, L, D), dtype=torch.float32, pin_memory=True)
        oc.copy_(dc)
        oh.copy_(dh)
        dc, dh = oc, oh
    return dc, dh, it.value, res.value, st


def pararnn_lstm_solve_async(u, a, c0, h0, c, h, workspace, tol=1e-6, max_iters=10, stream=None):
    B, L, G, D = u.shape
    st = lib.pararnn_lstm_solve_async(_ptr(u), _dtype_code(u), _ptr(a), _ptr(c0), _ptr(h0), _ptr(c), _ptr(h),
                                      B, L, D, float(tol), int(max_iters), _ptr(workspace),
                                      workspace.numel() * workspace.element_size(),
                                      _stream(u.device, stream))
    return _check(st)


def pararnn_read_result(workspace, stream=None):
    """Synchronise and return (status, iters, residual, residual0)."""
    r = Result()
    st = lib.pararnn_read_result(_ptr(workspace), _stream(workspace.device, stream), ctypes.byref(r))
    if st in (ERR_INVALID_ARG, ERR_WORKSPACE, ERR_CUDA):
        raise PararnnError(st, last_error())
    return r.status, r.iters, r.residual, r.residual0


def pararnn_read_pass_times(workspace, stream=None):
    """Synchronise and return the last solve's per-pass durations (us)."""
    buf = (ctypes.c_double * 16)()
    n = ctypes.c_int(0)
    st = lib.pararnn_read_pass_times(_ptr(workspace), _stream(workspace.device, stream), buf, 16, ctypes.byref(n))
    _check(st, allow=(OK,))
    return [buf[i] for i in range(n.value)]


# ---------------------------------------------------------------- adjoints

def pararnn_gru_adjoint(u, a, h0, h, dh, du=None, da=None, dh0=None, want_dh0=True, workspace=None,
                        stream=None):
    """Gradients through the ParaGRU solution.  Returns (du [B,L,3,D], da [3,D], dh0 [B,D] or None).
    Asynchronous on the stream."""
    B, L, G, D = u.shape
    dev = u.device
    du = du if du is not None else torch.empty((B, L, 3, D), dtype=torch.float32, device=dev)
    da = da if da is not None else torch.empty((3, D), dtype=torch.float32, device=dev)
    if dh0 is None and want_dh0:
        dh0 = torch.empty((B, D), dtype=torch.float32, device=dev)
    for t, n, s in ((a, "a", (3, D)), (h0, "h0", (B, D)), (h, "h", (B, L, D)), (dh, "dh", (B, L, D)),
                    (du, "du", (B, L, 3, D)), (da, "da", (3, D)), (dh0, "dh0", (B, D))):
        _need(t, n, s, device=dev)
    ws = _workspace(pararnn_gru_adjoint_workspace_size(B, L, D), dev, workspace)
    st = lib.pararnn_gru_adjoint(_ptr(u), _dtype_code(u), _ptr(a), _ptr(h0), _ptr(h), _ptr(dh), _ptr(du),
                                 _ptr(da), _ptr(dh0), B, L, D, _ptr(ws), ws.numel(), _stream(dev, stream))
    _check(st, allow=(OK,))
    return du, da, dh0


def pararnn_lstm_adjoint(u, a, c0, h0, c, h, dh, dc=None, du=None, da=None, dc0=None, dh0=None,
                         want_ds0=True, workspace=None, stream=None):
    """Gradients through the ParaLSTM solution.  Returns (du [B,L,4,D], da [4,D], dc0, dh0)."""
    B, L, G, D = u.shape
    dev = u.device
    du = du if du is not None else torch.empty((B, L, 4, D), dtype=torch.float32, device=dev)
    da = da if da is not None else torch.empty((4, D), dtype=torch.float32, device=dev)
    if want_ds0:
        dc0 = dc0 if dc0 is not None else torch.empty((B, D), dtype=torch.float32, device=dev)
        dh0 = dh0 if dh0 is not None else torch.empty((B, D), dtype=torch.float32, device=dev)
    for t, n, s in ((a, "a", (4, D)), (c0, "c0", (B, D)), (h0, "h0", (B, D)), (c, "c", (B, L, D)),
                    (h, "h", (B, L, D)), (dh, "dh", (B, L, D)), (dc, "dc", (B, L, D)),
                    (du, "du", (B, L, 4, D)), (da, "da", (4, D)), (dc0, "dc0", (B, D)), (dh0, "dh0", (B, D))):
        _need(t, n, s, device=dev)
    ws = _workspace(pararnn_lstm_adjoint_workspace_size(B, L, D), dev, workspace)
    st = lib.pararnn_lstm_adjoint(_ptr(u), _dtype_code(u), _ptr(a), _ptr(c0), _ptr(h0), _ptr(c), _ptr(h),
                                  _ptr(dh), _ptr(dc), _ptr(du), _ptr(da), _ptr(dc0), _ptr(dh0), B, L, D,
                                  _ptr(ws), ws.numel(), _stream(dev, stream))
    _check(st, allow=(OK,))
    return du, da, dc0, dh0


# ------------------------------------------------------ user-written cells

class CellHandle:
    """A compiled user cell (owns the library handle; destroyed with the object)."""

    def __init__(self, ptr, n_gates, n_state, log):
        self.ptr, self.n_gates, self.n_state, self.log = ptr, n_gates, n_state, log

    def __del__(self):
        if getattr(self, "ptr", None) and lib is not None:
            lib.pararnn_cell_destroy(self.ptr)
            self.ptr = None


CELL_FAST_MATH = 1


def pararnn_cell_create(source, n_gates, n_state, flags=0):
    """Compile `source` (which defines the templated recurrence_step) for the
    current CUDA device; raises PararnnError with the compiler's log on error.
    flags: CELL_FAST_MATH for the hardware approximations of the functions."""
    h = ctypes.c_void_p()
    st = lib.pararnn_cell_create(source.encode(), int(n_gates), int(n_state), int(flags), ctypes.byref(h))
    _check(st, allow=(OK,))
    return CellHandle(h, int(n_gates), int(n_state), pararnn_cell_compile_log())


def pararnn_cell_destroy(cell):
    if cell.ptr:
        lib.pararnn_cell_destroy(cell.ptr)
        cell.ptr = None


def pararnn_cell_compute_warps(cell, u_dtype):
    return int(lib.pararnn_cell_compute_warps(cell.ptr, BF16 if u_dtype == torch.bfloat16 else F32))


def pararnn_cell_compile_log():
    return lib.pararnn_cell_compile_log().decode()


def pararnn_cell_workspace_size(cell, u_dtype, B, L, D):
    code = BF16 if u_dtype == torch.bfloat16 else F32
    return int(lib.pararnn_cell_workspace_size(cell.ptr, code, B, L, D))


def pararnn_cell_solve(cell, u, a, s0=None, tol=1e-6, max_iters=10, s=None, workspace=None, stream=None):
    """u [B, L, G, D]; a [G, D]; s0 [NS, B, D] or None -> (s [NS, B, L, D], iters, residual, status)."""
    B, L, G, D = u.shape
    s = s if s is not None else torch.empty((cell.n_state, B, L, D), dtype=torch.float32, device=u.device)
    ws = _workspace(pararnn_cell_workspace_size(cell, u.dtype, B, L, D), u.device, workspace)
    it, res = ctypes.c_int(0), ctypes.c_float(0.0)
    with torch.cuda.device(u.device):
        st = lib.pararnn_cell_solve(cell.ptr, _ptr(u), _dtype_code(u), _ptr(a), _ptr(s0), _ptr(s), B, L, D,
                                    float(tol), int(max_iters), _ptr(ws), ws.numel(), _stream(u.device, stream),
                                    ctypes.byref(it), ctypes.byref(res))
    _check(st)
    return s, it.value, res.value, st


def pararnn_cell_adjoint_workspace_size(cell, B, L, D):
    return int(lib.pararnn_cell_adjoint_workspace_size(cell.ptr, B, L, D))


def pararnn_cell_adjoint(cell, u, a, s0, s, ds, du=None, da=None, ds0=None, want_ds0=True, workspace=None,
                         stream=None):
    """Gradients at converged states s [NS, B, L, D] for upstream ds [NS, B, L, D]
    -> (du [B, L, G, D], da [G, D], ds0 [NS, B, D] or None)."""
    B, L, G, D = u.shape
    dev = u.device
    du = du if du is not None else torch.empty((B, L, G, D), dtype=torch.float32, device=dev)
    da = da if da is not None else torch.empty((G, D), dtype=torch.float32, device=dev)
    if want_ds0 and ds0 is None:
        ds0 = torch.empty((cell.n_state, B, D), dtype=torch.float32, device=dev)
    ws = _workspace(pararnn_cell_adjoint_workspace_size(cell, B, L, D), dev, workspace)
    with torch.cuda.device(dev):
        st = lib.pararnn_cell_adjoint(cell.ptr, _ptr(u), _dtype_code(u), _ptr(a), _ptr(s0), _ptr(s), _ptr(ds),
                                      _ptr(du), _ptr(da), _ptr(ds0), B, L, D, _ptr(ws), ws.numel(),
                                      _stream(dev, stream))
    _check(st, allow=(OK,))
    return du, da, ds0


def pararnn_cell_solve_async(cell, u, a, s0, s, workspace, tol=1e-6, max_iters=10, stream=None):
    B, L, G, D = u.shape
    with torch.cuda.device(u.device):
        st = lib.pararnn_cell_solve_async(cell.ptr, _ptr(u), _dtype_code(u), _ptr(a), _ptr(s0), _ptr(s), B, L, D,
                                          float(tol), int(max_iters), _ptr(workspace), workspace.numel(),
                                          _stream(u.device, stream))
    _check(st, allow=(OK,))
    return st


# ------------------------------------------------- segments of a sequence

def _segment_pass(fn, u, a, s_in, s_lin, s_carry, s_out, s_end, workspace, stream):
    B, L, G, D = u.shape
    st = fn(_ptr(u), _dtype_code(u), _ptr(a), _ptr(s_in), _ptr(s_lin), _ptr(s_carry), _ptr(s_out), _ptr(s_end),
            B, L, D, _ptr(workspace), workspace.numel(), _stream(u.device, stream))
    _check(st, allow=(OK,))


def pararnn_gru_segment_pass(u, a, h_in, h_lin, h_carry, h_out, h_end=None, workspace=None, stream=None):
    """One Newton pass over a segment; states [1, B, Ls, D] / [1, B, D] (None = zeros)."""
    _segment_pass(lib.pararnn_gru_segment_pass, u, a, h_in, h_lin, h_carry, h_out, h_end, workspace, stream)


def pararnn_lstm_segment_pass(u, a, s_in, s_lin, s_carry, s_out, s_end=None, workspace=None, stream=None):
    """One Newton pass over a segment; states [2, B, Ls, D] / [2, B, D] (c, h; None = zeros)."""
    _segment_pass(lib.pararnn_lstm_segment_pass, u, a, s_in, s_lin, s_carry, s_out, s_end, workspace, stream)


def pararnn_result_to_device(workspace, out, stream=None):
    """Queue the last pass's residual and error flag into out (2 device floats)."""
    _check(lib.pararnn_result_to_device(_ptr(workspace), _ptr(out), _stream(workspace.device, stream)), allow=(OK,))


def pararnn_segment_record_floats(n_state, B, D):
    return int(lib.pararnn_segment_record_floats(n_state, B, D))


def pararnn_segment_fold_workspace_size(n_state, B, L, D):
    return int(lib.pararnn_segment_fold_workspace_size(n_state, B, L, D))


def _segment_fold(fn, u, a, s_in, record, workspace, stream):
    B, L, G, D = u.shape
    st = fn(_ptr(u), _dtype_code(u), _ptr(a), _ptr(s_in), _ptr(record), B, L, D, _ptr(workspace),
            workspace.numel() * workspace.element_size(), _stream(u.device, stream))
    _check(st, allow=(OK,))


def pararnn_gru_segment_fold(u, a, h_in, record, workspace, stream=None):
    """The segment's record (flat, pararnn_segment_record_floats(1, B, D)) from the
    iterate h_in [1, B, Ls, D] (None = the zero guess)."""
    _segment_fold(lib.pararnn_gru_segment_fold, u, a, h_in, record, workspace, stream)


def pararnn_lstm_segment_fold(u, a, s_in, record, workspace, stream=None):
    """The segment's record from the iterate s_in [2, B, Ls, D] (c, h; None = the zero guess)."""
    _segment_fold(lib.pararnn_lstm_segment_fold, u, a, s_in, record, workspace, stream)


def _segment_combine(fn, records, index, a, s0, carry, lin, residual, stream):
    R = records.shape[0]
    NS, B, D = carry.shape
    st = fn(_ptr(records), R, index, _ptr(a), _ptr(s0), _ptr(carry), _ptr(lin), _ptr(residual), B, D,
            _stream(records.device, stream))
    _check(st, allow=(OK,))


def pararnn_gru_segment_combine(records, index, a, h0, h_carry, h_lin, residual, stream=None):
    """records [R, record_floats] in segment order -> h_carry, h_lin [1, B, D]
    of segment `index` and residual (1 float) of the iterate over all segments."""
    _segment_combine(lib.pararnn_gru_segment_combine, records, index, a, h0, h_carry, h_lin, residual, stream)


def pararnn_lstm_segment_combine(records, index, a, s0, s_carry, s_lin, residual, stream=None):
    """As pararnn_gru_segment_combine with states [2, B, D] (c, h)."""
    _segment_combine(lib.pararnn_lstm_segment_combine, records, index, a, s0, s_carry, s_lin, residual, stream)


# ------------------------------------------------------------- decode step

def pararnn_gru_step(u, a, h_prev=None, h_next=None, stream=None):
    """One step for B sequences: u [B, 3, D], h_prev [B, D] (None = zeros).
    h_next may be h_prev itself (in place); a new tensor if None."""
    B, G, D = u.shape
    h_next = h_next if h_next is not None else torch.empty((B, D), dtype=torch.float32, device=u.device)
    st = lib.pararnn_gru_step(_ptr(u), _dtype_code(u), _ptr(a), _ptr(h_prev), _ptr(h_next), B, D,
                              _stream(u.device, stream))
    _check(st, allow=(OK,))
    return h_next


def pararnn_lstm_step(u, a, c_prev=None, h_prev=None, c_next=None, h_next=None, stream=None):
    """One step for B sequences: u [B, 4, D], c_prev, h_prev [B, D] (None = zeros)."""
    B, G, D = u.shape
    c_next = c_next if c_next is not None else torch.empty((B, D), dtype=torch.float32, device=u.device)
    h_next = h_next if h_next is not None else torch.empty((B, D), dtype=torch.float32, device=u.device)
    st = lib.pararnn_lstm_step(_ptr(u), _dtype_code(u), _ptr(a), _ptr(c_prev), _ptr(h_prev), _ptr(c_next),
                               _ptr(h_next), B, D, _stream(u.device, stream))
    _check(st, allow=(OK,))
    return c_next, h_next


# --------------------------------------------------------------- baselines

def pararnn_gru_sequential(u, a, h0=None, h=None, stream=None):
    B, L, G, D = u.shape
    h = h if h is not None else torch.empty((B, L, D), dtype=torch.float32, device=u.device)
    st = lib.pararnn_gru_sequential(_ptr(u), _dtype_code(u), _ptr(a), _ptr(h0), _ptr(h), B, L, D,
                                    _stream(u.device, stream))
    _check(st, allow=(OK,))
    return h


def pararnn_lstm_sequential(u, a, c0=None, h0=None, c=None, h=None, stream=None):
    B, L, G, D = u.shape
    c = c if c is not None else torch.empty((B, L, D), dtype=torch.float32, device=u.device)
    h = h if h is not None else torch.empty((B, L, D), dtype=torch.float32, device=u.device)
    st = lib.pararnn_lstm_sequential(_ptr(u), _dtype_code(u), _ptr(a), _ptr(c0), _ptr(h0), _ptr(c), _ptr(h),
                                     B, L, D, _stream(u.device, stream))
    _check(st, allow=(OK,))
    return c, h


def pararnn_linear_scan(u, h0=None, h=None, workspace=None, stream=None):
    B, L, G, D = u.shape
    h = h if h is not None else torch.empty((B, L, D), dtype=torch.float32, device=u.device)
    ws = _workspace(pararnn_linear_scan_workspace_size(B, L, D), u.device, workspace)
    st = lib.pararnn_linear_scan(_ptr(u), _dtype_code(u), _ptr(h0), _ptr(h), B, L, D, _ptr(ws), ws.numel(),
                                 _stream(u.device, stream))
    _check(st, allow=(OK,))
    return h


def pararnn_selftest_wait_timeout(which, limit_ns, workspace, stream=None):
    """Returns the status (ERR_TIMEOUT expected)."""
    return int(lib.pararnn_selftest_wait_timeout(int(which), int(limit_ns), _ptr(workspace),
                                                 workspace.numel(), _stream(workspace.device, stream)))
