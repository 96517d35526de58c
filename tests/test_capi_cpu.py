"""The C-ABI library on the CPU (no GPU needed): it loads, exports every entry
point the header declares, sizes workspaces, and rejects bad arguments before
queueing any GPU work."""
import ctypes
import os
import re

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
HEADER = os.path.join(ROOT, "include", "pararnn.h")


@pytest.fixture(scope="module")
def capi():
    from nonlinear_rnn_newton_b200 import build
    build.build()
    from nonlinear_rnn_newton_b200 import capi
    return capi


def declared_symbols():
    text = open(HEADER).read()
    return sorted(set(re.findall(r"PARARNN_API[^;(]*?\b(pararnn_\w+)\s*\(", text)))


def test_header_declares_the_entry_points():
    names = declared_symbols()
    for n in ("pararnn_gru_solve", "pararnn_lstm_solve", "pararnn_gru_adjoint", "pararnn_lstm_adjoint",
              "pararnn_gru_workspace_size", "pararnn_read_result", "pararnn_gru_sequential",
              "pararnn_linear_scan", "pararnn_status_string", "pararnn_last_error"):
        assert n in names


def test_library_exports_every_declared_symbol(capi):
    lib = ctypes.CDLL(capi.LIB_PATH)
    missing = [n for n in declared_symbols() if not hasattr(lib, n)]
    assert not missing, missing
    # and the binding wraps every one of them
    assert set(declared_symbols()) <= set(capi.SIGNATURES)


def test_version_and_status_strings(capi):
    assert re.match(r"^\d+\.\d+\.\d+$", capi.version())
    assert capi.status_string(0) == "ok"
    assert "timed out" in capi.status_string(-4)
    assert capi.status_string(123) == "unknown status"


def test_workspace_sizes(capi):
    from nonlinear_rnn_newton_b200 import capi as c
    g = c.pararnn_gru_workspace_size(8, 4096, 1024)
    l = c.pararnn_lstm_workspace_size(8, 4096, 1024)
    assert 0 < g < l
    assert g % 256 == 0 and l % 256 == 0
    assert c.pararnn_gru_workspace_size(8, 4096, 1020) == 0  # D not a multiple of 8
    assert c.pararnn_gru_workspace_size(0, 4096, 1024) == 0
    assert c.pararnn_gru_adjoint_workspace_size(4, 16384, 2048) > 0
    assert c.pararnn_lstm_adjoint_workspace_size(4, 16384, 2048) > 0
    assert c.pararnn_linear_scan_workspace_size(1, 65536, 2048) > 0
    # monotone in every dimension
    assert c.pararnn_gru_workspace_size(8, 8192, 1024) > g
    assert c.pararnn_gru_workspace_size(16, 4096, 1024) > g


def _solve(capi, u=16, a=16, h0=None, h=16, B=1, L=8, D=16, tol=1e-6, it=10, ws=256, wsb=1 << 30, dt=1):
    lib = capi.lib
    return lib.pararnn_gru_solve(u, dt, a, h0, h, B, L, D, tol, it, ws, wsb, None, None, None)


def test_argument_checks_before_any_gpu_work(capi):
    E = capi
    assert _solve(capi, u=None) == E.ERR_INVALID_ARG
    assert "u is NULL" in capi.last_error()
    assert _solve(capi, a=None) == E.ERR_INVALID_ARG
    assert _solve(capi, h=None) == E.ERR_INVALID_ARG
    assert _solve(capi, u=8) == E.ERR_INVALID_ARG  # misaligned
    assert "aligned" in capi.last_error()
    assert _solve(capi, D=12) == E.ERR_UNSUPPORTED
    assert _solve(capi, B=0) == E.ERR_INVALID_ARG
    assert _solve(capi, L=-3) == E.ERR_INVALID_ARG
    assert _solve(capi, tol=-1.0) == E.ERR_INVALID_ARG
    assert _solve(capi, tol=float("inf")) == E.ERR_INVALID_ARG
    assert _solve(capi, tol=float("nan")) == E.ERR_INVALID_ARG
    assert _solve(capi, it=-1) == E.ERR_INVALID_ARG
    assert _solve(capi, dt=7) == E.ERR_INVALID_ARG
    assert _solve(capi, ws=None) == E.ERR_WORKSPACE
    assert _solve(capi, ws=16) == E.ERR_WORKSPACE  # not 256-byte aligned
    assert _solve(capi, wsb=100) == E.ERR_WORKSPACE
    assert _solve(capi, B=1 << 20, L=1 << 20, D=1 << 10) == E.ERR_INVALID_ARG  # too large
    lib = capi.lib
    # LSTM, adjoints and baselines check too
    assert lib.pararnn_lstm_solve(16, 1, 16, None, None, None, 16, 1, 8, 16, 1e-6, 10, 256, 1 << 30, None,
                                  None, None) == E.ERR_INVALID_ARG
    assert lib.pararnn_gru_adjoint(16, 1, 16, None, 16, None, 16, 16, None, 1, 8, 16, 256, 1 << 30,
                                   None) == E.ERR_INVALID_ARG
    assert lib.pararnn_lstm_adjoint(16, 1, 16, None, None, 16, 16, 16, None, 16, 16, None, None, 1, 8, 12,
                                    256, 1 << 30, None) == E.ERR_UNSUPPORTED
    assert lib.pararnn_gru_sequential(16, 1, None, None, 16, 1, 8, 16, None) == E.ERR_INVALID_ARG
    assert lib.pararnn_linear_scan(16, 1, None, 16, 1, 8, 16, 256, 10, None) == E.ERR_WORKSPACE
    assert lib.pararnn_selftest_wait_timeout(5, 10, 256, 16384, None) == E.ERR_INVALID_ARG
    n = ctypes.c_int(0)
    assert lib.pararnn_read_pass_times(None, None, None, 0, ctypes.byref(n)) == E.ERR_WORKSPACE
    assert lib.pararnn_read_pass_times(256, None, None, 4, ctypes.byref(n)) == E.ERR_INVALID_ARG


def test_segment_checks(capi):
    """The sequence-split pieces check their arguments before any launch."""
    E, lib = capi, capi.lib
    seg = lambda u=16, a=16, si=None, so=4096, B=1, L=8, D=16, ws=256, wsb=1 << 20: lib.pararnn_gru_segment_pass(
        u, 1, a, si, None, None, so, None, B, L, D, ws, wsb, None)
    assert seg(u=None) == E.ERR_INVALID_ARG
    assert seg(so=None) == E.ERR_INVALID_ARG
    assert seg(D=12) == E.ERR_UNSUPPORTED
    assert seg(ws=None) == E.ERR_WORKSPACE
    assert seg(si=4096, so=4096 + 64) == E.ERR_INVALID_ARG  # output overlaps the iterate it reads
    assert "overlaps" in capi.last_error()
    assert lib.pararnn_lstm_segment_pass(16, 1, 16, None, None, None, None, None, 1, 8, 16, 256, 1 << 20,
                                         None) == E.ERR_INVALID_ARG
    fold = lambda u=16, rec=4096, D=16, ws=256, wsb=1 << 20: lib.pararnn_gru_segment_fold(
        u, 1, 16, None, rec, 1, 8, D, ws, wsb, None)
    assert fold(u=None) == E.ERR_INVALID_ARG
    assert fold(rec=None) == E.ERR_INVALID_ARG
    assert fold(D=12) == E.ERR_UNSUPPORTED
    assert fold(ws=None) == E.ERR_WORKSPACE
    assert fold(wsb=16) == E.ERR_WORKSPACE
    comb = lambda R=2, i=0, res=4096, B=1, D=16: lib.pararnn_gru_segment_combine(16, R, i, 16, None, 16, 16, res,
                                                                                  B, D, None)
    assert comb(R=0) == E.ERR_INVALID_ARG
    assert comb(i=2) == E.ERR_INVALID_ARG
    assert comb(res=None) == E.ERR_INVALID_ARG
    assert comb(B=0) == E.ERR_INVALID_ARG
    assert comb(D=12) == E.ERR_UNSUPPORTED
    # record: F = NC + 2 NS + G fields of B*D floats, then 4 floats
    assert lib.pararnn_segment_record_floats(1, 2, 16) == (2 + 2 + 3) * 32 + 4
    assert lib.pararnn_segment_record_floats(2, 2, 16) == (6 + 4 + 4) * 32 + 4
    assert lib.pararnn_segment_record_floats(3, 2, 16) == 0
    # partial folds of steps 2..L of the segment, 64 steps each, or twice as
    # many steps until at most 256 parts remain
    assert lib.pararnn_segment_fold_workspace_size(1, 1, 129, 16) == 256
    assert lib.pararnn_segment_fold_workspace_size(2, 4, 257, 64) == 4 * 6 * 4 * 64 * 4
    assert lib.pararnn_segment_fold_workspace_size(2, 4, 258, 64) == 5 * 6 * 4 * 64 * 4
    assert lib.pararnn_segment_fold_workspace_size(1, 1, 64 * 256 + 1, 16) == 256 * 2 * 16 * 4
    assert lib.pararnn_segment_fold_workspace_size(1, 1, 64 * 256 + 2, 16) == (129 * 2 * 16 * 4 + 255) // 256 * 256


def test_decode_step_checks(capi):
    """The decode step refuses bad shapes, pointers and partial overlaps
    before any launch; an output that is its own previous state passes."""
    E, lib = capi, capi.lib
    gru = lambda u=16, a=16, hp=None, hn=4096, B=1, D=16: lib.pararnn_gru_step(u, 1, a, hp, hn, B, D, None)
    assert gru(D=12) == E.ERR_UNSUPPORTED
    assert gru(B=0) == E.ERR_INVALID_ARG
    assert gru(u=None) == E.ERR_INVALID_ARG
    assert gru(hn=4104) == E.ERR_INVALID_ARG  # misaligned
    assert gru(hp=4096 - 48, hn=4096) == E.ERR_INVALID_ARG  # ranges of 64 bytes overlap
    assert "overlaps" in capi.last_error()
    lstm = lambda cp=None, hp=None, cn=4096, hn=8192, D=16: lib.pararnn_lstm_step(16, 1, 16, cp, hp, cn, hn, 1, D,
                                                                                   None)
    assert lstm(cn=8192, hn=8192) == E.ERR_INVALID_ARG
    assert lstm(hp=4096) == E.ERR_INVALID_ARG  # h_prev is c_next
    assert lstm(cp=8192) == E.ERR_INVALID_ARG  # c_prev is h_next
    assert lstm(D=4) == E.ERR_UNSUPPORTED


def test_valid_arguments_without_gpu_report_cuda_error(capi):
    import torch
    if torch.cuda.is_available():
        pytest.skip("a GPU is present")
    assert _solve(capi) == capi.ERR_CUDA
    assert capi.last_error()
    # in place (the output is its own previous state): accepted, then no device
    assert capi.lib.pararnn_gru_step(16, 1, 16, 4096, 4096, 1, 16, None) == capi.ERR_CUDA
    assert capi.lib.pararnn_lstm_step(16, 1, 16, 4096, 8192, 4096, 8192, 1, 16, None) == capi.ERR_CUDA


def test_binding_fails_loudly_without_library(tmp_path, monkeypatch):
    import importlib.util
    spec = importlib.util.spec_from_file_location(
        "capi_copy", os.path.join(ROOT, "nonlinear_rnn_newton_b200", "capi.py"))
    mod = importlib.util.module_from_spec(spec)
    monkeypatch.setattr(os.path, "exists", lambda p: False if p.endswith("libpararnn.so") else True)
    with pytest.raises(ImportError):
        spec.loader.exec_module(mod)
