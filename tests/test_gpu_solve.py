"""GPU parity of the Newton solves against the CPU oracle, through the C ABI.

States: max-abs error against the oracle's sequential stepping on the same
(bf16-decoded) inputs <= 1e-4 (fp32 state; the pages' method reaches the
sequential states exactly, so the oracle for states is plain stepping).  The
bound for bf16 inputs against fp32 inputs would be 2e-2; since both sides here
read the identical bf16 tensor, the stricter 1e-4 applies to every case.
Iterations: equal to the oracle's serial Newton, or +-1 where the oracle's
residual at that step is within 10x of tol.
"""
import math

import numpy as np
import pytest
import torch

import oracle
from nonlinear_rnn_newton_b200 import workloads as W
from tests import helpers as H

pytestmark = pytest.mark.gpu

TOL_STATE = 1e-4


def P():
    import nonlinear_rnn_newton_b200 as pkg
    return pkg


def run_gru(x, dev, tol=1e-6, max_iters=10):
    xd = x.to(dev)
    h, it, r, st = P().pararnn_gru_solve(xd.u, xd.a, xd.h0, tol=tol, max_iters=max_iters)
    torch.cuda.synchronize()
    return h.cpu().double().numpy(), it, r, st


def run_lstm(x, dev, tol=1e-6, max_iters=10):
    xd = x.to(dev)
    c, h, it, r, st = P().pararnn_lstm_solve(xd.u, xd.a, xd.c0, xd.h0, tol=tol, max_iters=max_iters)
    torch.cuda.synchronize()
    return c.cpu().double().numpy(), h.cpu().double().numpy(), it, r, st


# ------------------------------------------------------------- small, whole

GRU_CASES = [
    W.GRU_SMALL,                                            # fp32, D < one tile
    W.custom("gru", 3, 333, 200, "bf16", h0_std=0.1),       # ragged L and D
    W.custom("gru", 1, 64, 128, "bf16", h0_std=0.1),        # exactly one tile
    W.custom("gru", 2, 1000, 264, "f32", h0_std=0.1),       # several chunks, ragged
    W.custom("gru", 1, 1, 8, "bf16", h0_std=0.1),           # L = 1, smallest D
    W.custom("gru", 5, 2049, 136, "bf16", h0_std=0.1),      # many tiles
]


@pytest.mark.parametrize("w", GRU_CASES, ids=lambda w: w.name)
def test_gru_solve_matches_oracle(cuda, w):
    x = W.make_inputs(w, seed=0)
    h, it, r, st = run_gru(x, cuda, w.tol, w.max_iters)
    seq = oracle.gru_seq(x.u, x.a, x.h0)
    err = H.max_abs(h, seq)
    assert err <= TOL_STATE, f"max-abs error {err:.3e}"
    hn, oit, ores, ost, hist = oracle.gru_newton(x.u, x.a, x.h0, tol=w.tol, max_iters=w.max_iters)
    assert H.iters_agree(it, oit, hist, w.tol), (it, oit, hist)
    assert st == (0 if r <= w.tol else 1)
    if it == oit:
        # the returned residual is the residual of the returned states
        assert r <= max(10 * hist[it], 2e-6) or abs(r - hist[it]) <= 1e-3 * hist[it] + 1e-6, (r, hist)


LSTM_CASES = [
    W.custom("lstm", 2, 256, 64, "f32"),
    W.custom("lstm", 3, 300, 136, "bf16"),
    W.custom("lstm", 1, 1, 8, "bf16"),
    W.custom("lstm", 2, 1025, 256, "bf16"),
]


@pytest.mark.parametrize("w", LSTM_CASES, ids=lambda w: w.name)
def test_lstm_solve_matches_oracle(cuda, w):
    x = W.make_inputs(w, seed=0)
    c, h, it, r, st = run_lstm(x, cuda, w.tol, w.max_iters)
    cs, hs = oracle.lstm_seq(x.u, x.a, x.c0, x.h0)
    assert H.max_abs(c, cs) <= TOL_STATE
    assert H.max_abs(h, hs) <= TOL_STATE
    *_, oit, ores, ost, hist = oracle.lstm_newton(x.u, x.a, x.c0, x.h0, tol=w.tol, max_iters=w.max_iters)
    assert H.iters_agree(it, oit, hist, w.tol), (it, oit, hist)


def test_lstm_nonzero_initial_state(cuda):
    w = W.custom("lstm", 2, 200, 128, "bf16")
    x = W.make_inputs(w, seed=3)
    g = torch.Generator().manual_seed(9)
    x.c0 = torch.randn(2, 128, generator=g) * 0.5
    x.h0 = torch.randn(2, 128, generator=g) * 0.5
    c, h, it, r, st = run_lstm(x, cuda)
    cs, hs = oracle.lstm_seq(x.u, x.a, x.c0, x.h0)
    assert H.max_abs(c, cs) <= TOL_STATE and H.max_abs(h, hs) <= TOL_STATE


# ------------------------------------------------------- Newton properties

@pytest.mark.parametrize("k", [1, 2, 3])
def test_gru_first_k_states_exact(cuda, k):
    w = W.custom("gru", 2, 300, 136, "bf16", h0_std=0.1)
    x = W.make_inputs(w, seed=5)
    h, it, r, st = run_gru(x, cuda, tol=0.0, max_iters=k)
    assert it == k and st == 1
    seq = oracle.gru_seq(x.u, x.a, x.h0)
    assert H.max_abs(h[:, :k], seq[:, :k]) <= 2e-6
    # and the whole iterate equals the oracle's k-th Newton iterate
    hk, *_ = oracle.gru_newton(x.u, x.a, x.h0, tol=0.0, max_iters=k)
    assert H.max_abs(h, hk) <= 1e-4


@pytest.mark.parametrize("k", [1, 2])
def test_lstm_first_k_states_exact(cuda, k):
    w = W.custom("lstm", 2, 200, 128, "bf16")
    x = W.make_inputs(w, seed=6)
    c, h, it, r, st = run_lstm(x, cuda, tol=0.0, max_iters=k)
    assert it == k
    cs, hs = oracle.lstm_seq(x.u, x.a, x.c0, x.h0)
    assert H.max_abs(c[:, :k], cs[:, :k]) <= 2e-6 and H.max_abs(h[:, :k], hs[:, :k]) <= 2e-6
    ck, hk, *_ = oracle.lstm_newton(x.u, x.a, x.c0, x.h0, tol=0.0, max_iters=k)
    assert H.max_abs(c, ck) <= 1e-4 and H.max_abs(h, hk) <= 1e-4


def test_gru_zero_weights_one_iteration(cuda):
    w = W.custom("gru", 4, 777, 256, "bf16", h0_std=0.1)
    x = W.make_inputs(w, seed=7, a_scale=0.0)
    h, it, r, st = run_gru(x, cuda)
    assert it == 1 and st == 0 and r <= 1e-6
    assert H.max_abs(h, oracle.gru_seq(x.u, x.a, x.h0)) <= TOL_STATE


def test_lstm_zero_weights_two_iterations(cuda):
    w = W.custom("lstm", 4, 500, 128, "bf16")
    x = W.make_inputs(w, seed=8, a_scale=0.0)
    c, h, it, r, st = run_lstm(x, cuda)
    assert it == 2 and st == 0


def test_max_iters_zero_returns_initial_guess(cuda):
    w = W.custom("gru", 2, 100, 64, "bf16", h0_std=0.1)
    x = W.make_inputs(w, seed=9)
    h, it, r, st = run_gru(x, cuda, tol=1e-6, max_iters=0)
    _, oit, ores, ost, hist = oracle.gru_newton(x.u, x.a, x.h0, tol=1e-6, max_iters=0)
    assert it == 0 and st == 1 and np.all(h == 0)
    assert abs(r - hist[0]) <= 1e-5 * hist[0]


def test_huge_tolerance_converges_at_initial_guess(cuda):
    w = W.custom("lstm", 1, 100, 64, "f32")
    x = W.make_inputs(w, seed=10)
    c, h, it, r, st = run_lstm(x, cuda, tol=1e9, max_iters=5)
    assert it == 0 and st == 0 and np.all(h == 0) and np.all(c == 0)


def test_not_converged_status(cuda):
    w = W.custom("gru", 2, 500, 128, "bf16", h0_std=0.1)
    x = W.make_inputs(w, seed=11)
    h, it, r, st = run_gru(x, cuda, tol=1e-6, max_iters=2)
    assert it == 2 and st == 1 and r > 1e-6
    hk, *_ = oracle.gru_newton(x.u, x.a, x.h0, tol=0.0, max_iters=2)
    assert H.max_abs(h, hk) <= 1e-4


def test_nonfinite_input_reports_nonfinite(cuda):
    w = W.custom("gru", 1, 200, 64, "f32", h0_std=0.1)
    x = W.make_inputs(w, seed=12)
    x.u[0, 150, 1, 7] = float("nan")
    h, it, r, st = run_gru(x, cuda)
    assert st == -5 and math.isnan(r)
    w = W.custom("lstm", 1, 200, 64, "f32")
    x = W.make_inputs(w, seed=13)
    x.u[0, 10, 3, 0] = float("nan")
    c, h, it, r, st = run_lstm(x, cuda)
    assert st == -5


def _same_outcome(a, b):
    """(states, iters, residual, status) equal, NaN where NaN."""
    (ha, ia, ra, sa), (hb, ib, rb, sb) = a, b
    assert (ia, sa) == (ib, sb)
    assert (math.isnan(ra) and math.isnan(rb)) or ra == rb
    assert np.array_equal(np.isnan(ha), np.isnan(hb))
    assert np.array_equal(np.nan_to_num(ha), np.nan_to_num(hb))


@pytest.mark.parametrize("shape", [(8, 4096, 1024), (1, 8192, 2048)], ids=["B8", "B1"])
def test_partial_residuals_leave_the_outcome_unchanged(cuda, shape):
    """A ParaGRU pass that is not the last allowed one stops evaluating the
    residual once a tile has found one above tol.  The same solve capped at
    its own iteration count (every pass then evaluates it in full, the last
    one being the last allowed) must give the same states, count, residual
    and status."""
    B, L, D = shape
    w = W.custom("gru", B, L, D, "bf16", h0_std=0.1)
    x = W.make_inputs(w, seed=21)
    full = run_gru(x, cuda, max_iters=10)
    assert full[3] == 0 and full[1] >= 3
    capped = run_gru(x, cuda, max_iters=full[1])
    _same_outcome(full, capped)


def test_iterates_that_overflow_report_nonfinite(cuda):
    """Recurrence weights so large that the Newton update overflows: the
    non-finite states must be caught in the pass that makes them, as when
    that pass is the last allowed one (full residual)."""
    w = W.custom("gru", 2, 3000, 256, "bf16", h0_std=0.1)
    x = W.make_inputs(w, seed=22, a_scale=4000.0)
    out = run_gru(x, cuda, max_iters=10)
    assert out[3] == -5 and not np.isfinite(out[0]).all()
    capped = run_gru(x, cuda, max_iters=out[1])
    _same_outcome(out, capped)


def test_solve_is_deterministic(cuda):
    w = W.custom("gru", 4, 2048, 512, "bf16", h0_std=0.1)
    x = W.make_inputs(w, seed=14).to(cuda)
    pk = P()
    h1, i1, r1, _ = pk.pararnn_gru_solve(x.u, x.a, x.h0)
    h2, i2, r2, _ = pk.pararnn_gru_solve(x.u, x.a, x.h0)
    assert i1 == i2 and r1 == r2 and torch.equal(h1, h2)


def test_pass_times(cuda):
    """One timestamp per finished pass: as many passes as updates (one when
    the initial guess already satisfies the rule), each positive, summing to
    most of the launch's CUDA-event time."""
    pk = P()
    w = W.custom("gru", 4, 4096, 512, "bf16", h0_std=0.1)
    x = W.make_inputs(w, seed=17).to(cuda)
    h = torch.empty((w.B, w.L, w.D), device=cuda)
    ws = torch.empty(pk.pararnn_gru_workspace_size(w.B, w.L, w.D), dtype=torch.uint8, device=cuda)
    s = torch.cuda.current_stream()
    for tol, max_iters in ((1e-6, 10), (1e30, 10), (0.0, 3)):
        pk.pararnn_gru_solve_async(x.u, x.a, x.h0, h, ws, tol, max_iters)
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        e0.record(s)
        pk.pararnn_gru_solve_async(x.u, x.a, x.h0, h, ws, tol, max_iters)
        e1.record(s)
        st, it, r, r0 = pk.pararnn_read_result(ws)
        us = pk.pararnn_read_pass_times(ws)
        assert len(us) == max(it, 1), (tol, max_iters, it, us)
        assert all(t > 0 for t in us)
        total = e0.elapsed_time(e1) * 1e3
        assert 0.3 * total <= sum(us) <= 1.02 * total, (us, total)


def test_sequential_baselines_match_oracle(cuda):
    w = W.custom("gru", 3, 500, 136, "bf16", h0_std=0.1)
    x = W.make_inputs(w, seed=15)
    xd = x.to(cuda)
    h = P().pararnn_gru_sequential(xd.u, xd.a, xd.h0).cpu().double().numpy()
    assert H.max_abs(h, oracle.gru_seq(x.u, x.a, x.h0)) <= TOL_STATE
    w = W.custom("lstm", 2, 400, 64, "f32")
    x = W.make_inputs(w, seed=16)
    xd = x.to(cuda)
    c, h = P().pararnn_lstm_sequential(xd.u, xd.a, xd.c0, xd.h0)
    cs, hs = oracle.lstm_seq(x.u, x.a, x.c0, x.h0)
    assert H.max_abs(c.cpu().numpy(), cs) <= TOL_STATE and H.max_abs(h.cpu().numpy(), hs) <= TOL_STATE


# (2, 1000, 200): groups of one sequence step back over aggregates (few
# sequences), ragged tail and slab; (40, 300, 128): many sequences, so
# look-backs wait for inclusive values; fp32: the shorter tile
@pytest.mark.parametrize("shape,dt", [((2, 1000, 200), "bf16"), ((1, 64, 128), "bf16"), ((3, 1, 8), "bf16"),
                                      ((40, 300, 128), "bf16"), ((2, 777, 136), "f32")])
def test_linear_scan_matches_zero_weight_oracle(cuda, shape, dt):
    B, L, D = shape
    w = W.custom("gru", B, L, D, dt, h0_std=0.1)
    x = W.make_inputs(w, seed=17)
    xd = x.to(cuda)
    h = P().pararnn_linear_scan(xd.u, xd.h0).cpu().double().numpy()
    ref = oracle.gru_seq(x.u, torch.zeros_like(x.a), x.h0)
    assert H.max_abs(h, ref) <= TOL_STATE


# ---------------------------------------------------------------- errors

def test_argument_errors(cuda):
    from nonlinear_rnn_newton_b200 import capi
    pk = P()
    u = torch.zeros(1, 8, 3, 12, device=cuda)
    a = torch.zeros(3, 12, device=cuda)
    with pytest.raises(capi.PararnnError) as e:
        pk.pararnn_gru_solve(u, a)
    assert e.value.status == capi.ERR_UNSUPPORTED
    u = torch.zeros(1, 8, 3, 16, device=cuda)
    a = torch.zeros(3, 16, device=cuda)
    with pytest.raises(capi.PararnnError) as e:
        pk.pararnn_gru_solve(u, a, workspace=torch.empty(512, dtype=torch.uint8, device=cuda))
    assert e.value.status == capi.ERR_WORKSPACE
    with pytest.raises(capi.PararnnError) as e:
        pk.pararnn_gru_solve(u, a, tol=float("nan"))
    assert e.value.status == capi.ERR_INVALID_ARG
    with pytest.raises(capi.PararnnError):
        pk.pararnn_gru_solve(u, a, max_iters=-1)


@pytest.mark.parametrize("which", [0, 1])
def test_bounded_waits_time_out_without_hanging(cuda, which):
    from nonlinear_rnn_newton_b200 import capi
    ws = torch.zeros(16384, dtype=torch.uint8, device=cuda)
    st = P().pararnn_selftest_wait_timeout(which, 50_000_000, ws)  # 50 ms
    assert st == capi.ERR_TIMEOUT
    # the context is still usable afterwards
    w = W.custom("gru", 1, 64, 64, "bf16", h0_std=0.1)
    x = W.make_inputs(w, seed=0)
    h, it, r, st = run_gru(x, cuda)
    assert st == 0 and H.max_abs(h, oracle.gru_seq(x.u, x.a, x.h0)) <= TOL_STATE


def test_host_buffers_round_trip(cuda):
    w = W.custom("gru", 2, 300, 128, "bf16", h0_std=0.1)
    x = W.make_inputs(w, seed=18)
    h, it, r, st = P().pararnn_gru_solve(x.u.pin_memory(), x.a, x.h0)
    assert h.device.type == "cpu"
    assert H.max_abs(h.double().numpy(), oracle.gru_seq(x.u, x.a, x.h0)) <= TOL_STATE
