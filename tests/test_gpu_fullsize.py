"""Full-size parity on the benchmark workloads, through the same C-ABI entry
points and launch configuration the benchmark times.  The oracle steps
sampled (b, d) channels over the whole sequence (channels are independent),
and properties that hold at any size are checked on the whole output.
"""
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


@pytest.mark.parametrize("w", [W.GRU, W.GRU_SWEEP[0], W.GRU_SWEEP[2], W.GRU_SWEEP[4]], ids=lambda w: w.name)
def test_gru_fullsize_sampled(cuda, w):
    x = W.make_inputs(w, seed=0)
    xd = x.to(cuda)
    h, it, r, st = P().pararnn_gru_solve(xd.u, xd.a, xd.h0, tol=w.tol, max_iters=w.max_iters)
    torch.cuda.synchronize()
    assert st == 0 and r <= w.tol and 2 <= it <= w.max_iters
    assert bool(torch.isfinite(h).all())
    picks = H.sample_channels(w.B, w.D, 24)
    ref = H.gru_seq_channels(x, picks)
    hc = h.cpu()
    for (b, d), v in ref.items():
        assert H.max_abs(hc[b, :, d].double().numpy(), v) <= TOL_STATE, (b, d)
    del xd, h


@pytest.mark.parametrize("w", [W.GRU, W.GRU_SWEEP[4]], ids=lambda w: w.name)
def test_linear_scan_fullsize_sampled(cuda, w):
    """The plain linear scan (the zero-weight GRU) on the bench's inputs and
    launch: sampled channels against the oracle's stepping with a = 0."""
    x = W.make_inputs(w, seed=0)
    xd = x.to(cuda)
    h = P().pararnn_linear_scan(xd.u, xd.h0)
    torch.cuda.synchronize()
    assert bool(torch.isfinite(h).all())
    x0 = W.Inputs(u=x.u, a=torch.zeros_like(x.a), h0=x.h0)
    picks = H.sample_channels(w.B, w.D, 24)
    ref = H.gru_seq_channels(x0, picks)
    hc = h.cpu()
    for (b, d), v in ref.items():
        assert H.max_abs(hc[b, :, d].double().numpy(), v) <= TOL_STATE, (b, d)
    del xd, h


def test_lstm_fullsize_sampled(cuda):
    w = W.LSTM
    x = W.make_inputs(w, seed=0)
    xd = x.to(cuda)
    c, h, it, r, st = P().pararnn_lstm_solve(xd.u, xd.a, xd.c0, xd.h0, tol=w.tol, max_iters=w.max_iters)
    torch.cuda.synchronize()
    assert st == 0 and r <= w.tol
    picks = H.sample_channels(w.B, w.D, 24)
    ref = H.lstm_seq_channels(x, picks)
    cc, hc = c.cpu(), h.cpu()
    for (b, d), (vc, vh) in ref.items():
        assert H.max_abs(cc[b, :, d].double().numpy(), vc) <= TOL_STATE
        assert H.max_abs(hc[b, :, d].double().numpy(), vh) <= TOL_STATE


def test_lstm_training_step_fullsize_sampled(cuda):
    w = W.LSTM_TRAIN
    x = W.make_inputs(w, seed=0)
    xd = x.to(cuda)
    pk = P()
    c, h, it, r, st = pk.pararnn_lstm_solve(xd.u, xd.a, xd.c0, xd.h0, tol=w.tol, max_iters=w.max_iters)
    du, da, dc0, dh0 = pk.pararnn_lstm_adjoint(xd.u, xd.a, xd.c0, xd.h0, c, h, xd.dh)
    torch.cuda.synchronize()
    assert st == 0
    assert bool(torch.isfinite(du).all()) and bool(torch.isfinite(da).all())
    rng = np.random.default_rng(5)
    ds = sorted({0, w.D - 1, *[int(v) for v in rng.integers(0, w.D, 4)]})
    duc, dac = du.cpu(), da.cpu()
    for d in ds:
        # all batches of channel d (da sums over b and l)
        u = H.f64(x.u[:, :, :, d:d + 1])
        a = H.f64(x.a[:, d:d + 1])
        gh = H.f64(x.dh[:, :, d:d + 1])
        z = torch.zeros(w.B, 1, dtype=torch.float64)
        rdu, rda, rdc0, rdh0 = oracle.lstm_bptt(u, a, z, z, gh, None)
        scale = max(1.0, float(np.abs(rdu).max()))
        assert H.max_abs(duc[:, :, :, d].double().numpy(), rdu[:, :, :, 0]) <= 1e-4 * scale
        bound = 1e-5 * np.sum(np.abs(rdu[:, :, :, 0]), axis=(0, 1)) + 1e-6
        assert np.all(np.abs(dac[:, d].double().numpy() - rda[:, 0]) <= bound)


def test_gru_training_step_fullsize_sampled(cuda):
    w = W.GRU_TRAIN
    x = W.make_inputs(w, seed=0)
    xd = x.to(cuda)
    pk = P()
    h, it, r, st = pk.pararnn_gru_solve(xd.u, xd.a, xd.h0, tol=w.tol, max_iters=w.max_iters)
    du, da, dh0 = pk.pararnn_gru_adjoint(xd.u, xd.a, xd.h0, h, xd.dh)
    torch.cuda.synchronize()
    assert st == 0
    assert bool(torch.isfinite(du).all()) and bool(torch.isfinite(da).all())
    rng = np.random.default_rng(6)
    ds = sorted({0, w.D - 1, *[int(v) for v in rng.integers(0, w.D, 4)]})
    duc, dac, dh0c = du.cpu(), da.cpu(), dh0.cpu()
    for d in ds:
        # all batches of channel d (da sums over b and l)
        u = H.f64(x.u[:, :, :, d:d + 1])
        a = H.f64(x.a[:, d:d + 1])
        h0 = H.f64(x.h0[:, d:d + 1])
        gh = H.f64(x.dh[:, :, d:d + 1])
        rdu, rda, rdh0 = oracle.gru_bptt(u, a, h0, gh)
        scale = max(1.0, float(np.abs(rdu).max()))
        assert H.max_abs(duc[:, :, :, d].double().numpy(), rdu[:, :, :, 0]) <= 1e-4 * scale
        assert H.max_abs(dh0c[:, d].double().numpy(), rdh0[:, 0]) <= 1e-4 * scale
        bound = 1e-5 * np.sum(np.abs(rdu[:, :, :, 0]), axis=(0, 1)) + 1e-6
        assert np.all(np.abs(dac[:, d].double().numpy() - rda[:, 0]) <= bound)
