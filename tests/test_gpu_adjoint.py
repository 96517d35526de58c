"""GPU parity of the adjoint (reverse-time scan) against the oracle's BPTT.

The adjoint runs on the GPU solve's converged fp32 states; the oracle
backpropagates through its own fp64 sequential states.  Bounds: du and the
initial-state gradients within 1e-4 * max(1, max|ref|) (the fp32 states agree
to ~1e-6 and the reverse recurrence contracts); da, a sum of B*L terms per
channel, within 1e-5 of the sum of the absolute values of its terms.
"""
import numpy as np
import pytest
import torch

import oracle
from nonlinear_rnn_newton_b200 import workloads as W
from tests import helpers as H

pytestmark = pytest.mark.gpu


def P():
    import nonlinear_rnn_newton_b200 as pkg
    return pkg


def close_scaled(x, ref, rel=1e-4):
    scale = max(1.0, float(np.max(np.abs(ref))))
    err = H.max_abs(x, ref)
    assert err <= rel * scale, f"max-abs {err:.3e} vs scale {scale:.3e}"


def da_bound(du_ref, h_prev_abs_max=1.0):
    # sum over b, l of |term|, bounded using |d pre / d a| <= max |state|
    return np.sum(np.abs(du_ref), axis=(0, 1)) * h_prev_abs_max


GRU_ADJ = [
    W.custom("gru", 2, 256, 64, "f32", h0_std=0.1, train=True),
    W.custom("gru", 3, 333, 200, "bf16", h0_std=0.1, train=True),
    W.custom("gru", 1, 1, 8, "bf16", h0_std=0.1, train=True),
    W.custom("gru", 2, 1000, 136, "bf16", h0_std=0.1, train=True),
]


@pytest.mark.parametrize("w", GRU_ADJ, ids=lambda w: w.name)
def test_gru_adjoint_matches_bptt(cuda, w):
    x = W.make_inputs(w, seed=0)
    xd = x.to(cuda)
    pk = P()
    h, it, r, st = pk.pararnn_gru_solve(xd.u, xd.a, xd.h0, tol=1e-7, max_iters=20)
    du, da, dh0 = pk.pararnn_gru_adjoint(xd.u, xd.a, xd.h0, h, xd.dh)
    torch.cuda.synchronize()
    h0 = x.h0 if x.h0 is not None else torch.zeros(w.B, w.D)
    rdu, rda, rdh0 = oracle.gru_bptt(x.u, x.a, h0, x.dh)
    close_scaled(du.cpu().numpy(), rdu)
    close_scaled(dh0.cpu().numpy(), rdh0)
    hmax = max(1.0, float(np.abs(h.cpu().numpy()).max()))
    bound = 1e-5 * da_bound(rdu, hmax) + 1e-6
    assert np.all(np.abs(da.cpu().numpy() - rda) <= bound)


LSTM_ADJ = [
    W.custom("lstm", 2, 256, 64, "f32", train=True),
    W.custom("lstm", 3, 300, 136, "bf16", train=True),
    W.custom("lstm", 1, 1, 8, "bf16", train=True),
    W.custom("lstm", 2, 1000, 128, "bf16", train=True),
]


@pytest.mark.parametrize("with_dc", [False, True])
@pytest.mark.parametrize("w", LSTM_ADJ, ids=lambda w: w.name)
def test_lstm_adjoint_matches_bptt(cuda, w, with_dc):
    x = W.make_inputs(w, seed=1)
    g = torch.Generator().manual_seed(77)
    dc = torch.randn(w.B, w.L, w.D, generator=g) if with_dc else None
    xd = x.to(cuda)
    pk = P()
    c, h, it, r, st = pk.pararnn_lstm_solve(xd.u, xd.a, xd.c0, xd.h0, tol=1e-7, max_iters=20)
    du, da, dc0, dh0 = pk.pararnn_lstm_adjoint(xd.u, xd.a, xd.c0, xd.h0, c, h, xd.dh,
                                               dc=None if dc is None else dc.to(cuda))
    torch.cuda.synchronize()
    z = torch.zeros(w.B, w.D)
    rdu, rda, rdc0, rdh0 = oracle.lstm_bptt(x.u, x.a, z, z, x.dh, dc)
    close_scaled(du.cpu().numpy(), rdu)
    close_scaled(dc0.cpu().numpy(), rdc0)
    close_scaled(dh0.cpu().numpy(), rdh0)
    bound = 1e-5 * da_bound(rdu) + 1e-6
    assert np.all(np.abs(da.cpu().numpy() - rda) <= bound)


def test_adjoint_is_deterministic(cuda):
    w = W.custom("lstm", 4, 1024, 256, "bf16", train=True)
    x = W.make_inputs(w, seed=2).to(cuda)
    pk = P()
    c, h, *_ = pk.pararnn_lstm_solve(x.u, x.a, x.c0, x.h0)
    r1 = pk.pararnn_lstm_adjoint(x.u, x.a, x.c0, x.h0, c, h, x.dh)
    r2 = pk.pararnn_lstm_adjoint(x.u, x.a, x.c0, x.h0, c, h, x.dh)
    torch.cuda.synchronize()
    for a, b in zip(r1, r2):
        assert torch.equal(a, b)


def test_gru_zero_weights_adjoint_is_reverse_linear_recurrence(cuda):
    # a = 0: lambda_l = dh_l + (1 - z_{l+1}) lambda_{l+1}, du_c = lambda z (1 - c^2)
    w = W.custom("gru", 2, 500, 64, "f32", h0_std=0.1, train=True)
    x = W.make_inputs(w, seed=3, a_scale=0.0)
    xd = x.to(cuda)
    pk = P()
    h, *_ = pk.pararnn_gru_solve(xd.u, xd.a, xd.h0)
    du, da, dh0 = pk.pararnn_gru_adjoint(xd.u, xd.a, xd.h0, h, xd.dh)
    torch.cuda.synchronize()
    u = x.u.double().numpy()
    z = 1 / (1 + np.exp(-u[:, :, 0]))
    c = np.tanh(u[:, :, 2])
    lam = np.zeros((w.B, w.D))
    ref = np.zeros((w.B, w.L, w.D))
    for l in range(w.L - 1, -1, -1):
        lam = x.dh[:, l].double().numpy() + (lam * (1 - z[:, l + 1]) if l + 1 < w.L else 0)
        ref[:, l] = lam * z[:, l] * (1 - c[:, l] ** 2)
    close_scaled(du[:, :, 2].cpu().numpy(), ref)
