"""Pins of the user-cell oracle (oracle/generic.py) against things other than
itself: the C oracle on the same cells, torch.nn.RNN in float64, central
finite differences of the test cells' steps, a dense solve of the Newton
system, and the first-k-exact property of Newton on a recurrence."""
import numpy as np
import pytest
import torch

import oracle
from oracle import generic as OG
from nonlinear_rnn_newton_b200 import workloads as W
from tests.user_cells import CELLS


def inputs(cell, B, L, D, seed=0, h0_std=0.3):
    g = torch.Generator().manual_seed(seed)
    u = torch.randn((B, L, cell.G, D), generator=g, dtype=torch.float64)
    a = torch.rand((cell.G, D), generator=g, dtype=torch.float64) - 0.5
    s0 = torch.randn((cell.NS, B, D), generator=g, dtype=torch.float64) * h0_std
    return u.numpy(), a.numpy(), s0.numpy()


def test_seq_matches_c_oracle_gru_and_lstm():
    x = W.make_inputs(W.custom("gru", 3, 50, 24, "bf16", h0_std=0.1), seed=4)
    want = oracle.gru_seq(x.u, x.a, x.h0)
    got = OG.generic_seq(CELLS["gru"].step, x.u, x.a, x.h0.double().numpy()[None], 1)[0]
    assert np.max(np.abs(got - want)) < 1e-12
    x = W.make_inputs(W.custom("lstm", 2, 40, 16, "f32", h0_std=0.1), seed=5)
    wc, wh = oracle.lstm_seq(x.u, x.a, None, x.h0)
    s0 = np.stack([np.zeros((2, 16)), x.h0.double().numpy()])
    got = OG.generic_seq(CELLS["lstm"].step, x.u, x.a, s0, 2)
    assert np.max(np.abs(got[0] - wc)) < 1e-12 and np.max(np.abs(got[1] - wh)) < 1e-12


def test_seq_matches_torch_rnn_for_elman():
    cell = CELLS["elman"]
    u, a, s0 = inputs(cell, 2, 30, 8)
    rnn = torch.nn.RNN(8, 8, nonlinearity="tanh", bias=False, batch_first=True).double()
    with torch.no_grad():
        rnn.weight_ih_l0.copy_(torch.eye(8, dtype=torch.float64))
        rnn.weight_hh_l0.copy_(torch.diag(torch.from_numpy(a[0])))
        want, _ = rnn(torch.from_numpy(u[:, :, 0]), torch.from_numpy(s0))
    got = OG.generic_seq(cell.step, u, a, s0, 1)[0]
    assert np.max(np.abs(got - want.numpy())) < 1e-12


@pytest.mark.parametrize("name", sorted(CELLS))
def test_jacobians_match_finite_differences(name):
    cell = CELLS[name]
    g = np.random.default_rng(7)
    s = g.normal(size=(cell.NS, 3, 5)) * 0.7
    u = g.normal(size=(cell.G, 3, 5))
    a = g.uniform(-0.5, 0.5, size=(cell.G, 5))
    J = cell.jac(s, u, a)
    eps = 1e-6
    for r in range(cell.NS):
        sp, sm = s.copy(), s.copy()
        sp[r] += eps
        sm[r] -= eps
        fd = (cell.step(sp, u, a) - cell.step(sm, u, a)) / (2 * eps)
        assert np.max(np.abs(fd - J[:, r])) < 1e-8, (name, r)


def test_newton_matches_c_oracle_gru():
    x = W.make_inputs(W.custom("gru", 2, 64, 16, "bf16", h0_std=0.1), seed=8)
    h, it, r, st, hist = oracle.gru_newton(x.u, x.a, x.h0, tol=1e-6, max_iters=10)
    H, it2, r2, st2, hist2 = OG.generic_newton(CELLS["gru"].step, CELLS["gru"].jac, x.u, x.a,
                                               x.h0.double().numpy()[None], 1)
    assert it == it2 and st == st2
    assert np.allclose(hist, hist2, rtol=1e-9, atol=1e-15)
    assert np.max(np.abs(H[0] - h)) < 1e-12


def test_one_newton_step_is_the_dense_solve():
    """From H^0 = 0 one update solves J_F delta = -F(0), J_F the (L*NS) x
    (L*NS) unit block-lower-bidiagonal Jacobian of F(H)_l = H_l - f(H_{l-1})."""
    cell = CELLS["mixed"]
    L, ns = 6, 2
    u, a, s0 = inputs(cell, 1, L, 1, seed=3)
    H1, it, *_ = OG.generic_newton(cell.step, cell.jac, u, a, s0, ns, tol=0.0, max_iters=1)
    assert it == 1
    ug = np.transpose(u, (1, 2, 0, 3))
    H0 = np.zeros((ns, 1, L, 1))
    F = OG.residual(cell.step, ug, a, H0, s0)
    M = np.eye(L * ns)
    for l in range(1, L):
        J = cell.jac(H0[:, :, l - 1], ug[l], a)[:, :, 0, 0]
        M[l * ns:(l + 1) * ns, (l - 1) * ns:l * ns] = -J
    rhs = -np.transpose(F[:, 0, :, 0]).reshape(-1)
    delta = np.linalg.solve(M, rhs).reshape(L, ns).T
    assert np.max(np.abs(H1[:, 0, :, 0] - delta)) < 1e-12


@pytest.mark.parametrize("name", ["mixed", "lstm"])
def test_first_k_steps_exact_after_k_updates(name):
    cell = CELLS[name]
    u, a, s0 = inputs(cell, 2, 12, 3, seed=11)
    seq = OG.generic_seq(cell.step, u, a, s0, cell.NS)
    for k in (1, 2, 3):
        H, it, *_ = OG.generic_newton(cell.step, cell.jac, u, a, s0, cell.NS, tol=0.0, max_iters=k)
        assert it == k
        assert np.max(np.abs(H[:, :, :k] - seq[:, :, :k])) < 1e-12


@pytest.mark.parametrize("name", sorted(CELLS))
def test_newton_converges_to_the_sequential_states(name):
    cell = CELLS[name]
    u, a, s0 = inputs(cell, 2, 80, 5, seed=13)
    H, it, r, st, hist = OG.generic_newton(cell.step, cell.jac, u, a, s0, cell.NS, tol=1e-10, max_iters=30)
    assert st == OG.OK and r <= 1e-10
    assert np.max(np.abs(H - OG.generic_seq(cell.step, u, a, s0, cell.NS))) < 1e-9
    assert all(np.diff(hist[-3:]) < 0)  # fast final decrease


def test_bptt_matches_c_oracle_gru_and_lstm():
    x = W.make_inputs(W.custom("gru", 2, 30, 16, "bf16", h0_std=0.1), seed=9)
    g = torch.Generator().manual_seed(1)
    dh = torch.randn((2, 30, 16), generator=g, dtype=torch.float64)
    du, da, dh0 = oracle.gru_bptt(x.u, x.a, x.h0, dh)
    gdu, gda, gds0 = OG.generic_bptt(CELLS["gru"].step, x.u, x.a, x.h0.double().numpy()[None], dh.numpy()[None], 1)
    assert np.max(np.abs(gdu - du)) < 1e-12 and np.max(np.abs(gda - da)) < 1e-11
    assert np.max(np.abs(gds0[0] - dh0)) < 1e-12
    x = W.make_inputs(W.custom("lstm", 2, 25, 8, "f32", h0_std=0.1), seed=10)
    dh = torch.randn((2, 25, 8), generator=g, dtype=torch.float64)
    dc = torch.randn((2, 25, 8), generator=g, dtype=torch.float64)
    du, da, dc0, dh0 = oracle.lstm_bptt(x.u, x.a, None, x.h0, dh, dc)
    s0 = np.stack([np.zeros((2, 8)), x.h0.double().numpy()])
    gdu, gda, gds0 = OG.generic_bptt(CELLS["lstm"].step, x.u, x.a, s0, np.stack([dc.numpy(), dh.numpy()]), 2)
    assert np.max(np.abs(gdu - du)) < 1e-12 and np.max(np.abs(gda - da)) < 1e-11
    assert np.max(np.abs(gds0[0] - dc0)) < 1e-12 and np.max(np.abs(gds0[1] - dh0)) < 1e-12


@pytest.mark.parametrize("name", sorted(CELLS))
def test_bptt_matches_finite_differences(name):
    """d Loss / d u, d a, d s0 by central differences of the sequential
    states, on a tiny problem, for a few sampled entries."""
    cell = CELLS[name]
    B, L, D = 1, 6, 2
    u, a, s0 = inputs(cell, B, L, D, seed=17)
    ds = np.random.default_rng(3).normal(size=(cell.NS, B, L, D))
    du, da, ds0 = OG.generic_bptt(cell.step, u, a, s0, ds, cell.NS)
    loss = lambda uu, aa, ss: float(np.sum(ds * OG.generic_seq(cell.step, uu, aa, ss, cell.NS)))
    eps = 1e-6
    for idx in [(0, 0, 0, 0), (0, L - 1, cell.G - 1, 1), (0, 2, 0, 1)]:
        up, um = u.copy(), u.copy()
        up[idx] += eps
        um[idx] -= eps
        assert abs((loss(up, a, s0) - loss(um, a, s0)) / (2 * eps) - du[idx]) < 1e-7
    for idx in [(0, 0), (cell.G - 1, 1)]:
        ap, am = a.copy(), a.copy()
        ap[idx] += eps
        am[idx] -= eps
        assert abs((loss(u, ap, s0) - loss(u, am, s0)) / (2 * eps) - da[idx]) < 1e-7
    for idx in [(0, 0, 0), (cell.NS - 1, 0, 1)]:
        sp, sm = s0.copy(), s0.copy()
        sp[idx] += eps
        sm[idx] -= eps
        assert abs((loss(u, a, sp) - loss(u, a, sm)) / (2 * eps) - ds0[idx]) < 1e-7
