"""Pins for the CPU oracle (no GPU).  Each test checks the oracle against
something other than itself: torch.nn.GRU / nn.LSTM in float64, torch
autograd, a dense linear solve of the whole Newton system, central finite
differences, and properties of Newton's method on a unit lower-bidiagonal
system (exact after k steps on the first k states; one step for a linear
recurrence).

Page: "ParaRNN: Apple destrava treino paralelo de RNNs não-lineares e escala
pra 7B parâmetros" -- "O compromisso que SSMs fizeram" (sequential
recurrence), "A sacada: método de Newton" (the whole sequence as one system
solved by Newton, each step a linear SSM), "Engenharia pra escalar" (diagonal
and 2x2 block-diagonal Jacobians).
"""
import math

import numpy as np
import pytest
import torch

import oracle
from tests import torch_cells as tc

f64 = torch.float64


def rnd(B, L, D, G, seed=0, a_scale=1.0, h0_std=0.1):
    g = torch.Generator().manual_seed(seed)
    u = torch.randn(B, L, G, D, generator=g, dtype=f64)
    a = (torch.rand(G, D, generator=g, dtype=f64) - 0.5) * a_scale
    h0 = torch.randn(B, D, generator=g, dtype=f64) * h0_std
    c0 = torch.randn(B, D, generator=g, dtype=f64) * h0_std
    return u, a, h0, c0


# ----------------------------------------------------------------- sequential

@pytest.mark.parametrize("B,L,D", [(1, 1, 1), (2, 37, 5), (3, 64, 8)])
def test_gru_seq_matches_torch_gru(B, L, D):
    u, a, h0, _ = rnd(B, L, D, 3, seed=B * 100 + L)
    h = oracle.gru_seq(u, a, h0)
    ref = tc.gru_run(u, a, h0).numpy()
    np.testing.assert_allclose(h, ref, rtol=0, atol=1e-13)


def test_gru_seq_h0_none_is_zero():
    u, a, _, _ = rnd(2, 9, 3, 3)
    np.testing.assert_array_equal(oracle.gru_seq(u, a, None),
                                  oracle.gru_seq(u, a, torch.zeros(2, 3, dtype=f64)))


@pytest.mark.parametrize("B,L,D", [(1, 1, 1), (2, 29, 4), (2, 50, 7)])
def test_lstm_seq_matches_torch_lstm(B, L, D):
    u, a, h0, c0 = rnd(B, L, D, 4, seed=7 + L)
    c, h = oracle.lstm_seq(u, a, c0, h0)
    # h from nn.LSTM (whole-sequence kernel) ...
    m = tc.lstm_module(a)
    with torch.no_grad():
        out, _ = m(u.reshape(B, L, 4 * D), (h0.reshape(1, B, D), c0.reshape(1, B, D)))
    np.testing.assert_allclose(h, out.numpy(), rtol=0, atol=1e-13)
    # ... and c from nn.LSTMCell stepped over L.
    cr, hr = tc.lstm_run(u, a, c0, h0)
    np.testing.assert_allclose(c, cr.numpy(), rtol=0, atol=1e-13)
    np.testing.assert_allclose(h, hr.numpy(), rtol=0, atol=1e-13)


def test_gru_seq_textbook_limits():
    # z -> 1 (u_z large): h_l = tanh(u_c + a_c r h_{l-1}) with a = 0 -> tanh(u_c).
    B, L, D = 1, 6, 3
    u, _, h0, _ = rnd(B, L, D, 3)
    a = torch.zeros(3, D, dtype=f64)
    u[:, :, 0] = 40.0
    h = oracle.gru_seq(u, a, h0)
    np.testing.assert_allclose(h, np.tanh(u[:, :, 2].numpy()), atol=1e-15)
    # z -> 0: the state is carried unchanged.
    u[:, :, 0] = -40.0
    h = oracle.gru_seq(u, a, h0)
    np.testing.assert_allclose(h, np.broadcast_to(h0.numpy()[:, None, :], h.shape), atol=1e-15)


# ---------------------------------------------------------------- Jacobians

def test_gru_cell_jacobian_matches_autograd_and_fd():
    g = torch.Generator().manual_seed(3)
    m_a = torch.rand(3, 1, generator=g, dtype=f64) - 0.5
    cell = tc.gru_cell_module(m_a)
    for _ in range(20):
        u3 = torch.randn(3, generator=g, dtype=f64) * 2
        h = float(torch.randn(1, generator=g, dtype=f64))
        f, A = oracle.gru_cell(h, u3, m_a[:, 0])
        ht = torch.tensor([[h]], dtype=f64, requires_grad=True)
        ft = cell(u3.reshape(1, 3), ht)
        (dA,) = torch.autograd.grad(ft.sum(), ht)
        assert abs(f - float(ft.detach())) < 1e-15
        assert abs(A - float(dA)) < 1e-14
        eps = 1e-6
        fp, _ = oracle.gru_cell(h + eps, u3, m_a[:, 0])
        fm, _ = oracle.gru_cell(h - eps, u3, m_a[:, 0])
        assert abs(A - (fp - fm) / (2 * eps)) < 1e-8


def test_lstm_cell_jacobian_matches_autograd():
    g = torch.Generator().manual_seed(4)
    a = torch.rand(4, 1, generator=g, dtype=f64) - 0.5
    cell = tc.lstm_cell_module(a)
    for _ in range(20):
        u4 = torch.randn(4, generator=g, dtype=f64) * 2
        c, h = [float(x) for x in torch.randn(2, generator=g, dtype=f64)]
        cn, hn, J = oracle.lstm_cell(c, h, u4, a[:, 0])

        def step(ch):
            hh, cc = cell(u4.reshape(1, 4), (ch[1].reshape(1, 1), ch[0].reshape(1, 1)))
            return torch.stack([cc.reshape(()), hh.reshape(())])

        x = torch.tensor([c, h], dtype=f64)
        out = step(x)
        Jt = torch.autograd.functional.jacobian(step, x)
        assert abs(cn - float(out[0])) < 1e-15 and abs(hn - float(out[1])) < 1e-15
        np.testing.assert_allclose(J, Jt.numpy(), atol=1e-14)


# --------------------------------------------------------------------- BPTT

def test_gru_bptt_matches_torch_autograd():
    B, L, D = 2, 23, 4
    u, a, h0, _ = rnd(B, L, D, 3, seed=11)
    gh = torch.randn(B, L, D, generator=torch.Generator().manual_seed(12), dtype=f64)
    du, da, dh0 = oracle.gru_bptt(u, a, h0, gh)
    m = tc.gru_module(a)
    x = u.reshape(B, L, 3 * D).clone().requires_grad_(True)
    hx = h0.reshape(1, B, D).clone().requires_grad_(True)
    out, _ = m(x, hx)
    (out * gh).sum().backward()
    np.testing.assert_allclose(du, x.grad.reshape(B, L, 3, D).numpy(), atol=1e-12)
    np.testing.assert_allclose(dh0, hx.grad.reshape(B, D).numpy(), atol=1e-12)
    np.testing.assert_allclose(da, tc.gru_da_from_grad(m, D).numpy(), atol=1e-11)


def test_lstm_bptt_matches_torch_autograd():
    B, L, D = 2, 19, 3
    u, a, h0, c0 = rnd(B, L, D, 4, seed=21)
    g = torch.Generator().manual_seed(22)
    gh = torch.randn(B, L, D, generator=g, dtype=f64)
    gc = torch.randn(B, L, D, generator=g, dtype=f64)
    du, da, dc0, dh0 = oracle.lstm_bptt(u, a, c0, h0, gh, gc)
    cell = tc.lstm_cell_module(a)
    x = u.clone().requires_grad_(True)
    h = h0.clone().requires_grad_(True)
    c = c0.clone().requires_grad_(True)
    hh, cc, loss = h, c, 0.0
    for l in range(L):
        hh, cc = cell(x[:, l].reshape(B, 4 * D), (hh, cc))
        loss = loss + (hh * gh[:, l]).sum() + (cc * gc[:, l]).sum()
    loss.backward()
    np.testing.assert_allclose(du, x.grad.numpy(), atol=1e-12)
    np.testing.assert_allclose(dh0, h.grad.numpy(), atol=1e-12)
    np.testing.assert_allclose(dc0, c.grad.numpy(), atol=1e-12)
    np.testing.assert_allclose(da, tc.lstm_da_from_grad(cell.weight_hh.grad, D).numpy(),
                               atol=1e-11)


def test_lstm_bptt_gc_none_equals_zero():
    B, L, D = 1, 7, 2
    u, a, h0, c0 = rnd(B, L, D, 4, seed=5)
    gh = torch.randn(B, L, D, dtype=f64, generator=torch.Generator().manual_seed(1))
    r1 = oracle.lstm_bptt(u, a, c0, h0, gh, None)
    r2 = oracle.lstm_bptt(u, a, c0, h0, gh, torch.zeros(B, L, D, dtype=f64))
    for x, y in zip(r1, r2):
        np.testing.assert_array_equal(x, y)


def _fd_grad(loss, x, eps=1e-6):
    g = np.zeros_like(x)
    it = np.nditer(x, flags=["multi_index"])
    for _ in it:
        i = it.multi_index
        old = x[i]
        x[i] = old + eps
        lp = loss(x)
        x[i] = old - eps
        lm = loss(x)
        x[i] = old
        g[i] = (lp - lm) / (2 * eps)
    return g


def test_gru_bptt_matches_finite_differences():
    B, L, D = 1, 9, 2
    u, a, h0, _ = rnd(B, L, D, 3, seed=31)
    gh = torch.randn(B, L, D, generator=torch.Generator().manual_seed(32), dtype=f64).numpy()
    un, an, h0n = u.numpy().copy(), a.numpy().copy(), h0.numpy().copy()
    du, da, dh0 = oracle.gru_bptt(un, an, h0n, gh)
    fu = _fd_grad(lambda x: float((oracle.gru_seq(x, an, h0n) * gh).sum()), un.copy())
    fa = _fd_grad(lambda x: float((oracle.gru_seq(un, x, h0n) * gh).sum()), an.copy())
    fh = _fd_grad(lambda x: float((oracle.gru_seq(un, an, x) * gh).sum()), h0n.copy())
    np.testing.assert_allclose(du, fu, atol=1e-8)
    np.testing.assert_allclose(da, fa, atol=1e-8)
    np.testing.assert_allclose(dh0, fh, atol=1e-8)


def test_lstm_bptt_matches_finite_differences():
    B, L, D = 1, 8, 2
    u, a, h0, c0 = rnd(B, L, D, 4, seed=41)
    gh = torch.randn(B, L, D, generator=torch.Generator().manual_seed(42), dtype=f64).numpy()
    un, an, h0n, c0n = u.numpy().copy(), a.numpy().copy(), h0.numpy().copy(), c0.numpy().copy()
    du, da, dc0, dh0 = oracle.lstm_bptt(un, an, c0n, h0n, gh, None)
    L_ = lambda uu, aa, cc, hh: float((oracle.lstm_seq(uu, aa, cc, hh)[1] * gh).sum())
    np.testing.assert_allclose(du, _fd_grad(lambda x: L_(x, an, c0n, h0n), un.copy()), atol=1e-8)
    np.testing.assert_allclose(da, _fd_grad(lambda x: L_(un, x, c0n, h0n), an.copy()), atol=1e-8)
    np.testing.assert_allclose(dc0, _fd_grad(lambda x: L_(un, an, x, h0n), c0n.copy()), atol=1e-8)
    np.testing.assert_allclose(dh0, _fd_grad(lambda x: L_(un, an, c0n, x), h0n.copy()), atol=1e-8)


# ------------------------------------------------------------------- Newton

def test_gru_newton_converges_to_sequential():
    u, a, h0, _ = rnd(2, 200, 6, 3, seed=51)
    h, it, r, st, hist = oracle.gru_newton(u, a, h0, tol=1e-12, max_iters=50)
    assert st == oracle.OK and r <= 1e-12
    np.testing.assert_allclose(h, tc.gru_run(u, a, h0).numpy(), atol=1e-12)
    assert len(hist) == it + 1 and hist[-1] == r


def test_lstm_newton_converges_to_sequential():
    u, a, h0, c0 = rnd(2, 150, 5, 4, seed=52)
    c, h, it, r, st, hist = oracle.lstm_newton(u, a, c0, h0, tol=1e-12, max_iters=50)
    assert st == oracle.OK and r <= 1e-12
    cr, hr = tc.lstm_run(u, a, c0, h0)
    np.testing.assert_allclose(c, cr.numpy(), atol=1e-12)
    np.testing.assert_allclose(h, hr.numpy(), atol=1e-12)


@pytest.mark.parametrize("k", [1, 2, 3, 5])
def test_gru_newton_first_k_states_exact(k):
    # Newton on a unit lower-bidiagonal system: after k updates from any guess
    # the first k states equal the sequential ones.
    u, a, h0, _ = rnd(2, 40, 4, 3, seed=60 + k)
    h, it, r, st, _ = oracle.gru_newton(u, a, h0, tol=0.0, max_iters=k)
    assert it == k and st == oracle.NOT_CONVERGED
    ref = tc.gru_run(u, a, h0).numpy()
    np.testing.assert_allclose(h[:, :k], ref[:, :k], atol=1e-14)
    if k == 1:  # the rest is not yet exact (later k may already be at rounding level)
        assert np.abs(h[:, k:] - ref[:, k:]).max() > 1e-6


@pytest.mark.parametrize("k", [1, 2, 4])
def test_lstm_newton_first_k_states_exact(k):
    u, a, h0, c0 = rnd(1, 30, 3, 4, seed=70 + k)
    c, h, it, r, st, _ = oracle.lstm_newton(u, a, c0, h0, tol=0.0, max_iters=k)
    assert it == k
    cr, hr = tc.lstm_run(u, a, c0, h0)
    np.testing.assert_allclose(c[:, :k], cr.numpy()[:, :k], atol=1e-14)
    np.testing.assert_allclose(h[:, :k], hr.numpy()[:, :k], atol=1e-14)


def test_newton_tiny_L_equals_brute_force():
    # L <= max_iters: the full solve equals stepping (brute force on tiny L).
    for L in (1, 2, 3, 4):
        u, a, h0, c0 = rnd(2, L, 3, 3, seed=80 + L)
        h, it, r, st, _ = oracle.gru_newton(u, a, h0, tol=0.0, max_iters=L)
        np.testing.assert_allclose(h, tc.gru_run(u, a, h0).numpy(), atol=1e-14)
        u4, a4, _, _ = rnd(2, L, 3, 4, seed=90 + L)
        c, h, it, r, st, _ = oracle.lstm_newton(u4, a4, c0, h0, tol=0.0, max_iters=L)
        cr, hr = tc.lstm_run(u4, a4, c0, h0)
        np.testing.assert_allclose(h, hr.numpy(), atol=1e-14)
        np.testing.assert_allclose(c, cr.numpy(), atol=1e-14)


def test_gru_zero_weights_one_iteration():
    # a = 0: the recurrence is linear in h, so Newton is exact after one update.
    u, _, h0, _ = rnd(2, 300, 8, 3, seed=90)
    a = torch.zeros(3, 8, dtype=f64)
    h, it, r, st, hist = oracle.gru_newton(u, a, h0, tol=1e-12, max_iters=10)
    assert st == oracle.OK and it == 1 and r < 1e-14
    np.testing.assert_allclose(h, tc.gru_run(u, a, h0).numpy(), atol=1e-14)


def test_lstm_zero_weights_two_iterations():
    # a = 0: c is linear (exact after one update) but h_l = o tanh(c_l) is not
    # linear in c_{l-1}, so the second update is needed and suffices.
    u, _, h0, c0 = rnd(2, 200, 6, 4, seed=91)
    a = torch.zeros(4, 6, dtype=f64)
    c, h, it, r, st, hist = oracle.lstm_newton(u, a, c0, h0, tol=1e-12, max_iters=10)
    assert st == oracle.OK and it == 2 and r < 1e-14


def _gru_F_torch(u, a, h0):
    """F(H) = H_l - GRUCell(u_l, H_{l-1}) for one batch row, via torch.nn.GRUCell."""
    cell = tc.gru_cell_module(a)
    L, G, D = u.shape

    def F(H):
        prev = torch.cat([h0.reshape(1, D), H[:-1]], 0)
        return H - cell(u.reshape(L, G * D), prev)
    return F


def test_gru_newton_step_equals_dense_solve():
    # One Newton update = H + solve(J_F(H), -F(H)), J_F from autograd of torch's
    # GRUCell and the dense solve from torch.linalg.
    L, D = 7, 2
    u, a, h0, _ = rnd(1, L, D, 3, seed=100)
    F = _gru_F_torch(u[0], a, h0[0])
    H = torch.zeros(L, D, dtype=f64)
    for k in (1, 2, 3):
        J = torch.autograd.functional.jacobian(F, H).reshape(L * D, L * D)
        H = H + torch.linalg.solve(J, -F(H).reshape(-1)).reshape(L, D)
        h, it, r, st, hist = oracle.gru_newton(u, a, h0, tol=0.0, max_iters=k)
        np.testing.assert_allclose(h[0], H.detach().numpy(), atol=1e-13)
        # reported residual = max |F| of the returned states
        assert abs(r - float(F(torch.from_numpy(h[0])).abs().max())) < 1e-15


def test_lstm_newton_step_equals_dense_solve():
    L, D = 6, 2
    u, a, h0, c0 = rnd(1, L, D, 4, seed=101)
    cell = tc.lstm_cell_module(a)

    def F(X):  # X [L, 2, D] = (c_l, h_l)
        cp = torch.cat([c0[0].reshape(1, D), X[:-1, 0]], 0)
        hp = torch.cat([h0[0].reshape(1, D), X[:-1, 1]], 0)
        hn, cn = cell(u[0].reshape(L, 4 * D), (hp, cp))
        return X - torch.stack([cn, hn], 1)

    X = torch.zeros(L, 2, D, dtype=f64)
    for k in (1, 2, 3):
        J = torch.autograd.functional.jacobian(F, X).reshape(2 * L * D, 2 * L * D)
        X = X + torch.linalg.solve(J, -F(X).reshape(-1)).reshape(L, 2, D)
        c, h, it, r, st, hist = oracle.lstm_newton(u, a, c0, h0, tol=0.0, max_iters=k)
        np.testing.assert_allclose(c[0], X[:, 0].detach().numpy(), atol=1e-13)
        np.testing.assert_allclose(h[0], X[:, 1].detach().numpy(), atol=1e-13)
        assert abs(r - float(F(torch.stack([torch.from_numpy(c[0]), torch.from_numpy(h[0])], 1))
                             .abs().max())) < 1e-15


def test_newton_converges_quadratically():
    u, a, h0, _ = rnd(2, 128, 8, 3, seed=110)
    _, it, r, st, hist = oracle.gru_newton(u, a, h0, tol=1e-14, max_iters=30)
    assert st == oracle.OK
    tail = [(x, y) for x, y in zip(hist[:-1], hist[1:]) if 1e-7 < x < 1e-2]
    assert tail, hist
    for x, y in tail:
        assert y <= 50.0 * x * x, hist


def test_newton_stopping_rule_and_status():
    u, a, h0, _ = rnd(2, 64, 4, 3, seed=120)
    # max_iters = 0 returns the initial guess H^0 = 0 and its residual r_0.
    h, it, r, st, hist = oracle.gru_newton(u, a, h0, tol=1e-6, max_iters=0)
    assert it == 0 and st == oracle.NOT_CONVERGED and np.all(h == 0)
    F0 = _gru_F_torch(u[0], a, h0[0])(torch.zeros(64, 4, dtype=f64)).abs().max()
    F1 = _gru_F_torch(u[1], a, h0[1])(torch.zeros(64, 4, dtype=f64)).abs().max()
    assert abs(r - max(float(F0), float(F1))) < 1e-15
    # a huge tolerance stops before any update
    h, it, r, st, hist = oracle.gru_newton(u, a, h0, tol=1e9, max_iters=5)
    assert it == 0 and st == oracle.OK
    # residual history is non-increasing once close
    _, it, r, st, hist = oracle.gru_newton(u, a, h0, tol=1e-10, max_iters=20)
    assert st == oracle.OK and it >= 2 and r <= 1e-10


def test_newton_nonfinite_input():
    u, a, h0, _ = rnd(1, 16, 3, 3, seed=130)
    u[0, 5, 1, 2] = float("nan")
    h, it, r, st, hist = oracle.gru_newton(u, a, h0)
    assert st == oracle.NONFINITE and math.isnan(r)
    # an infinite input to a saturating gate stays finite; an infinite state does not
    u, a, h0, _ = rnd(1, 16, 3, 3, seed=130)
    h0[0, 1] = float("inf")
    h, it, r, st, hist = oracle.gru_newton(u, a, h0)
    assert st == oracle.NONFINITE and it == 0 and r == float("inf")
    u4, a4, _, _ = rnd(1, 16, 3, 4, seed=131)
    u4[0, 3, 0, 0] = float("nan")
    c, h, it, r, st, hist = oracle.lstm_newton(u4, a4)
    assert st == oracle.NONFINITE and math.isnan(r)


def test_channel_and_batch_independence():
    u, a, h0, _ = rnd(3, 50, 6, 3, seed=140)
    pd = torch.randperm(6, generator=torch.Generator().manual_seed(1))
    pb = torch.tensor([2, 0, 1])
    h = oracle.gru_seq(u, a, h0)
    hp = oracle.gru_seq(u[pb][:, :, :, pd], a[:, pd], h0[pb][:, pd])
    np.testing.assert_array_equal(hp, h[pb.numpy()][:, :, pd.numpy()])
    hn, *_ = oracle.gru_newton(u, a, h0, tol=1e-12, max_iters=30)
    hnp, *_ = oracle.gru_newton(u[pb][:, :, :, pd], a[:, pd], h0[pb][:, pd], tol=1e-12, max_iters=30)
    np.testing.assert_allclose(hnp, hn[pb.numpy()][:, :, pd.numpy()], atol=1e-13)


def test_regression_fixture_unchanged():
    import json
    import os
    from nonlinear_rnn_newton_b200 import workloads as W
    fx = json.load(open(os.path.join(os.path.dirname(__file__), "golden", "oracle_small.json")))
    w = W.GRU_SMALL
    x = W.make_inputs(w, seed=0)
    h, it, r, st, hist = oracle.gru_newton(x.u, x.a, x.h0, tol=w.tol, max_iters=w.max_iters)
    g = fx[w.name]
    assert it == g["iters"] and st == g["status"]
    np.testing.assert_allclose(hist, g["residual_history"], rtol=1e-9, atol=1e-15)
    for b, l, d, v in g["samples"]:
        assert abs(h[b, l, d] - v) < 1e-13
    wl = W.custom("lstm", 2, 256, 64, "f32")
    x = W.make_inputs(wl, seed=0)
    c, h, it, r, st, hist = oracle.lstm_newton(x.u, x.a, None, None, tol=1e-6, max_iters=10)
    g = fx[wl.name]
    assert it == g["iters"] and st == g["status"]
    for b, l, d, vc, vh in g["samples"]:
        assert abs(c[b, l, d] - vc) < 1e-13 and abs(h[b, l, d] - vh) < 1e-13


# ------------------------------------------------------- input projection

def test_projection_matches_brute_force_sum():
    """oracle.project against the definition summed term by term in Python."""
    g = torch.Generator().manual_seed(11)
    B, L, Din, G, D = 2, 3, 5, 3, 2
    x = torch.randn((B, L, Din), generator=g, dtype=torch.float64)
    w = torch.randn((G, D, Din), generator=g, dtype=torch.float64)
    bias = torch.randn((G, D), generator=g, dtype=torch.float64)
    u = oracle.project(x, w, bias)
    for b in range(B):
        for l in range(L):
            for gg in range(G):
                for d in range(D):
                    ref = float(bias[gg, d])
                    for k in range(Din):
                        ref += float(x[b, l, k]) * float(w[gg, d, k])
                    assert abs(u[b, l, gg, d] - ref) < 1e-12


def test_projection_special_cases():
    """Identity weights give x + bias (the weight row g*D+d picks input g*D+d);
    zero input gives the bias."""
    g = torch.Generator().manual_seed(12)
    B, L, G, D = 2, 4, 3, 5
    x = torch.randn((B, L, G * D), generator=g, dtype=torch.float64)
    bias = torch.randn((G, D), generator=g, dtype=torch.float64)
    eye = torch.eye(G * D, dtype=torch.float64).reshape(G, D, G * D)
    u = oracle.project(x, eye, bias)
    np.testing.assert_allclose(u, (x.reshape(B, L, G, D) + bias).numpy(), rtol=0, atol=1e-15)
    z = oracle.project(torch.zeros((B, L, 7), dtype=torch.float64), torch.randn((G, D, 7), generator=g,
                                                                                dtype=torch.float64), bias)
    np.testing.assert_array_equal(z, np.broadcast_to(bias.numpy(), (B, L, G, D)))
