"""GPU parity of the ParaGRU solve from the layer input (pararnn_gru_project_solve):
the input projection on the tensor cores with Newton pass 0 in the same kernel.

- u: against the float64 projection of the oracle, within the bf16 rounding
  of the result plus the fp32 accumulation bound of the sum;
- states: against the oracle's sequential stepping on the u the kernel wrote
  (the solve runs on those rounded values), max-abs 1e-4, with the oracle's
  Newton iteration count;
- against the plain solve of the same u (pass 0 scanned in different tiles:
  equal up to rounding, same iteration count).
Shapes cover several tiles of 128 steps and 64 channels, a ragged step tail,
a channel count and an input width that are not multiples of the tile, L = 1,
and h0 / bias present or absent."""
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


def check_projection(x, w, bias, u):
    ref = oracle.project(x, w, bias)
    mag = np.einsum("blk,gdk->blgd", np.abs(H.f64(x).numpy()), np.abs(H.f64(w).numpy()))
    got = u.cpu().double().numpy()
    # the fp32 sum of Din products is within acc = Din * 2^-24 * sum|x w| of
    # the exact value; bf16 keeps 8 significant bits, so rounding it to
    # nearest moves it by at most half a unit in the last place, at most
    # 2^-8 of its magnitude
    Din = x.shape[-1]
    acc = Din * 2.0 ** -24 * mag
    bound = 2.0 ** -8 * (np.abs(ref) + acc) + acc + 1e-30
    bad = np.abs(got - ref) > bound
    assert not bad.any(), (np.argwhere(bad)[:5], got[bad][:5], ref[bad][:5])


CASES = [  # B, L, Din, D, h0, bias
    (2, 300, 72, 136, True, True),
    (1, 1, 8, 64, True, False),
    (3, 1024, 256, 256, False, True),
    (2, 129, 64, 64, True, True),
]


@pytest.mark.parametrize("B,L,Din,D,with_h0,with_bias", CASES)
def test_project_solve_matches_oracle(cuda, B, L, Din, D, with_h0, with_bias):
    xi = W.make_projection_inputs(B, L, Din, D, seed=B * 1000 + L, h0_std=0.1 if with_h0 else 0.0,
                                  bias_std=0.1 if with_bias else 0.0)
    xd = xi.to(cuda)
    u, h, it, res, st = P().pararnn_gru_project_solve(xd.x, xd.w, xd.bias, xd.a, xd.h0)
    torch.cuda.synchronize()
    assert st == 0 and res <= 1e-6
    check_projection(xi.x, xi.w, xi.bias, u)
    uc = u.cpu()
    seq = oracle.gru_seq(uc, xi.a, xi.h0)
    assert H.max_abs(h.cpu(), seq) <= 1e-4
    _, oit, _, _, hist = oracle.gru_newton(uc, xi.a, xi.h0)
    assert H.iters_agree(it, oit, hist, 1e-6), (it, oit, hist)
    # the plain solve of the same gates
    h2, it2, r2, st2 = P().pararnn_gru_solve(u, xd.a, xd.h0)
    torch.cuda.synchronize()
    assert st2 == 0 and abs(it2 - it) <= 1
    assert float((h2 - h).abs().max()) <= 1e-5


def test_project_solve_stopping_rules(cuda):
    """max_iters = 0 returns the zero guess with its residual; max_iters = 1
    returns H^1 (the fused pass alone), equal to the oracle's first iterate."""
    B, L, Din, D = 2, 200, 64, 64
    xi = W.make_projection_inputs(B, L, Din, D, seed=5)
    xd = xi.to(cuda)
    u, h, it, res, st = P().pararnn_gru_project_solve(xd.x, xd.w, xd.bias, xd.a, xd.h0, max_iters=0)
    torch.cuda.synchronize()
    uc = u.cpu()
    h00, oit, ores, ost, _ = oracle.gru_newton(uc, xi.a, xi.h0, max_iters=0)
    assert it == 0 and st == 1 and abs(res - ores) <= 1e-5 * max(1.0, ores)
    assert float(h.abs().max()) == 0.0
    u, h, it, res, st = P().pararnn_gru_project_solve(xd.x, xd.w, xd.bias, xd.a, xd.h0, tol=0.0, max_iters=1)
    torch.cuda.synchronize()
    h1, oit, ores, ost, _ = oracle.gru_newton(u.cpu(), xi.a, xi.h0, tol=0.0, max_iters=1)
    assert it == 1 and st == 1 and H.max_abs(h.cpu(), h1) <= 1e-4
    assert abs(res - ores) <= 1e-4 * max(1.0, ores)


@pytest.mark.slow
def test_project_solve_fullsize_sampled(cuda):
    """The bench shape (B=8, L=4096, D=1024, Din=1024): u on sampled rows
    against the float64 projection, states on sampled channels against the
    oracle's stepping on the kernel's u."""
    B, L, Din, D = 8, 4096, 1024, 1024
    xi = W.make_projection_inputs(B, L, Din, D, seed=1)
    xd = xi.to(cuda)
    u, h, it, res, st = P().pararnn_gru_project_solve(xd.x, xd.w, xd.bias, xd.a, xd.h0)
    torch.cuda.synchronize()
    assert st == 0
    rows = [(0, 0), (3, 1234), (7, L - 1)]
    for b, l in rows:
        check_projection(xi.x[b:b + 1, l:l + 1], xi.w, xi.bias, u[b:b + 1, l:l + 1])
    uc = u.cpu()
    picks = H.sample_channels(B, D, 12)
    x = W.Inputs(u=uc, a=xi.a, h0=xi.h0)
    ref = H.gru_seq_channels(x, picks)
    hc = h.cpu()
    for (b, d), r in ref.items():
        assert H.max_abs(hc[b, :, d], r) <= 1e-4
