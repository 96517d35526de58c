"""GPU parity of the runtime-compiled solve for user-written cells, through the
C ABI, against the user-cell oracle (sequential stepping and serial Newton in
float64 on the same inputs).

Bounds: states max-abs <= 1e-4 against the sequential states (as for the
built-in cells); iterations equal to the oracle's Newton, or +-1 where its
residual at that step is within 10x of tol.  The GRU and LSTM written as user
cells also agree with the built-in kernels to 2e-5 (the user path evaluates
the cells with dual numbers and expf/tanhf, or with PARARNN_CELL_FAST_MATH the
hardware approximations; the built-in one with its own exp2/reciprocal
forms).  Every parity case runs in both modes."""
import numpy as np
import pytest
import torch

from oracle import generic as OG
from tests import helpers as H
from tests.user_cells import CELLS

pytestmark = pytest.mark.gpu

TOL_STATE = 1e-4


def P():
    import nonlinear_rnn_newton_b200 as pkg
    return pkg


@pytest.fixture(scope="module")
def compiled(cuda):
    """Every test cell, accurate (flags 0) and with the fast functions (1)."""
    return {(name, f): P().pararnn_cell_create(c.source, c.G, c.NS, f) for name, c in CELLS.items() for f in (0, 1)}


def draw(cell, B, L, D, dt, seed, s0_std=0.1):
    g = torch.Generator().manual_seed(seed)
    u = torch.randn((B, L, cell.G, D), generator=g)
    if dt == "bf16":
        u = u.to(torch.bfloat16)
    a = torch.rand((cell.G, D), generator=g) - 0.5
    s0 = torch.randn((cell.NS, B, D), generator=g) * s0_std
    return u, a, s0


SHAPES = [(2, 300, 136, "bf16"), (1, 1, 8, "bf16"), (3, 257, 64, "f32"), (4, 1500, 256, "bf16")]


@pytest.mark.parametrize("fast", [0, 1])
@pytest.mark.parametrize("name", sorted(CELLS))
@pytest.mark.parametrize("B,L,D,dt", SHAPES, ids=lambda v: str(v))
def test_user_cell_solve_matches_oracle(cuda, compiled, name, B, L, D, dt, fast):
    cell = CELLS[name]
    u, a, s0 = draw(cell, B, L, D, dt, seed=B * 7 + L)
    s, it, r, st = P().pararnn_cell_solve(compiled[name, fast], u.to(cuda), a.to(cuda), s0.to(cuda))
    torch.cuda.synchronize()
    seq = OG.generic_seq(cell.step, u, a, s0, cell.NS)
    err = H.max_abs(s.cpu(), seq)
    assert err <= TOL_STATE, f"max-abs error {err:.3e}"
    _, oit, ores, ost, hist = OG.generic_newton(cell.step, cell.jac, u, a, s0, cell.NS)
    assert H.iters_agree(it, oit, hist, 1e-6), (it, oit, hist)
    assert st == (0 if r <= 1e-6 else 1)


@pytest.mark.parametrize("fast", [0, 1])
@pytest.mark.parametrize("name", ["gru", "lstm"])
def test_user_gru_and_lstm_match_the_builtin_kernels(cuda, compiled, name, fast):
    cell = CELLS[name]
    B, L, D = 4, 2048, 512
    u, a, s0 = draw(cell, B, L, D, "bf16", seed=21)
    ud, ad = u.to(cuda), a.to(cuda)
    s, it, r, st = P().pararnn_cell_solve(compiled[name, fast], ud, ad, s0.to(cuda))
    if name == "gru":
        h, it2, r2, st2 = P().pararnn_gru_solve(ud, ad, s0[0].to(cuda))
        want = h[None]
    else:
        c, h, it2, r2, st2 = P().pararnn_lstm_solve(ud, ad, s0[0].to(cuda), s0[1].to(cuda))
        want = torch.stack([c, h])
    torch.cuda.synchronize()
    assert it == it2
    assert float((s - want).abs().max()) <= 2e-5


def test_tile_choice(cuda, compiled):
    """One-component cells get the 15-warp tile (their kernels fit in 128
    registers with few spills); two-component cells at most 7 (one CTA of 8
    warps), fewer when the ring does not fit (fp32 gates) or the kernel would
    spill a lot."""
    assert P().pararnn_cell_compute_warps(compiled["gru", 0], torch.bfloat16) == 15
    assert P().pararnn_cell_compute_warps(compiled["elman", 1], torch.float32) == 15
    assert P().pararnn_cell_compute_warps(compiled["lstm", 1], torch.bfloat16) == 7
    for f in (0, 1):
        for dt in (torch.bfloat16, torch.float32):
            assert 1 <= P().pararnn_cell_compute_warps(compiled["lstm", f], dt) <= 7


def test_bad_source_on_gpu(cuda):
    from nonlinear_rnn_newton_b200 import capi
    with pytest.raises(capi.PararnnError) as e:
        P().pararnn_cell_create("template <class T, class U> __device__ void recurrence_step(const T* s, const U* u, "
                                "const U* a, T* out) { out[0] = nothing; }", 1, 1)
    assert "nothing" in str(e.value)


def test_max_iters_and_tol_rules(cuda, compiled):
    """max_iters = 0 returns the zero guess with its residual; a huge tol stops
    at once; max_iters = 1 gives the oracle's first iterate."""
    cell = CELLS["mixed"]
    u, a, s0 = draw(cell, 2, 200, 64, "f32", seed=5)
    ud, ad, sd = u.to(cuda), a.to(cuda), s0.to(cuda)
    s, it, r, st = P().pararnn_cell_solve(compiled["mixed", 0], ud, ad, sd, max_iters=0)
    assert it == 0 and st == 1 and float(s.abs().max()) == 0.0
    H0, oit, ores, *_ = OG.generic_newton(cell.step, cell.jac, u, a, s0, 2, max_iters=0)
    assert abs(r - ores) <= 1e-5 * max(1.0, ores)
    s, it, r, st = P().pararnn_cell_solve(compiled["mixed", 0], ud, ad, sd, tol=1e30)
    assert it == 0 and st == 0
    s, it, r, st = P().pararnn_cell_solve(compiled["mixed", 0], ud, ad, sd, max_iters=1)
    H1, *_ = OG.generic_newton(cell.step, cell.jac, u, a, s0, 2, tol=0.0, max_iters=1)
    assert it == 1 and H.max_abs(s.cpu(), H1) <= TOL_STATE


@pytest.mark.parametrize("fast", [0, 1])
def test_partial_residuals_leave_a_user_cell_outcome_unchanged(cuda, compiled, fast):
    """A one-component user cell on enough tiles that passes which continue
    leave residuals out: the solve capped at its own iteration count (every
    pass evaluating the residual in full) gives the same states, count,
    residual and status."""
    cell = CELLS["gru"]
    u, a, s0 = draw(cell, 8, 2048, 512, "bf16", seed=9)
    ud, ad, sd = u.to(cuda), a.to(cuda), s0.to(cuda)
    s1, it1, r1, st1 = P().pararnn_cell_solve(compiled["gru", fast], ud, ad, sd, max_iters=10)
    assert st1 == 0 and it1 >= 3
    s2, it2, r2, st2 = P().pararnn_cell_solve(compiled["gru", fast], ud, ad, sd, max_iters=it1)
    assert (it2, st2, r2) == (it1, st1, r1)
    assert torch.equal(s1, s2)


ADJ_SHAPES = [(2, 300, 136, "bf16"), (3, 257, 64, "f32"), (1, 1, 8, "bf16")]


@pytest.mark.parametrize("fast", [0, 1])
@pytest.mark.parametrize("name", sorted(CELLS))
@pytest.mark.parametrize("B,L,D,dt", ADJ_SHAPES, ids=lambda v: str(v))
def test_user_cell_adjoint_matches_bptt(cuda, compiled, name, B, L, D, dt, fast):
    """Adjoint on the GPU solve's converged states against the oracle's BPTT
    (torch autograd in float64 through its own sequential states).  du and
    ds0 within 1e-4 * max(1, max|ref|); da within 1e-5 of sum_{b,l} |du| *
    max|s| (every test cell takes its weights as a * (a state value) inside
    a gate, so that bounds the sum of the absolute terms)."""
    cell = CELLS[name]
    u, a, s0 = draw(cell, B, L, D, dt, seed=3 * B + L)
    ds = torch.randn((cell.NS, B, L, D), generator=torch.Generator().manual_seed(L))
    ud, ad, sd = u.to(cuda), a.to(cuda), s0.to(cuda)
    h = compiled[name, fast]
    s, it, r, st = P().pararnn_cell_solve(h, ud, ad, sd, tol=1e-7, max_iters=20)
    du, da, ds0 = P().pararnn_cell_adjoint(h, ud, ad, sd, s, ds.to(cuda))
    torch.cuda.synchronize()
    rdu, rda, rds0 = OG.generic_bptt(cell.step, u, a, s0, ds, cell.NS)
    for x, ref in ((du, rdu), (ds0, rds0)):
        scale = max(1.0, float(np.max(np.abs(ref))))
        assert H.max_abs(x.cpu(), ref) <= 1e-4 * scale
    smax = max(1.0, float(s.abs().max()))
    bound = 1e-5 * np.sum(np.abs(rdu), axis=(0, 1)) * smax + 1e-6
    assert np.all(np.abs(da.cpu().numpy() - rda) <= bound)


def test_user_adjoints_match_the_builtin_ones(cuda, compiled):
    """The GRU and LSTM written as user cells give the built-in adjoints'
    gradients (to fp32 rounding of two different evaluation orders)."""
    for name in ("gru", "lstm"):
        cell = CELLS[name]
        u, a, s0 = draw(cell, 2, 1024, 256, "bf16", seed=77)
        ds = torch.randn((cell.NS, 2, 1024, 256), generator=torch.Generator().manual_seed(2)).to(cuda)
        ud, ad, sd = u.to(cuda), a.to(cuda), s0.to(cuda)
        s, *_ = P().pararnn_cell_solve(compiled[name, 0], ud, ad, sd, tol=1e-7, max_iters=20)
        du, da, ds0 = P().pararnn_cell_adjoint(compiled[name, 0], ud, ad, sd, s, ds)
        if name == "gru":
            bdu, bda, bdh0 = P().pararnn_gru_adjoint(ud, ad, sd[0], s[0], ds[0])
            bds0 = bdh0[None]
        else:
            bdu, bda, bdc0, bdh0 = P().pararnn_lstm_adjoint(ud, ad, sd[0], sd[1], s[0], s[1], ds[1], dc=ds[0])
            bds0 = torch.stack([bdc0, bdh0])
        torch.cuda.synchronize()
        for x, ref in ((du, bdu), (ds0, bds0)):
            scale = max(1.0, float(ref.abs().max()))
            assert float((x - ref).abs().max()) <= 2e-5 * scale, name
        smax = max(1.0, float(s.abs().max()))
        bound = 1e-5 * bdu.abs().sum(dim=(0, 1)) * smax + 1e-6
        assert bool(((da - bda).abs() <= bound).all()), name
