"""GPU parity of the decode step (one recurrence step for a batch) against the
CPU oracle's sequential stepping, through the C ABI.

One step from a given state is the oracle's stepping with L = 1 and that state
as the initial one.  Bounds: 1e-5 max-abs for one step (fp32 cell with the
hardware exp2 and reciprocal, inputs of order one), 1e-4 after a run of steps
(the same bound as the solves' states after L steps).
"""
import numpy as np
import pytest
import torch

import oracle
from nonlinear_rnn_newton_b200 import workloads as W
from tests import helpers as H

pytestmark = pytest.mark.gpu

TOL_STEP = 1e-5
TOL_RUN = 1e-4


def P():
    import nonlinear_rnn_newton_b200 as pkg
    return pkg


def state(B, D, seed, std=0.5):
    g = torch.Generator().manual_seed(seed)
    return torch.randn((B, D), generator=g, dtype=torch.float32) * std


CASES = [("gru", 8, 1024, "bf16"), ("gru", 3, 136, "f32"), ("gru", 1, 8, "bf16"),
         ("lstm", 8, 1024, "bf16"), ("lstm", 5, 264, "f32"), ("lstm", 1, 8, "bf16")]


@pytest.mark.parametrize("cell,B,D,dt", CASES, ids=lambda v: str(v))
def test_one_step_matches_oracle(cuda, cell, B, D, dt):
    x = W.make_inputs(W.custom(cell, B, 1, D, dt), seed=3)
    u = x.u[:, 0].contiguous()
    h = state(B, D, 4)
    if cell == "gru":
        got = P().pararnn_gru_step(u.to(cuda), x.a.to(cuda), h.to(cuda))
        want = oracle.gru_seq(x.u, x.a, h)[:, 0]
        assert H.max_abs(got.cpu(), want) <= TOL_STEP
    else:
        c = state(B, D, 5)
        gc, gh = P().pararnn_lstm_step(u.to(cuda), x.a.to(cuda), c.to(cuda), h.to(cuda))
        wc, wh = oracle.lstm_seq(x.u, x.a, c, h)
        assert H.max_abs(gc.cpu(), wc[:, 0]) <= TOL_STEP
        assert H.max_abs(gh.cpu(), wh[:, 0]) <= TOL_STEP


@pytest.mark.parametrize("cell", ["gru", "lstm"])
def test_zero_state_is_none(cuda, cell):
    x = W.make_inputs(W.custom(cell, 2, 1, 64, "bf16"), seed=7)
    u, a = x.u[:, 0].contiguous().to(cuda), x.a.to(cuda)
    z = torch.zeros((2, 64), device=cuda)
    if cell == "gru":
        assert torch.equal(P().pararnn_gru_step(u, a, None), P().pararnn_gru_step(u, a, z))
    else:
        c1, h1 = P().pararnn_lstm_step(u, a, None, None)
        c2, h2 = P().pararnn_lstm_step(u, a, z, z)
        assert torch.equal(c1, c2) and torch.equal(h1, h2)


@pytest.mark.parametrize("cell", ["gru", "lstm"])
def test_run_of_steps_in_place_matches_oracle_and_sequential_kernel(cuda, cell):
    """T steps updating the state in place give the oracle's states at every
    step, and the sequential kernel's states bit for bit (same cell code)."""
    B, T, D = 4, 96, 200
    x = W.make_inputs(W.custom(cell, B, T, D, "bf16", h0_std=0.1), seed=11)
    xd = x.to(cuda)
    h = (xd.h0.clone() if xd.h0 is not None else torch.zeros((B, D), device=cuda))
    c = torch.zeros((B, D), device=cuda)
    hs, cs = [], []
    steps = [xd.u[:, t].contiguous() for t in range(T)]
    for t in range(T):
        if cell == "gru":
            P().pararnn_gru_step(steps[t], xd.a, h, h)
        else:
            P().pararnn_lstm_step(steps[t], xd.a, c, h, c, h)
            cs.append(c.clone())
        hs.append(h.clone())
    hs = torch.stack(hs, 1).cpu()
    if cell == "gru":
        want = oracle.gru_seq(x.u, x.a, x.h0)
        seq = P().pararnn_gru_sequential(xd.u, xd.a, xd.h0).cpu()
    else:
        wc, want = oracle.lstm_seq(x.u, x.a, None, x.h0)
        sc, seq = P().pararnn_lstm_sequential(xd.u, xd.a, None, xd.h0)
        seq = seq.cpu()
        cs = torch.stack(cs, 1).cpu()
        assert H.max_abs(cs, wc) <= TOL_RUN
        assert torch.equal(cs, sc.cpu())
    assert H.max_abs(hs, want) <= TOL_RUN
    assert torch.equal(hs, seq)


def test_graph_of_steps(cuda):
    """A CUDA graph of T steps (the serving loop) replays the eager run."""
    B, T, D = 8, 32, 1024
    x = W.make_inputs(W.custom("gru", B, T, D, "bf16", h0_std=0.1), seed=2)
    xd = x.to(cuda)
    steps = [xd.u[:, t].contiguous() for t in range(T)]
    h_eager = xd.h0.clone()
    for t in range(T):
        P().pararnn_gru_step(steps[t], xd.a, h_eager, h_eager)
    h = xd.h0.clone()
    s = torch.cuda.Stream()
    s.wait_stream(torch.cuda.current_stream())
    g = torch.cuda.CUDAGraph()
    with torch.cuda.stream(s):
        P().pararnn_gru_step(steps[0], xd.a, h, h)  # warm up outside capture
        h.copy_(xd.h0)
        with torch.cuda.graph(g, stream=s):
            for t in range(T):
                P().pararnn_gru_step(steps[t], xd.a, h, h, stream=s)
    torch.cuda.current_stream().wait_stream(s)
    h.copy_(xd.h0)
    g.replay()
    torch.cuda.synchronize()
    assert torch.equal(h, h_eager)


def test_rejects_bad_arguments(cuda):
    from nonlinear_rnn_newton_b200 import capi
    u = torch.zeros((2, 3, 12), device=cuda)
    with pytest.raises(capi.PararnnError):
        P().pararnn_gru_step(u, torch.zeros((3, 12), device=cuda))  # D not a multiple of 8
    h = torch.zeros((2 * 64 + 8,), device=cuda)
    u = torch.zeros((2, 3, 64), device=cuda)
    with pytest.raises(capi.PararnnError):
        P().pararnn_gru_step(u, torch.zeros((3, 64), device=cuda), h[:128].view(2, 64), h[4:132].view(2, 64))
