"""GPU parity of the solve with the sequence split into segments (the
multi-GPU sequence sharding), run here as R segments one after another on one
GPU: the iterates are those of the single-GPU solve, so the states match it
(1e-5) and the oracle's sequential states (1e-4), and the iteration count is
the oracle's Newton count (+-1 where its residual is within 10x of tol)."""
import numpy as np
import pytest
import torch

import oracle
from nonlinear_rnn_newton_b200 import sharded as SH
from nonlinear_rnn_newton_b200 import workloads as W
from tests import helpers as H

pytestmark = pytest.mark.gpu


def P():
    import nonlinear_rnn_newton_b200 as pkg
    return pkg


SPLITS = [[1000], [500, 500], [1, 333, 666], [128, 256, 7, 409, 200]]


@pytest.mark.parametrize("cell", ["gru", "lstm"])
@pytest.mark.parametrize("lens", SPLITS, ids=lambda v: f"R{len(v)}")
@pytest.mark.parametrize("dt", ["bf16", "f32"])
def test_segments_match_single_gpu_and_oracle(cuda, cell, lens, dt):
    B, L, D = 3, sum(lens), 136
    w = W.custom(cell, B, L, D, dt, h0_std=0.1)
    x = W.make_inputs(w, seed=len(lens))
    xd = x.to(cuda)
    NS = 1 if cell == "gru" else 2
    s0 = torch.zeros((NS, B, D), device=cuda)
    if xd.h0 is not None:
        s0[NS - 1] = xd.h0
    edges = np.cumsum([0] + lens)
    segs = [SH.Segment(cell, xd.u[:, edges[r]:edges[r + 1]].contiguous(), xd.a, r) for r in range(len(lens))]
    it, res, st = SH.solve_segments(segs, SH.LocalComm(), s0, w.tol, w.max_iters)
    Hs = torch.cat([sg.H for sg in segs], dim=2)
    if cell == "gru":
        h, it1, r1, st1 = P().pararnn_gru_solve(xd.u, xd.a, xd.h0)
        one = h[None]
        seq = oracle.gru_seq(x.u, x.a, x.h0)[None]
        _, oit, _, _, hist = oracle.gru_newton(x.u, x.a, x.h0)
    else:
        c, h, it1, r1, st1 = P().pararnn_lstm_solve(xd.u, xd.a, None, xd.h0)
        one = torch.stack([c, h])
        sc, sh = oracle.lstm_seq(x.u, x.a, None, x.h0)
        seq = np.stack([sc, sh])
        *_, oit, _, _, hist = oracle.lstm_newton(x.u, x.a, None, x.h0)
    torch.cuda.synchronize()
    assert st == 0 and H.iters_agree(it, oit, hist, w.tol), (it, oit, hist)
    assert float((Hs - one).abs().max()) <= 1e-5
    assert H.max_abs(Hs.cpu(), seq) <= 1e-4


def test_long_segments_fold_longer_parts(cuda):
    """Segments longer than 64 * 256 steps fold 128 steps a part (and a short
    one 64): the split solve still matches the single-GPU solve and sampled
    oracle channels."""
    lens = [20000, 700]
    B, L, D = 1, sum(lens), 64
    w = W.custom("gru", B, L, D, "bf16", h0_std=0.1)
    x = W.make_inputs(w, seed=21)
    xd = x.to(cuda)
    s0 = xd.h0[None].contiguous()
    edges = np.cumsum([0] + lens)
    segs = [SH.Segment("gru", xd.u[:, edges[r]:edges[r + 1]].contiguous(), xd.a, r) for r in range(len(lens))]
    it, res, st = SH.solve_segments(segs, SH.LocalComm(), s0, w.tol, w.max_iters)
    Hs = torch.cat([sg.H for sg in segs], dim=2)[0]
    h, it1, r1, st1 = P().pararnn_gru_solve(xd.u, xd.a, xd.h0)
    torch.cuda.synchronize()
    assert st == 0 and st1 == 0 and abs(it - it1) <= 1, (it, it1)
    assert float((Hs - h).abs().max()) <= 1e-5
    picks = H.sample_channels(B, D, 6)
    ref = H.gru_seq_channels(x, picks)
    hc = Hs.cpu()
    for (b, d), v in ref.items():
        assert H.max_abs(hc[b, :, d].double().numpy(), v) <= 1e-4, (b, d)


def test_segment_stopping_rules(cuda):
    """max_iters = 0 and a huge tol stop at the zero guess; max_iters = 1
    gives the oracle's first iterate; each piece checks its arguments."""
    w = W.custom("gru", 2, 300, 64, "f32", h0_std=0.1)
    x = W.make_inputs(w, seed=3)
    xd = x.to(cuda)
    s0 = xd.h0[None].contiguous()
    segs = [SH.Segment("gru", xd.u[:, :100].contiguous(), xd.a, 0),
            SH.Segment("gru", xd.u[:, 100:].contiguous(), xd.a, 1)]
    it, r, st = SH.solve_segments(segs, SH.LocalComm(), s0, max_iters=0)
    h0, oit, ores, ost, hist = oracle.gru_newton(x.u, x.a, x.h0, max_iters=0)
    assert it == 0 and st == 1 and abs(r - ores) <= 1e-6 * max(1.0, ores)
    it, r, st = SH.solve_segments(segs, SH.LocalComm(), s0, tol=1e30)
    assert it == 0 and st == 0
    it, r, st = SH.solve_segments(segs, SH.LocalComm(), s0, tol=0.0, max_iters=1)
    h1, *_ = oracle.gru_newton(x.u, x.a, x.h0, tol=0.0, max_iters=1)
    Hs = torch.cat([sg.H for sg in segs], dim=2)[0]
    assert it == 1 and st == 1 and H.max_abs(Hs.cpu(), h1) <= 1e-4
    from nonlinear_rnn_newton_b200 import capi
    with pytest.raises(capi.PararnnError):  # output overlapping the iterate it reads, shifted by one row
        P().pararnn_gru_segment_pass(segs[0].u, xd.a, segs[0].H, None, None, segs[0].H.view(-1)[64:], None,
                                     segs[0].ws)


def test_segment_memory_is_the_iterate_plus_small_buffers(cuda):
    """A segment holds its iterate (updated in place), B*D-sized buffers, the
    fold's partial maps (one per 64 steps or more) and the fused pass's workspace:
    nothing else of the iterate's size."""
    B, Ls, D = 2, 1024, 256
    u = torch.zeros((B, Ls, 3, D), dtype=torch.bfloat16, device=cuda)
    a = torch.zeros((3, D), device=cuda)
    sg = SH.Segment("gru", u, a, 0)
    state = sg.H.numel() * 4
    extra = sg.rec.numel() * 4 + sg.carry.numel() * 4 + sg.lin.numel() * 4 + sg.res.numel() * 4
    assert sg.H.shape == (1, B, Ls, D) and extra <= 16 * B * D * 4
    assert sg.ws.numel() == max(P().pararnn_gru_workspace_size(B, Ls, D),
                                P().pararnn_segment_fold_workspace_size(1, B, Ls, D))
    assert P().pararnn_segment_fold_workspace_size(1, B, Ls, D) <= state // 32
