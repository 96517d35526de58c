"""The fixed-scratch ParaGRU solve (pararnn_gru_solve_noalloc).

It must give what the workspace entry point gives on the same inputs, on two
calls in a row (the second reuses the scratch the first left behind), and
reject a shape whose scratch need exceeds the fixed size before touching the
device.  This file is collected last so that the GPU case also runs after
every other test has used the device."""
import pytest
import torch

from nonlinear_rnn_newton_b200 import workloads as W

TOL_STATE = 1e-5  # both sides are the same kernels; only the look-back order may differ


@pytest.fixture(scope="module")
def capi():
    from nonlinear_rnn_newton_b200 import build
    build.build()
    from nonlinear_rnn_newton_b200 import capi
    return capi


def test_rejects_shape_beyond_fixed_scratch(capi):
    cap = capi.pararnn_gru_solve_noalloc_max_scratch()
    assert cap == 16 << 20
    B, L, D = 8, 4096, 1024
    assert capi.pararnn_gru_workspace_size(B, L, D) > cap
    # checked on the host before any device call: no GPU needed
    st = capi.lib.pararnn_gru_solve_noalloc(16, capi.BF16, 16, None, 16, B, L, D, 1e-6, 10, None, None, None)
    assert st == capi.ERR_WORKSPACE
    msg = capi.last_error()
    assert "fixed scratch" in msg and str(cap) in msg


@pytest.mark.gpu
def test_matches_workspace_entry_point_twice(capi, cuda):
    import nonlinear_rnn_newton_b200 as P
    w = W.custom("gru", 2, 2048, 512, "bf16", h0_std=0.1)
    assert P.pararnn_gru_workspace_size(w.B, w.L, w.D) <= P.pararnn_gru_solve_noalloc_max_scratch()
    x = W.make_inputs(w, seed=7).to(cuda)
    h_ref, it_ref, r_ref, st_ref = P.pararnn_gru_solve(x.u, x.a, x.h0, tol=w.tol, max_iters=w.max_iters)
    torch.cuda.synchronize()
    assert st_ref == capi.OK
    for _ in range(2):
        h = torch.full_like(h_ref, float("nan"))
        it, r, st = P.pararnn_gru_solve_noalloc(x.u, x.a, x.h0, h, tol=w.tol, max_iters=w.max_iters)
        torch.cuda.synchronize()
        assert st == capi.OK
        assert it == it_ref
        assert r <= w.tol
        assert float((h - h_ref).abs().max()) <= TOL_STATE
