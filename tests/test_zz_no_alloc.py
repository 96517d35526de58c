"""The fixed-scratch ParaGRU solve (pararnn_gru_solve_noalloc).

It must give what the workspace entry point gives on the same inputs, on two
calls in a row (the second reuses the scratch the first left behind), match
the oracle's sequential states, and reject a bad call on the host before
touching the device: a shape whose scratch need exceeds the fixed size, a
shape the solve does not support, or tensors of the wrong shape.  This file
is collected last so that the GPU case also runs after every other test has
used the device."""
import numpy as np
import pytest
import torch

from nonlinear_rnn_newton_b200 import workloads as W

TOL_STATE = 1e-5   # both sides are the same kernels; only the look-back order may differ
TOL_ORACLE = 1e-4  # fp32 states against the fp64 oracle on the same inputs


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


def test_rejects_unsupported_shape_on_the_host(capi):
    # D = 12 needs no scratch beyond the limit (its size query says 0), but
    # the solve does not take it: refused before the scratch lookup, which
    # would be the first device call
    st = capi.lib.pararnn_gru_solve_noalloc(16, capi.BF16, 16, None, 16, 1, 8, 12, 1e-6, 10, None, None, None)
    assert st == capi.ERR_UNSUPPORTED
    assert "multiple of 8" in capi.last_error()
    st = capi.lib.pararnn_gru_solve_noalloc(16, capi.BF16, 16, None, 16, 0, 8, 16, 1e-6, 10, None, None, None)
    assert st == capi.ERR_INVALID_ARG


def test_binding_checks_tensor_shapes_before_the_call(capi):
    import nonlinear_rnn_newton_b200 as P
    u = torch.zeros((1, 8, 3, 16), dtype=torch.bfloat16)
    a = torch.zeros((3, 16))
    with pytest.raises(ValueError, match="h: expected shape"):
        P.pararnn_gru_solve_noalloc(u, a, None, torch.zeros((1, 7, 16)))
    with pytest.raises(ValueError, match="GRU gates"):
        P.pararnn_gru_solve_noalloc(torch.zeros((1, 8, 4, 16), dtype=torch.bfloat16), a, None,
                                    torch.zeros((1, 8, 16)))
    with pytest.raises(ValueError, match="a: expected shape"):
        P.pararnn_gru_solve_noalloc(u, torch.zeros((4, 16)), None, torch.zeros((1, 8, 16)))
    with pytest.raises(ValueError, match="contiguous"):
        P.pararnn_gru_solve_noalloc(u, a, None, torch.zeros((1, 16, 8)).transpose(1, 2))


@pytest.mark.gpu
def test_matches_workspace_entry_point_twice(capi, cuda):
    import oracle
    import nonlinear_rnn_newton_b200 as P
    w = W.custom("gru", 2, 2048, 512, "bf16", h0_std=0.1)
    assert P.pararnn_gru_workspace_size(w.B, w.L, w.D) <= P.pararnn_gru_solve_noalloc_max_scratch()
    x = W.make_inputs(w, seed=7)
    xd = x.to(cuda)
    h_ref, it_ref, r_ref, st_ref = P.pararnn_gru_solve(xd.u, xd.a, xd.h0, tol=w.tol, max_iters=w.max_iters)
    torch.cuda.synchronize()
    assert st_ref == capi.OK
    seq = oracle.gru_seq(x.u, x.a, x.h0)
    for _ in range(2):
        h = torch.full_like(h_ref, float("nan"))
        it, r, st = P.pararnn_gru_solve_noalloc(xd.u, xd.a, xd.h0, h, tol=w.tol, max_iters=w.max_iters)
        torch.cuda.synchronize()
        assert st == capi.OK
        assert it == it_ref
        assert r <= w.tol
        assert float((h - h_ref).abs().max()) <= TOL_STATE
        assert float(np.abs(h.cpu().double().numpy() - seq).max()) <= TOL_ORACLE
