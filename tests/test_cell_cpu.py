"""The runtime-compiled cell path on the CPU: NVRTC compiles for sm_100a
without a device, so source errors, argument checks and the generated
kernels' resource use are checked here; loading the module needs a GPU."""
import ctypes

import pytest

from tests.user_cells import CELLS


@pytest.fixture(scope="module")
def capi():
    from nonlinear_rnn_newton_b200 import build
    build.build()
    from nonlinear_rnn_newton_b200 import capi
    return capi


def create(capi, src, G, NS, flags=0):
    h = ctypes.c_void_p()
    st = capi.lib.pararnn_cell_create(src.encode() if src is not None else None, G, NS, flags, ctypes.byref(h))
    return st, h


def test_argument_checks(capi):
    assert create(capi, None, 1, 1)[0] == capi.ERR_INVALID_ARG
    assert capi.lib.pararnn_cell_create(b"x", 1, 1, 0, None) == capi.ERR_INVALID_ARG
    assert create(capi, CELLS["elman"].source, 1, 1, flags=6)[0] == capi.ERR_INVALID_ARG
    assert capi.lib.pararnn_cell_compute_warps(None, 1) == 0
    assert create(capi, CELLS["elman"].source, 0, 1)[0] == capi.ERR_UNSUPPORTED
    assert create(capi, CELLS["elman"].source, 5, 1)[0] == capi.ERR_UNSUPPORTED
    assert create(capi, CELLS["elman"].source, 1, 3)[0] == capi.ERR_UNSUPPORTED
    assert capi.lib.pararnn_cell_workspace_size(None, 1, 1, 64, 64) == 0
    assert capi.lib.pararnn_cell_solve(None, 16, 1, 16, None, 16, 1, 8, 16, 1e-6, 10, 256, 1 << 20, None, None,
                                       None) == capi.ERR_INVALID_ARG
    capi.lib.pararnn_cell_destroy(None)  # no-op


def test_source_errors_are_reported_with_the_log(capi):
    bad = CELLS["elman"].source.replace("a[0] * s[0]", "a[0] * s_missing[0]")
    st, h = create(capi, bad, 1, 1)
    assert st == capi.ERR_INVALID_ARG and not h.value
    assert "s_missing" in capi.last_error()
    log = capi.lib.pararnn_cell_compile_log().decode()
    assert "s_missing" in log and "recurrence_step" in log  # located in the user's source


def test_a_step_without_the_template_signature_fails(capi):
    st, _ = create(capi, "__device__ void recurrence_step(const float* s, const float* u, const float* a, "
                         "float* out) { out[0] = s[0]; }", 1, 1)
    assert st == capi.ERR_INVALID_ARG
    # one number type for state and inputs is not enough either (the adjoint
    # differentiates through u and a)
    st, _ = create(capi, "template <class T> __device__ void recurrence_step(const T* s, const float* u, "
                         "const float* a, T* out) { out[0] = s[0] * a[0] + u[0]; }", 1, 1)
    assert st == capi.ERR_INVALID_ARG


@pytest.mark.parametrize("flags", [0, 1])
@pytest.mark.parametrize("name", sorted(CELLS))
def test_cells_compile(capi, name, flags):
    """Every test cell compiles, accurate and fast; without a GPU the module
    load then fails."""
    import torch
    cell = CELLS[name]
    st, h = create(capi, cell.source, cell.G, cell.NS, flags)
    if torch.cuda.is_available():
        assert st == capi.OK
        capi.lib.pararnn_cell_destroy(h)
    else:
        assert st == capi.ERR_CUDA, capi.last_error()


def _synthetic_step(G, NS):
    body = "\n".join(f"    acc = acc + tanh(u[{g}] + a[{g}] * s[{g % NS}]);" for g in range(G))
    outs = "\n".join(f"    out[{q}] = 0.5f * s[{q}] + 0.25f * sigmoid(acc + s[{(q + 1) % NS}]);" for q in range(NS))
    return ("template <class T, class U>\n__device__ void recurrence_step(const T* s, const U* u, const U* a, T* out)\n"
            "{\n    T acc = 0.0f;\n" + body + "\n" + outs + "\n}\n")


@pytest.mark.parametrize("G,NS", [(2, 1), (4, 1), (1, 2), (3, 2)])
def test_every_accepted_shape_compiles(capi, G, NS):
    """The shapes the test cells do not cover (those cover (3,1), (4,2), (1,1),
    (2,2)): the solve and adjoint instantiations compile and their tiles fit."""
    import torch
    st, h = create(capi, _synthetic_step(G, NS), G, NS)
    if torch.cuda.is_available():
        assert st == capi.OK, capi.last_error()
        capi.lib.pararnn_cell_destroy(h)
    else:
        assert st == capi.ERR_CUDA, capi.last_error()
