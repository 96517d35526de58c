"""The oracle's pins must catch plausible mistakes.

Each case plants one mistake (a dropped term, a wrong sign, a wrong index, a
transposed operand, a swapped gate) in a temporary copy of ``oracle/oracle.c``,
builds it, points the oracle wrapper at the broken library and runs the pin
tests of ``tests/test_oracle.py``: at least one of them must fail.  The
mistakes live only in the temporary copy, on the CPU.
"""
import ctypes
import inspect
import os
import subprocess

import pytest

import oracle
from tests import test_oracle as pins

SRC = os.path.join(os.path.dirname(oracle.__file__), "oracle.c")

MUTANTS = {
    "gru_jac_sign": ("dz * (c - h)", "dz * (h - c)"),
    "gru_jac_drop_reset_term": ("a[2] * (r + h * dr)", "a[2] * (r)"),
    "gru_candidate_drops_r": ("tanh(u[2] + a[2] * r * h)", "tanh(u[2] + a[2] * h)"),
    "gru_update_swapped": ("*f_out = (1.0 - z) * h + z * c;", "*f_out = z * h + (1.0 - z) * c;"),
    "lstm_jac_drop_term": ("double dcn_dh = df * c + di * g + i * dg;",
                           "double dcn_dh = df * c + di * g;"),
    "lstm_jac_transposed": ("J[1] = dcn_dh;\n        J[2] = o * (1.0 - t * t) * f;",
                            "J[2] = dcn_dh;\n        J[1] = o * (1.0 - t * t) * f;"),
    "lstm_gate_order": ("double o = logistic(u[2] + a[2] * h);\n    double g = tanh(u[3] + a[3] * h);",
                        "double o = logistic(u[3] + a[3] * h);\n    double g = tanh(u[2] + a[2] * h);"),
    "newton_rhs_sign": ("delta = A[idx] * delta - F[idx];", "delta = A[idx] * delta + F[idx];"),
    "newton_prev_index": (": H[(b * L + l - 1) * D + d];", ": H[(b * L + l) * D + d];"),
    "lstm_newton_transposed": ("double ndc = Jl[0] * dc + Jl[1] * dh - Fc[idx];",
                               "double ndc = Jl[0] * dc + Jl[2] * dh - Fc[idx];"),
    "residual_signed_max": ("else if (fabs(v) > r->m) r->m = fabs(v);", "else if (v > r->m) r->m = v;"),
    "seq_ignores_h0": ("double hp = h0 ? h0[b * D + d] : 0.0;\n            for (int64_t l = 0; l < L; ++l) {\n                gather_u(u, L, 3, D, b, l, d, ul);\n                oracle_gru_cell(hp, ul, ad, &f, NULL);",
                       "double hp = 0.0;\n            for (int64_t l = 0; l < L; ++l) {\n                gather_u(u, L, 3, D, b, l, d, ul);\n                oracle_gru_cell(hp, ul, ad, &f, NULL);"),
    "gru_bptt_drop_reset_path": ("g_r * ad[1] + g_c * ad[2] * r;", "g_r * ad[1];"),
    "gru_bptt_da_c_missing_r": ("sc += g_c * r * h;", "sc += g_c * h;"),
    "lstm_bptt_forget_carry": ("lc = gcn * f;", "lc = gcn;"),
    "lstm_bptt_wrong_operand": ("double g_f = gcn * cp * f * (1.0 - f);",
                                "double g_f = gcn * hp * f * (1.0 - f);"),
    "lstm_bptt_drop_tanh_path": ("double gcn = lc + lh * o * (1.0 - t * t);", "double gcn = lc;"),
}


def _pin_tests():
    out = []
    for name, fn in sorted(vars(pins).items()):
        if not name.startswith("test_") or not callable(fn):
            continue
        marks = getattr(fn, "pytestmark", [])
        args = {}
        for m in marks:
            if m.name == "parametrize":
                names = [n.strip() for n in m.args[0].split(",")]
                first = m.args[1][0]
                first = first if isinstance(first, tuple) else (first,)
                args.update(dict(zip(names, first)))
        if set(inspect.signature(fn).parameters) - set(args):
            continue
        out.append((name, fn, args))
    return out


@pytest.mark.parametrize("mutant", sorted(MUTANTS))
def test_pins_catch_mutant(mutant, tmp_path, monkeypatch):
    old, new = MUTANTS[mutant]
    src = open(SRC).read()
    assert src.count(old) >= 1, f"mutation site for {mutant} not found"
    path_c = tmp_path / "mutant.c"
    path_c.write_text(src.replace(old, new, 1))
    path_so = tmp_path / "libmutant.so"
    subprocess.run(["gcc", "-O1", "-fPIC", "-shared", "-fopenmp", "-ffp-contract=off",
                    str(path_c), "-o", str(path_so), "-lm"], check=True)
    monkeypatch.setattr(oracle, "_lib", oracle.configure(ctypes.CDLL(str(path_so))))
    caught = []
    for name, fn, args in _pin_tests():
        try:
            fn(**args)
        except AssertionError:
            caught.append(name)
            break
    assert caught, f"no pin caught mutant {mutant}"
