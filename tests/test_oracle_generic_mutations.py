"""The user-cell oracle's pins must catch plausible mistakes.

Each case plants one mistake (a dropped initial state, an off-by-one in the
state before a step, a wrong sign, a transposed Jacobian, a signed residual,
an off-by-one in the stopping rule, a gradient path cut) in a copy of
``oracle/generic.py``, loaded as a separate module, and runs every pin of
``tests/test_oracle_generic.py`` (all parameter sets) against it: at least
one must fail.  The mistakes live only in the copy, on the CPU.
"""
import os
import types

import pytest

from oracle import generic as OG
from tests import test_oracle_generic as pins

SRC = open(os.path.join(os.path.dirname(OG.__file__), "generic.py")).read()

MUTANTS = {
    "seq_ignores_s0": ("s = np.zeros((ns, B, D)) if s0 is None else _f64(s0).reshape(ns, B, D).copy()",
                       "s = np.zeros((ns, B, D))"),
    "seq_output_shifted": ("        out[:, :, l] = s\n", "        out[:, :, l - 1] = s\n"),
    "prev_ignores_s0": ("    P[:, :, 0] = s0\n", "    P[:, :, 0] = 0.0\n"),
    "prev_off_by_one": ("    P[:, :, 1:] = H[:, :, :-1]\n", "    P[:, :, 1:] = H[:, :, 1:]\n"),
    "newton_rhs_sign": ('delta = np.einsum("qrbd,rbd->qbd", J, delta) - F[:, :, l]',
                        'delta = np.einsum("qrbd,rbd->qbd", J, delta) + F[:, :, l]'),
    "newton_jacobian_transposed": ('delta = np.einsum("qrbd,rbd->qbd", J, delta) - F[:, :, l]',
                                   'delta = np.einsum("rqbd,rbd->qbd", J, delta) - F[:, :, l]'),
    "residual_signed": ("r = float(np.max(np.abs(F))) if F.size else 0.0",
                        "r = float(np.max(F)) if F.size else 0.0"),
    "stopping_off_by_one": ("if r <= tol or k == max_iters:", "if r <= tol or k == max_iters + 1:"),
    "bptt_loss_detached": ("loss = loss + (dst[:, :, l] * s).sum()", "loss = loss + (dst[:, :, l] * s.detach()).sum()"),
    "bptt_wrong_upstream_step": ("loss = loss + (dst[:, :, l] * s).sum()",
                                 "loss = loss + (dst[:, :, max(l - 1, 0)] * s).sum()"),
}


def _load(src):
    mod = types.ModuleType("generic_mutant")
    exec(compile(src, "generic_mutant", "exec"), mod.__dict__)
    return mod


def _pin_calls():
    """(name, function, kwargs) for every pin and every parameter set."""
    out = []
    for name, fn in sorted(vars(pins).items()):
        if not name.startswith("test_") or not callable(fn):
            continue
        sets = [{}]
        for m in getattr(fn, "pytestmark", []):
            if m.name != "parametrize":
                continue
            names = [n.strip() for n in m.args[0].split(",")]
            vals = [v if isinstance(v, tuple) else (v,) for v in m.args[1]]
            sets = [dict(s, **dict(zip(names, v))) for s in sets for v in vals]
        out += [(name, fn, kw) for kw in sets]
    return out


def test_unmutated_oracle_passes_every_pin():
    for name, fn, kw in _pin_calls():
        fn(**kw)


@pytest.mark.parametrize("mutant", sorted(MUTANTS))
def test_pins_catch_the_mistake(mutant, monkeypatch):
    a, b = MUTANTS[mutant]
    assert SRC.count(a) == 1, mutant
    monkeypatch.setattr(pins, "OG", _load(SRC.replace(a, b)))
    caught = []
    for name, fn, kw in _pin_calls():
        try:
            fn(**kw)
        except Exception:  # an assertion, or a crash the mistake causes
            caught.append(name)
    assert caught, f"no pin catches {mutant}"
