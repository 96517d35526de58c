"""Write the regression fixtures in this folder.  Calls only ``oracle/`` and
the seeded input generator; run from the repository root:
    python tests/golden/make_golden.py
The pages print no worked numeric example for this method, so no fixture here
holds a page value; these fixtures lock the oracle's own results on the small
fp32 ParaGRU workload and on a small ParaLSTM case so that a later change to
the oracle's arithmetic shows up as a diff.
"""
import json
import os
import sys

HERE = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, os.path.dirname(os.path.dirname(HERE)))

import numpy as np  # noqa: E402

import oracle  # noqa: E402
from nonlinear_rnn_newton_b200 import workloads as W  # noqa: E402

SAMPLES = [(0, 0, 0), (0, 17, 5), (1, 100, 33), (1, 255, 63), (0, 128, 40)]


def main():
    out = {}
    w = W.GRU_SMALL
    x = W.make_inputs(w, seed=0)
    h, it, r, st, hist = oracle.gru_newton(x.u, x.a, x.h0, tol=w.tol, max_iters=w.max_iters)
    out[w.name] = {
        "source": "oracle.gru_newton, seed 0, tol 1e-6, max_iters 10",
        "iters": it, "status": st, "residual_history": [float(v) for v in hist],
        "samples": [[b, l, d, float(h[b, l, d])] for b, l, d in SAMPLES],
    }
    wl = W.custom("lstm", 2, 256, 64, "f32")
    x = W.make_inputs(wl, seed=0)
    c, h, it, r, st, hist = oracle.lstm_newton(x.u, x.a, None, None, tol=1e-6, max_iters=10)
    out[wl.name] = {
        "source": "oracle.lstm_newton, seed 0, tol 1e-6, max_iters 10",
        "iters": it, "status": st, "residual_history": [float(v) for v in hist],
        "samples": [[b, l, d, float(c[b, l, d]), float(h[b, l, d])] for b, l, d in SAMPLES],
    }
    with open(os.path.join(HERE, "oracle_small.json"), "w") as f:
        json.dump(out, f, indent=1)


if __name__ == "__main__":
    main()
