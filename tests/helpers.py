"""Shared helpers for the GPU parity tests: run the oracle on the same seeded
inputs (whole problem, or sampled channels of a full-size problem)."""
import numpy as np
import torch

import oracle


def f64(t):
    return None if t is None else t.detach().to("cpu").double()


def channel_slice(x, b, d):
    """Inputs of one (b, d) channel as a B=1, D=1 problem (exact widening)."""
    u = f64(x.u[b:b + 1, :, :, d:d + 1])
    a = f64(x.a[:, d:d + 1])
    h0 = None if x.h0 is None else f64(x.h0[b:b + 1, d:d + 1])
    c0 = None if x.c0 is None else f64(x.c0[b:b + 1, d:d + 1])
    return u, a, h0, c0


def sample_channels(B, D, n, seed=1234):
    g = np.random.default_rng(seed)
    picks = {(0, 0), (B - 1, D - 1)}
    while len(picks) < min(n, B * D):
        picks.add((int(g.integers(B)), int(g.integers(D))))
    return sorted(picks)


def max_abs(a, b):
    a = np.asarray(a, dtype=np.float64)
    b = np.asarray(b, dtype=np.float64)
    return float(np.max(np.abs(a - b))) if a.size else 0.0


def iters_agree(gpu_iters, ora_iters, ora_hist, tol):
    """GPU and oracle Newton iteration counts agree, or differ by one where
    the oracle's residual at the boundary step is within 10x of tol (fp32
    rounding can then decide the test either way)."""
    if gpu_iters == ora_iters:
        return True
    if abs(gpu_iters - ora_iters) != 1:
        return False
    k = min(gpu_iters, ora_iters)
    return k < len(ora_hist) and ora_hist[k] < 10 * tol


def gru_seq_channels(x, picks):
    out = {}
    for b, d in picks:
        u, a, h0, _ = channel_slice(x, b, d)
        out[(b, d)] = oracle.gru_seq(u, a, h0)[0, :, 0]
    return out


def lstm_seq_channels(x, picks):
    out = {}
    for b, d in picks:
        u, a, h0, c0 = channel_slice(x, b, d)
        c, h = oracle.lstm_seq(u, a, c0, h0)
        out[(b, d)] = (c[0, :, 0], h[0, :, 0])
    return out


def cuda_inputs(x, device):
    return x.to(device)


def torch_sync():
    torch.cuda.synchronize()
