"""Newton solve with the sequence split into segments, one per GPU.

Page: "ParaRNN: Apple destrava treino paralelo de RNNs não-lineares e escala
pra 7B parâmetros" -- "A sacada: método de Newton".  Every Newton iteration
solves a linear recurrence; over one segment its solution is affine in the
state entering the segment.  Each GPU runs 1 + NS passes over its segment
(the state entering it set to 0 and to each unit vector), the segments' last
steps are gathered from every GPU (the one exchange of an iteration), every
GPU composes them in order into the state entering each segment, and a
fix-up gives the next iterate and its residual; the largest residual over
the GPUs takes the stopping decision.  The iterates are those of the
single-GPU solve, up to rounding.

This module is the host side only: buffers, the order of the library's
calls (all computation is in libpararnn's kernels) and the collectives.
`solve_segments` runs one segment per process under torch.distributed
(`DistComm`), or any number of segments one after another in one process
(`LocalComm`), which is how a one-GPU machine runs the same algorithm.
"""
import math

import torch

from . import capi

OK, NOT_CONVERGED, NONFINITE = capi.OK, capi.NOT_CONVERGED, capi.ERR_NONFINITE


class Segment:
    """One segment of every sequence: its gates and its slice of the iterate.

    u [B, Ls, G, D] (this segment's steps), a [G, D]; `index` is the
    segment's position along the sequence."""

    def __init__(self, cell, u, a, index, stream=None):
        if cell not in ("gru", "lstm"):
            raise ValueError(f"unknown cell {cell}")
        self.cell, self.u, self.a, self.index = cell, u, a, index
        self.NS = 1 if cell == "gru" else 2
        B, Ls, G, D = u.shape
        dev = u.device
        self.stream = stream if stream is not None else torch.cuda.current_stream(dev)
        f32 = dict(dtype=torch.float32, device=dev)
        self.H = torch.zeros((self.NS, B, Ls, D), **f32)          # iterate k on the segment
        self.P = torch.zeros((1 + self.NS, self.NS, B, Ls, D), **f32)  # passes: beta, unit_j
        self.ends = torch.empty((1 + self.NS, self.NS, B, D), **f32)
        self.lin = torch.zeros((self.NS, B, D), **f32)             # iterate k before the segment
        self.unit_carry = torch.zeros((self.NS, self.NS, B, D), **f32)
        for j in range(self.NS):
            self.unit_carry[j, j] = 1.0
        self.res = torch.zeros(1, **f32)
        size = capi.pararnn_gru_workspace_size if cell == "gru" else capi.pararnn_lstm_workspace_size
        self.ws = torch.empty(max(size(B, Ls, D), 256), dtype=torch.uint8, device=dev)

    def _pass(self, s_in, carry, out, end):
        fn = capi.pararnn_gru_segment_pass if self.cell == "gru" else capi.pararnn_lstm_segment_pass
        fn(self.u, self.a, s_in, self.lin, carry, out, end, self.ws, stream=self.stream)

    def _update(self, beta, unit, carry):
        fn = capi.pararnn_gru_segment_update if self.cell == "gru" else capi.pararnn_lstm_segment_update
        with torch.cuda.stream(self.stream):
            self.res.zero_()
        fn(self.u, self.a, beta, unit, carry, self.H, self.res, stream=self.stream)

    def start(self, s0):
        """The zero guess and its residual (the state before segment 0 is s0)."""
        with torch.cuda.stream(self.stream):
            self.H.zero_()
            self.P.zero_()
            self.lin.zero_()
            if self.index == 0 and s0 is not None:
                self.lin.copy_(s0)
        self._update(self.P[0], self.P[1:], self.lin)

    def passes(self, k):
        """The 1 + NS passes of iteration k from the iterate H (k = 0: the zero guess)."""
        s_in = None if k == 0 else self.H
        self._pass(s_in, None, self.P[0], self.ends[0])
        for j in range(self.NS):
            self._pass(s_in, self.unit_carry[j], self.P[1 + j], self.ends[1 + j])

    def carries(self, ends, s0):
        """The state entering every segment from all segments' ends [R, 1 + NS, NS, B, D]."""
        R, _, NS, B, D = ends.shape
        out = torch.empty((R, NS, B, D), dtype=torch.float32, device=ends.device)
        capi.pararnn_segment_carries(ends, s0, out, stream=self.stream)
        return out

    def update(self, carry):
        """Iterate k+1 = beta + A carry, its residual; carry is the new state before the segment."""
        self._update(self.P[0], self.P[1:], carry)
        with torch.cuda.stream(self.stream):
            self.lin.copy_(carry)


class LocalComm:
    """All segments in this process (a one-GPU stand-in for the collectives)."""

    def gather(self, ends_list):
        return torch.stack(ends_list)

    def max(self, res_list):
        vals = [float(r.item()) for r in res_list]
        return math.nan if any(v != v for v in vals) else max(vals)


class DistComm:
    """One segment per process, over torch.distributed (NCCL on GPUs, gloo on
    CPU); segment r lives on rank r."""

    def __init__(self, group=None):
        import torch.distributed as dist
        self.dist, self.group = dist, group
        self.world = dist.get_world_size(group)

    def gather(self, ends_list):
        (local,) = ends_list
        parts = [torch.empty_like(local) for _ in range(self.world)]
        self.dist.all_gather(parts, local.contiguous(), group=self.group)
        return torch.stack(parts)

    def max(self, res_list):
        (local,) = res_list
        t = local.clone()
        self.dist.all_reduce(t, op=self.dist.ReduceOp.MAX, group=self.group)
        return float(t.item())


def solve_segments(segments, comm, s0=None, tol=1e-6, max_iters=10, n_segments=None):
    """Newton solve over segments of the sequences.  `segments` are the
    segments this process holds (ordered by index), `n_segments` all of them
    (default: len(segments)); s0 [NS, B, D] or None on every process.
    Returns (iters, residual, status); each segment's states are in its H.
    Stopping rule as in the single-GPU solve: stop at the first iterate whose
    residual is <= tol, or after max_iters updates."""
    R = n_segments or len(segments)
    sg0 = segments[0]
    if any(sg.stream != sg0.stream for sg in segments):
        raise ValueError("the segments of one process share one stream")
    with torch.cuda.stream(sg0.stream):  # collectives and reads follow the segments' work
        return _solve(segments, comm, s0, tol, max_iters, R, sg0)


def _solve(segments, comm, s0, tol, max_iters, R, sg0):
    for sg in segments:
        sg.start(s0)
    r = comm.max([sg.res for sg in segments])
    if r != r or math.isinf(r):
        return 0, r, NONFINITE
    if r <= tol or max_iters == 0:
        return 0, r, (OK if r <= tol else NOT_CONVERGED)
    for k in range(max_iters):
        for sg in segments:
            sg.passes(k)
        ends = comm.gather([sg.ends for sg in segments])
        if ends.shape[0] != R:
            raise ValueError(f"gathered {ends.shape[0]} segment ends, expected {R}")
        carries = sg0.carries(ends, s0)
        for sg in segments:
            sg.update(carries[sg.index])
        r = comm.max([sg.res for sg in segments])
        if r != r or math.isinf(r):
            return k + 1, r, NONFINITE
        if r <= tol:
            return k + 1, r, OK
    return max_iters, r, NOT_CONVERGED
