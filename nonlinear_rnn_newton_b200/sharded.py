"""Newton solve with the sequence split into segments, one per GPU.

Page: "ParaRNN: Apple destrava treino paralelo de RNNs não-lineares e escala
pra 7B parâmetros" -- "A sacada: método de Newton".  Every Newton iteration
solves a linear recurrence s^{k+1}_l = J_l s^{k+1}_{l-1} + o_l whose step
maps depend only on the iterate H^k; over a segment they compose into one
affine map of the state entering the segment.  Per iteration each GPU folds
its segment's maps into a record (one pass that reads the segment once and
writes B*D-sized fields only), the records are all-gathered (the one data
exchange), every GPU composes them in order into the state entering its own
segment, and one fused pass in segment mode writes the next iterate in place
with its residual; the largest residual over the GPUs (an all-reduce of one
float) takes the stopping decision.  The iterates are those of the
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
    segment's position along the sequence.  Device memory beyond the iterate
    H is O(B*D) plus the fold's partial maps (1/128 of a state array per map
    entry) and the fused pass's workspace."""

    def __init__(self, cell, u, a, index, stream=None):
        if cell not in ("gru", "lstm"):
            raise ValueError(f"unknown cell {cell}")
        self.cell, self.u, self.a, self.index = cell, u, a, index
        self.NS = 1 if cell == "gru" else 2
        B, Ls, G, D = u.shape
        dev = u.device
        self.stream = stream if stream is not None else torch.cuda.current_stream(dev)
        f32 = dict(dtype=torch.float32, device=dev)
        self.H = torch.zeros((self.NS, B, Ls, D), **f32)          # iterate k on the segment, updated in place
        self.rec = torch.empty(capi.pararnn_segment_record_floats(self.NS, B, D), **f32)
        self.carry = torch.zeros((self.NS, B, D), **f32)           # new state entering the segment
        self.lin = torch.zeros((self.NS, B, D), **f32)             # iterate k before the segment
        self.res = torch.zeros(4, **f32)
        size = capi.pararnn_gru_workspace_size if cell == "gru" else capi.pararnn_lstm_workspace_size
        nbytes = max(size(B, Ls, D), capi.pararnn_segment_fold_workspace_size(self.NS, B, Ls, D), 256)
        self.ws = torch.empty(nbytes, dtype=torch.uint8, device=dev)
        pre = "pararnn_gru_" if cell == "gru" else "pararnn_lstm_"
        self._fold = getattr(capi, pre + "segment_fold")
        self._combine = getattr(capi, pre + "segment_combine")
        self._pass = getattr(capi, pre + "segment_pass")

    def start(self, s0):
        """The zero guess H^0 = 0."""
        with torch.cuda.stream(self.stream):
            self.H.zero_()

    def fold(self, k):
        """This segment's record of iteration k (k = 0: from the zero guess)."""
        self._fold(self.u, self.a, None if k == 0 else self.H, self.rec, self.ws, stream=self.stream)

    def combine(self, records, s0):
        """From every segment's record [R, record_floats]: this segment's carry
        and linearisation point; returns max |F(H^k)| over all segments (a
        one-float device tensor, the same on every process)."""
        self._combine(records, self.index, self.a, s0, self.carry, self.lin, self.res, stream=self.stream)
        return self.res[:1]

    def apply(self, k):
        """H^{k+1} on the segment, in place."""
        self._pass(self.u, self.a, None if k == 0 else self.H, self.lin, self.carry, self.H, None, self.ws,
                   stream=self.stream)

    def pass_outcome(self):
        """[max |F(H^{k+1})| over this segment, device-side error flag] as a
        device tensor (after apply; no synchronisation)."""
        out = torch.empty(2, dtype=torch.float32, device=self.H.device)
        capi.pararnn_result_to_device(self.ws, out, stream=self.stream)
        return out


class LocalComm:
    """All segments in this process (a one-GPU stand-in for the collectives)."""

    def gather(self, recs):
        return torch.stack(recs)

    def max(self, vals):
        """Element-wise maximum of equal-shaped tensors, NaN kept, read once."""
        t = torch.stack(vals)
        m = t.max(dim=0).values if t.shape[0] > 1 else t[0]
        return m.tolist()


class DistComm:
    """One segment per process, over torch.distributed (NCCL on GPUs, gloo on
    CPU); segment r lives on rank r."""

    def __init__(self, group=None):
        import torch.distributed as dist
        self.dist, self.group = dist, group
        self.world = dist.get_world_size(group)

    def gather(self, recs):
        (local,) = recs
        parts = [torch.empty_like(local) for _ in range(self.world)]
        self.dist.all_gather(parts, local.contiguous(), group=self.group)
        return torch.stack(parts)

    def max(self, vals):
        """Element-wise maximum over the ranks, read once."""
        (local,) = vals
        t = local.clone()
        self.dist.all_reduce(t, op=self.dist.ReduceOp.MAX, group=self.group)
        return t.tolist()


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
        return _solve(segments, comm, s0, tol, max_iters, R)


def _exchange(segments, comm, s0, k, R):
    """Fold, gather and combine of iteration k; returns the residual of H^k
    (a device tensor)."""
    for sg in segments:
        sg.fold(k)
    recs = comm.gather([sg.rec for sg in segments])
    if recs.shape[0] != R:
        raise ValueError(f"gathered {recs.shape[0]} segment records, expected {R}")
    res = [sg.combine(recs, s0) for sg in segments]
    return res[0]


def _solve(segments, comm, s0, tol, max_iters, R):
    for sg in segments:
        sg.start(s0)
    # residual of the zero guess (the same on every process), carries of iteration 0
    r = float(_exchange(segments, comm, s0, 0, R).item())
    k = 0
    while True:
        if r != r or math.isinf(r):
            return k, r, NONFINITE
        if r <= tol:
            return k, r, OK
        if k == max_iters:
            return k, r, NOT_CONVERGED
        if k > 0:
            _exchange(segments, comm, s0, k, R)  # carries; its residual is r already
        for sg in segments:
            sg.apply(k)
        r, err = comm.max([sg.pass_outcome() for sg in segments])
        if err > 0:
            raise capi.PararnnError(capi.ERR_TIMEOUT, "a segment pass raised a device-side error")
        k += 1
