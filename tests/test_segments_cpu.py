"""The host logic of the sequence-split solve (nonlinear_rnn_newton_b200.sharded)
on CPU ranks (gloo, world size 2 and 3): every rank holds one segment, the
segments' records are all-gathered in segment order, the residual maximum is
all-reduced, and the stopping decision is common.  The per-segment
computations are a float64 stand-in written here from the method (the fold
of a segment's step maps at the iterate; their composition segment by segment
into the state entering each one; one Newton pass over a segment from its
linearisation point and carry), so the test checks the orchestration and the
algebra, not the kernels (which the GPU tests check).  Expected: the oracle's
sequential states and its Newton iteration count."""
import os
import socket

import numpy as np
import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


class Float64Segment:
    """The interface of sharded.Segment, computed in float64 on the CPU.
    Record (flat): fold matrix M [NS][NS][B][D], fold offset v [NS][B][D],
    last and first iterate states [NS][B][D] each, first-step gates
    [G][B][D], then the residual over steps 2..Ls."""

    def __init__(self, cell, u, a, index):
        self.cell, self.index, self.stream = cell, index, None
        self.step, self.jac = cell.step, cell.jac
        self.NS, self.G = cell.NS, cell.G
        self.a = a.numpy()
        self.ug = np.transpose(u.numpy(), (1, 2, 0, 3))  # [Ls, G, B, D]
        B, Ls, G, D = u.shape
        self.B, self.Ls, self.D = B, Ls, D
        self.H = torch.zeros((self.NS, B, Ls, D), dtype=torch.float64)
        self.carry = np.zeros((self.NS, B, D))
        self.lin = np.zeros((self.NS, B, D))
        self.res = 0.0

    def _map(self, prev, l):
        J = self.jac(prev, self.ug[l], self.a)                 # [NS][NS][B][D]
        f = self.step(prev, self.ug[l], self.a)
        return J, f - np.einsum("qrbd,rbd->qbd", J, prev)

    def start(self, s0):
        self.H.zero_()

    def fold(self, k):
        Hk = self.H.numpy()
        NS, B, D = self.NS, self.B, self.D
        M = np.broadcast_to(np.eye(NS)[:, :, None, None], (NS, NS, B, D)).copy()
        v = np.zeros((NS, B, D))
        r = 0.0
        for l in range(1, self.Ls):
            J, o = self._map(Hk[:, :, l - 1], l)
            M = np.einsum("qrbd,rsbd->qsbd", J, M)
            v = np.einsum("qrbd,rbd->qbd", J, v) + o
            f = self.step(Hk[:, :, l - 1], self.ug[l], self.a)
            r = float(np.maximum(r, np.max(np.abs(Hk[:, :, l] - f))))
        parts = [M.ravel(), v.ravel(), Hk[:, :, -1].ravel(), Hk[:, :, 0].ravel(), self.ug[0].ravel(), [r, 0, 0, 0]]
        self.rec = torch.from_numpy(np.concatenate(parts))

    def combine(self, recs, s0):
        NS, G, B, D = self.NS, self.G, self.B, self.D
        c = s0.numpy().copy() if s0 is not None else np.zeros((NS, B, D))
        lin = c.copy()
        r = 0.0
        for j, rec in enumerate(recs.numpy()):
            o = 0
            M = rec[o:o + NS * NS * B * D].reshape(NS, NS, B, D); o += NS * NS * B * D
            v = rec[o:o + NS * B * D].reshape(NS, B, D); o += NS * B * D
            last = rec[o:o + NS * B * D].reshape(NS, B, D); o += NS * B * D
            first = rec[o:o + NS * B * D].reshape(NS, B, D); o += NS * B * D
            u1 = rec[o:o + G * B * D].reshape(G, B, D); o += G * B * D
            r = float(np.maximum(r, rec[o]))
            J = self.jac(lin, u1, self.a)
            f = self.step(lin, u1, self.a)
            r = float(np.maximum(r, np.max(np.abs(first - f))))
            if j == self.index:
                self.carry, self.lin = c.copy(), lin.copy()
            x = np.einsum("qrbd,rbd->qbd", J, c - lin) + f
            c = np.einsum("qrbd,rbd->qbd", M, x) + v
            lin = last
        return torch.tensor([r], dtype=torch.float64)

    def apply(self, k):
        Hk = self.H.numpy()
        Hn = np.empty_like(Hk)
        prev_k, s = self.lin, self.carry
        for l in range(self.Ls):
            J, o = self._map(prev_k, l)
            s = np.einsum("qrbd,rbd->qbd", J, s) + o
            Hn[:, :, l] = s
            prev_k = Hk[:, :, l]
        prev, r = self.carry, 0.0
        for l in range(self.Ls):
            # NaN kept, like the kernels' max.NaN (Python's max would drop it)
            r = float(np.maximum(r, np.max(np.abs(Hn[:, :, l] - self.step(prev, self.ug[l], self.a)))))
            prev = Hn[:, :, l]
        self.H = torch.from_numpy(Hn)
        self.res = r

    def pass_outcome(self):
        return torch.tensor([self.res, 0.0], dtype=torch.float64)


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _draw(name, B, L, D):
    from tests.user_cells import CELLS
    cell = CELLS[name]
    g = torch.Generator().manual_seed(5)
    u = torch.randn((B, L, cell.G, D), generator=g, dtype=torch.float64)
    a = torch.rand((cell.G, D), generator=g, dtype=torch.float64) - 0.5
    s0 = torch.randn((cell.NS, B, D), generator=g, dtype=torch.float64) * 0.1
    return cell, u, a, s0


def _rank_main(rank, world, port, name, edges, out):
    import sys
    sys.path.insert(0, ROOT)
    from nonlinear_rnn_newton_b200 import sharded as SH
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), RANK=str(rank), WORLD_SIZE=str(world))
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        cell, u, a, s0 = _draw(name, 2, edges[-1], 3)
        seg = Float64Segment(cell, u[:, edges[rank]:edges[rank + 1]].contiguous(), a, rank)
        it, r, st = SH.solve_segments([seg], SH.DistComm(), s0, tol=1e-10, max_iters=30, n_segments=world)
        parts = [None] * world  # segments differ in length: gathered as objects, for the test only
        dist.all_gather_object(parts, seg.H.numpy())
        out[rank] = (it, r, st, np.concatenate(parts, axis=2))
    finally:
        dist.destroy_process_group()


@pytest.mark.parametrize("name,edges", [("gru", [0, 23, 40]), ("lstm", [0, 9, 20, 31]), ("mixed", [0, 1, 16])])
def test_ranks_solve_their_segments(name, edges):
    from oracle import generic as OG
    world = len(edges) - 1
    ctx = mp.get_context("spawn")
    mgr = ctx.Manager()
    out = mgr.dict()
    port = _free_port()
    procs = [ctx.Process(target=_rank_main, args=(r, world, port, name, edges, out)) for r in range(world)]
    for p in procs:
        p.start()
    for p in procs:
        p.join(timeout=180)
        assert p.exitcode == 0
    cell, u, a, s0 = _draw(name, 2, edges[-1], 3)
    seq = OG.generic_seq(cell.step, u, a, s0, cell.NS)
    _, oit, ores, ost, hist = OG.generic_newton(cell.step, cell.jac, u, a, s0, cell.NS, tol=1e-10, max_iters=30)
    for r in range(world):
        it, res, st, Hs = out[r]
        assert (it, st) == (oit, ost)                  # same decision on every rank
        assert abs(res - ores) <= 1e-12 + 1e-9 * ores
        assert np.max(np.abs(Hs - seq)) < 1e-9


def test_stopping_paths_in_one_process():
    """LocalComm (all segments in this process): max_iters = 0 and a huge tol
    stop at the zero guess with its residual; max_iters = 1 gives the oracle's
    first iterate; a NaN input stops with the non-finite status."""
    from nonlinear_rnn_newton_b200 import sharded as SH
    from oracle import generic as OG
    cell, u, a, s0 = _draw("lstm", 2, 30, 3)
    edges = [0, 7, 30]
    segs = lambda uu: [Float64Segment(cell, uu[:, edges[r]:edges[r + 1]].contiguous(), a, r) for r in range(2)]
    seq = segs(u)
    it, r, st = SH.solve_segments(seq, SH.LocalComm(), s0, max_iters=0)
    _, oit, ores, ost, hist = OG.generic_newton(cell.step, cell.jac, u, a, s0, cell.NS, max_iters=0)
    assert (it, st) == (0, SH.NOT_CONVERGED) and abs(r - ores) <= 1e-12
    it, r, st = SH.solve_segments(seq, SH.LocalComm(), s0, tol=1e30)
    assert (it, st) == (0, SH.OK)
    it, r, st = SH.solve_segments(seq, SH.LocalComm(), s0, tol=0.0, max_iters=1)
    H1, *_ = OG.generic_newton(cell.step, cell.jac, u, a, s0, cell.NS, tol=0.0, max_iters=1)
    Hs = np.concatenate([sg.H.numpy() for sg in seq], axis=2)
    assert (it, st) == (1, SH.NOT_CONVERGED) and np.max(np.abs(Hs - H1)) < 1e-12
    bad = u.clone()
    bad[1, 20, 0, 2] = float("nan")
    it, r, st = SH.solve_segments(segs(bad), SH.LocalComm(), s0)
    assert st == SH.NONFINITE and r != r
