"""The multi-rank host logic of bench.py on CPU ranks (gloo, world size 2):
every rank solves its own independent problem (different seeds, no data
exchange), the step time is the max over ranks, and the job value counts the
work of all ranks."""
import os
import socket

import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _rank_main(rank, world, port, out):
    import sys
    sys.path.insert(0, ROOT)
    import bench
    from nonlinear_rnn_newton_b200 import workloads as W
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), RANK=str(rank), WORLD_SIZE=str(world))
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        local_ms = [3.0, 5.0][rank]
        ms = bench.max_over_ranks(local_ms, world, device="cpu")
        w = W.GRU_SMALL
        x = W.make_inputs(w, seed=rank)
        # what each rank would solve: a digest of its inputs, gathered only for the test
        dig = torch.tensor([float(x.u.double().sum()), float(x.a.double().sum())], dtype=torch.float64)
        all_dig = [torch.zeros(2, dtype=torch.float64) for _ in range(world)]
        dist.all_gather(all_dig, dig)
        bench.barrier(world)
        out[rank] = (ms, bench.job_value(w.N, world, ms), [d.tolist() for d in all_dig])
    finally:
        dist.destroy_process_group()


def test_two_ranks_max_time_and_weak_scaling_value():
    ctx = mp.get_context("spawn")
    mgr = ctx.Manager()
    out = mgr.dict()
    port = _free_port()
    procs = [ctx.Process(target=_rank_main, args=(r, 2, port, out)) for r in range(2)]
    for p in procs:
        p.start()
    for p in procs:
        p.join(timeout=120)
        assert p.exitcode == 0
    from nonlinear_rnn_newton_b200 import workloads as W
    n = W.GRU_SMALL.N
    for r in range(2):
        ms, value, digs = out[r]
        assert ms == 5.0                       # slowest rank
        assert value == pytest.approx(2 * n / 5e-3)
        assert digs[0] != digs[1]              # independent problems (seed = rank)
