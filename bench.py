"""Benchmark of the ParaRNN Newton solve on B200.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl ours|reference]
                    [--workload NAME] [--no-cpu-baseline]

A step is one full Newton solve (every iteration until convergence) of the
workload, through the C ABI (pararnn_*_solve_async), with inputs resident in
HBM.  Default workload: ParaGRU, bf16 gate pre-activations / fp32 state,
B=8, L=4096, D=1024 (u ~ N(0,1), a ~ U(-0.5,0.5), h0 ~ N(0,0.1), seed 0).
Metric: tokens*channels per second = B*L*D / solve time.  Under torchrun
every rank solves its own independent problem (seed + rank; no collective on
the data path) and the time is the max over ranks.

Rank 0 prints one JSON line.  `--impl reference` times the CPU oracle
instead (the reference arm; rank 0 only).
"""
import argparse
import json
import os
import statistics
import subprocess
import sys
import threading
import time

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

import torch  # noqa: E402

from nonlinear_rnn_newton_b200 import workloads as W  # noqa: E402

PEAKS_PATH = os.path.join(ROOT, "MEASURED_PEAKS.json")
FALLBACK_HBM_GBS = 6650.0
METRIC = "Newton-solve tokens\u00b7channels/s and % of HBM roofline; iters to converge"


def hbm_peak():
    try:
        with open(PEAKS_PATH) as f:
            return float(json.load(f)["hbm_gbs"]), "measured"
    except Exception:
        return FALLBACK_HBM_GBS, "fallback"


def algorithmic_bytes(w: W.Workload, iters: int) -> int:
    """Bytes a Newton solve must move: every pass reads the gates and writes the
    states; every pass after the first (initial guess 0) also reads the states."""
    es = 2 if w.u_dtype == "bf16" else 4
    ns = 1 if w.cell == "gru" else 2
    per_first = w.G * es + ns * 4
    per_next = w.G * es + 2 * ns * 4
    passes = max(iters, 1)
    return w.N * (per_first + (passes - 1) * per_next)


class ClockSampler:
    """Samples nvidia-smi clocks and throttle reasons while running."""

    FIELDS = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, gpu_index):
        self.gpu = gpu_index
        self.proc = None
        self.lines = []
        self.t = None

    def __enter__(self):
        try:
            self.proc = subprocess.Popen(
                ["nvidia-smi", f"--id={self.gpu}", f"--query-gpu={self.FIELDS}", "--format=csv,noheader,nounits",
                 "-lms", "100"], stdout=subprocess.PIPE, stderr=subprocess.DEVNULL, text=True)
            self.t = threading.Thread(target=self._read, daemon=True)
            self.t.start()
            time.sleep(0.3)
        except Exception:
            self.proc = None
        return self

    def _read(self):
        for line in self.proc.stdout:
            self.lines.append(line.strip())

    def __exit__(self, *exc):
        if self.proc is not None:
            time.sleep(0.25)
            self.proc.terminate()
            try:
                self.proc.wait(timeout=5)
            except Exception:
                self.proc.kill()

    def summary(self):
        sm, smax, reasons = [], None, set()
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        for ln in self.lines:
            parts = [p.strip() for p in ln.split(",")]
            if len(parts) < 9:
                continue
            try:
                sm.append(float(parts[1]))
                smax = float(parts[2])
            except ValueError:
                continue
            for n, v in zip(names, parts[5:9]):
                if v.lower().startswith("active"):
                    reasons.add(n)
        if not sm:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["unsampled"], "samples": 0}
        return {"sm_mhz": statistics.median(sm), "sm_max_mhz": smax, "reasons": sorted(reasons),
                "samples": len(sm)}


def dist_setup(n_gpus):
    rank = int(os.environ.get("RANK", "0"))
    world = int(os.environ.get("WORLD_SIZE", "1"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    if world > 1:
        import datetime
        import torch.distributed as dist
        torch.cuda.set_device(local)
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120),
                                device_id=torch.device("cuda", local))
    return rank, world, local


def max_over_ranks(value, world):
    if world == 1:
        return value
    import torch.distributed as dist
    t = torch.tensor([value], dtype=torch.float64, device="cuda")
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def barrier(world):
    if world > 1:
        import torch.distributed as dist
        dist.barrier()


def solve_fn(w, xd, out, ws, stream):
    import nonlinear_rnn_newton_b200 as P
    if w.cell == "gru":
        return lambda: P.pararnn_gru_solve_async(xd.u, xd.a, xd.h0, out[0], ws, w.tol, w.max_iters, stream)
    return lambda: P.pararnn_lstm_solve_async(xd.u, xd.a, xd.c0, xd.h0, out[0], out[1], ws, w.tol,
                                              w.max_iters, stream)


def time_baselines(w, xd, out, stream, reps=5):
    """Device time of the two GPU baselines on the same input: the naive
    sequential step kernel (one thread per channel walks L) and one pass of the
    plain diagonal linear scan (zero-weight GRU)."""
    import nonlinear_rnn_newton_b200 as P
    wsl = torch.empty(P.pararnn_linear_scan_workspace_size(w.B, w.L, w.D), dtype=torch.uint8, device=out.device)
    res = {}
    for name, fn, nbytes in (
            ("sequential_gpu", lambda: P.pararnn_gru_sequential(xd.u, xd.a, xd.h0, out, stream=stream),
             w.N * (w.G * (2 if w.u_dtype == "bf16" else 4) + 4)),
            ("linear_scan_gpu", lambda: P.pararnn_linear_scan(xd.u, xd.h0, out, wsl, stream=stream),
             w.N * (2 * (2 if w.u_dtype == "bf16" else 4) + 4))):
        for _ in range(2):
            fn()
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        e0.record(stream)
        for _ in range(reps):
            fn()
        e1.record(stream)
        stream.synchronize()
        ms = e0.elapsed_time(e1) / reps
        res[name] = {"ms": ms, "value": w.N / (ms * 1e-3), "unit": "tokens\u00b7channels/s",
                     "gbs": nbytes / (ms * 1e-3) / 1e9}
    return res


def cpu_oracle_sample(w, x, max_batches=1):
    """Time the oracle's Newton solve on a bounded sample (the first batch rows)
    of the workload.  Returns (tokens*channels/s, description, cores)."""
    import oracle
    nb = min(max_batches, w.B)
    u = x.u[:nb]
    h0 = None if x.h0 is None else x.h0[:nb]
    t0 = time.perf_counter()
    if w.cell == "gru":
        _, it, _, _, _ = oracle.gru_newton(u, x.a, h0, tol=w.tol, max_iters=w.max_iters)
    else:
        _, _, it, _, _, _ = oracle.lstm_newton(u, x.a, None, h0, tol=w.tol, max_iters=w.max_iters)
    dt = time.perf_counter() - t0
    n = nb * w.L * w.D
    return n / dt, f"oracle Newton solve (fp64, serial C) on batch rows 0..{nb - 1} of the workload " \
                   f"(B={nb}, L={w.L}, D={w.D}; {it} iterations), input conversion excluded", 1


def run_reference(args, w):
    rank = int(os.environ.get("RANK", "0"))
    if rank != 0:
        return
    x = W.make_inputs(w, seed=0)
    vals = []
    desc = ""
    for i in range(args.warmup + args.steps):
        v, desc, cores = cpu_oracle_sample(w, x, max_batches=1)
        if i >= args.warmup:
            vals.append(v)
    value = statistics.median(vals)
    line = {
        "impl": "reference", "metric": METRIC, "value": value,
        "unit": "tokens\u00b7channels/s", "n_gpus": args.gpus, "steps": args.steps, "warmup": args.warmup,
        "ms_per_step": 1e3 * (w.L * w.D) / value, "higher_is_better": True, "dtype": "f64",
        "data": "synthetic", "config": {"workload": w.name},
        "cpu_baseline": {"value": value, "unit": "tokens\u00b7channels/s", "cores": 1, "kind": "oracle",
                         "sample": desc},
        "e2e": {"value": value, "unit": "tokens\u00b7channels/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
        "vs_baseline": None,
    }
    print(json.dumps(line), flush=True)


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=20)
    ap.add_argument("--warmup", type=int, default=3)
    ap.add_argument("--impl", default="ours", choices=["ours", "reference"])
    ap.add_argument("--workload", default=W.GRU.name, choices=sorted(W.BY_NAME))
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--e2e-steps", type=int, default=5)
    ap.add_argument("--baselines", type=int, default=1, help="also time the sequential GPU kernel and "
                    "the plain linear scan on the same input (GRU workloads)")
    args = ap.parse_args()
    args.warmup = max(args.warmup, 3)
    w = W.BY_NAME[args.workload]

    if args.impl == "reference":
        run_reference(args, w)
        return

    rank, world, local = dist_setup(args.gpus)
    dev = torch.device("cuda", local)
    torch.cuda.set_device(dev)
    import nonlinear_rnn_newton_b200 as P
    from nonlinear_rnn_newton_b200 import capi

    x = W.make_inputs(w, seed=rank)
    xd = x.to(dev)
    ns = 1 if w.cell == "gru" else 2
    out = [torch.empty((w.B, w.L, w.D), dtype=torch.float32, device=dev) for _ in range(ns)]
    wsz = (P.pararnn_gru_workspace_size if w.cell == "gru" else P.pararnn_lstm_workspace_size)(w.B, w.L, w.D)
    ws = torch.empty(wsz, dtype=torch.uint8, device=dev)
    stream = torch.cuda.Stream(dev)
    step = solve_fn(w, xd, out, ws, stream)

    # warm-up (also validates the solve)
    for _ in range(args.warmup):
        step()
    st, iters, resid, resid0 = P.pararnn_read_result(ws, stream)
    if st not in (0, 1):
        raise SystemExit(f"solve failed: status {st} ({capi.status_string(st)})")

    # timed region: K back-to-back solves on one stream, CUDA events around each
    evs = [torch.cuda.Event(enable_timing=True) for _ in range(args.steps + 1)]
    barrier(world)
    torch.cuda.synchronize(dev)
    launches0 = capi.kernel_launch_count()
    with ClockSampler(local) as clk:
        evs[0].record(stream)
        for i in range(args.steps):
            step()
            evs[i + 1].record(stream)
        stream.synchronize()
    launches = capi.kernel_launch_count() - launches0
    barrier(world)
    torch.cuda.synchronize(dev)
    per = [evs[i].elapsed_time(evs[i + 1]) for i in range(args.steps)]
    total_ms = evs[0].elapsed_time(evs[-1])
    total_ms = max_over_ranks(total_ms, world)
    ms_per_step = total_ms / args.steps
    st2, iters2, resid2, _ = P.pararnn_read_result(ws, stream)

    value = world * w.N / (ms_per_step * 1e-3)
    peak, peak_kind = hbm_peak()
    algo = algorithmic_bytes(w, iters2)
    mean_launch_ms = statistics.mean(per)
    achieved = algo / (mean_launch_ms * 1e-3) / 1e9

    # end to end through the public API with host buffers (pinned)
    e2e = None
    if args.e2e_steps > 0:
        hu = x.u.pin_memory()
        ha = x.a.pin_memory()
        hh0 = None if x.h0 is None else x.h0.pin_memory()
        hout = [torch.empty((w.B, w.L, w.D), dtype=torch.float32).pin_memory() for _ in range(ns)]
        du_, da_ = torch.empty_like(xd.u), torch.empty_like(xd.a)
        dh0_ = None if x.h0 is None else torch.empty_like(xd.h0)

        class _X:
            pass
        xe = _X()
        xe.u, xe.a, xe.h0, xe.c0 = du_, da_, dh0_, None
        estep = solve_fn(w, xe, out, ws, stream)
        h2d = hu.numel() * hu.element_size() + ha.numel() * 4 + (0 if hh0 is None else hh0.numel() * 4)
        d2h = sum(o.numel() * 4 for o in hout)

        def e2e_step():
            with torch.cuda.stream(stream):
                du_.copy_(hu, non_blocking=True)
                da_.copy_(ha, non_blocking=True)
                if hh0 is not None:
                    dh0_.copy_(hh0, non_blocking=True)
                estep()
                for o, ho in zip(out, hout):
                    ho.copy_(o, non_blocking=True)

        e2e_step()
        stream.synchronize()
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        barrier(world)
        e0.record(stream)
        for _ in range(args.e2e_steps):
            e2e_step()
        e1.record(stream)
        stream.synchronize()
        ems = max_over_ranks(e0.elapsed_time(e1), world) / args.e2e_steps
        e2e = {"value": world * w.N / (ems * 1e-3), "unit": "tokens\u00b7channels/s", "ms_per_step": ems,
               "h2d_bytes_per_step": h2d, "d2h_bytes_per_step": d2h}

    baselines = None
    if args.baselines and w.cell == "gru":
        baselines = time_baselines(w, xd, out[0], stream, reps=5)

    cpu = None
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        v, desc, cores = cpu_oracle_sample(w, x, max_batches=1)
        cpu = {"value": v, "unit": "tokens\u00b7channels/s", "cores": cores, "kind": "oracle", "sample": desc}

    if rank == 0:
        line = {
            "metric": METRIC, "value": value, "unit": "tokens\u00b7channels/s",
            "n_gpus": world, "steps": args.steps, "warmup": args.warmup, "ms_per_step": ms_per_step,
            "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f32",
            "data": "synthetic",
            "config": {"workload": w.name, "cell": w.cell, "B": w.B, "L": w.L, "D": w.D,
                       "u_dtype": w.u_dtype, "tol": w.tol, "max_iters": w.max_iters,
                       "l2": "inputs larger than L2 (gates + states > 126 MB); no flush",
                       "per_rank": "independent problem, seed = rank"},
            "iters": iters2, "residual": resid2, "status": st2,
            "roofline": {"bound": "hbm", "achieved": achieved, "peak": peak, "unit": "GB/s",
                         "frac": achieved / peak, "traffic": None, "peak_kind": peak_kind,
                         "algorithmic_bytes_per_launch": algo,
                         "kernel_ms_mean": mean_launch_ms},
            "per_iteration_frac": achieved / peak,
            "gpu_launches": launches,
            "clocks": clk.summary(),
            "e2e": e2e,
            "cpu_baseline": cpu,
            "baselines": baselines,
        }
        print(json.dumps(line), flush=True)
    if world > 1:
        import torch.distributed as dist
        dist.destroy_process_group()


if __name__ == "__main__":
    main()
