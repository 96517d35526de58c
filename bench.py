"""Benchmark of the ParaRNN Newton solve on B200.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl ours|reference]
                    [--workload NAME] [--no-extras] [--no-cpu-baseline]
                    [--decode] [--cells] [--seq-segments R1,R2,...]

A step is one pass of the whole hot path over the workload through the C ABI:
one full Newton solve (every iteration until convergence, the convergence
test included) -- followed, for the training workload, by the reverse-time
adjoint -- with inputs resident in HBM.  The headline workload is the largest
single-GPU Newton solve: ParaGRU, bf16 gate pre-activations / fp32 state,
B=1, L=65536, D=2048 (u ~ N(0,1), a ~ U(-0.5,0.5), h0 ~ N(0,0.1),
seed = rank).  Metric: tokens*channels per second = B*L*D / step time.
Under torchrun every rank solves its own independent problem (no collective
on the data path) and the time is the max over ranks.

On one GPU the same line also carries, under "configs", every other solve
workload (ParaGRU and ParaLSTM at B=8, L=4096, D=1024; the B=1, D=2048
sequence-length sweep with the sequential GPU kernel and the plain linear scan
at each L; the ParaLSTM and ParaGRU training steps, solve plus adjoint, at
B=4, L=16384, D=2048), each with its roofline and per-pass figures, and the
CPU oracle's sequential stepping timed on all host cores and on one core.

Rank 0 prints one JSON line.  `--impl reference` times the CPU oracle on a
bounded sample of the same workload instead (the reference arm; rank 0 only).
"""
import argparse
import itertools
import hashlib
import json
import os
import re
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
PROFILES = os.path.join(ROOT, "profiles")
CSRC = os.path.join(ROOT, "nonlinear_rnn_newton_b200", "csrc")
FALLBACK_HBM_GBS = 6650.0
METRIC = "Newton-solve tokens·channels/s and % of HBM roofline; iters to converge"
UNIT = "tokens·channels/s"


def hbm_peak():
    try:
        with open(PEAKS_PATH) as f:
            return float(json.load(f)["hbm_gbs"]), "measured (MEASURED_PEAKS.json hbm_gbs)"
    except Exception:
        return FALLBACK_HBM_GBS, "fallback"


def solve_bytes(w: W.Workload, iters: int) -> int:
    """Bytes a Newton solve must move: every pass reads the gates and writes
    the states; every pass after the first (initial guess 0) also reads the
    states.  Weights and workspace are < 0.1% and not counted."""
    es = 2 if w.u_dtype == "bf16" else 4
    ns = 1 if w.cell == "gru" else 2
    first = w.G * es + ns * 4
    later = w.G * es + 2 * ns * 4
    return w.N * (first + (max(iters, 1) - 1) * later)


def pass_bytes(w: W.Workload, k: int) -> int:
    """Bytes Newton pass k must move (pass 0 starts from the zero guess and
    reads no states)."""
    es = 2 if w.u_dtype == "bf16" else 4
    ns = 1 if w.cell == "gru" else 2
    return w.N * (w.G * es + (1 if k == 0 else 2) * ns * 4)


def per_pass(w: W.Workload, pass_us, peak):
    """Per-iteration roofline from the solve's device pass timestamps."""
    return [{"pass": k, "us": round(us, 2), "bytes": pass_bytes(w, k),
             "gbs": pass_bytes(w, k) / (us * 1e-6) / 1e9, "frac": pass_bytes(w, k) / (us * 1e-6) / 1e9 / peak}
            for k, us in enumerate(pass_us) if us > 0]


def adjoint_bytes(w: W.Workload) -> int:
    """The adjoint reads gates, forward states (and the state before each
    step, which is the previous row of the same arrays) and the upstream
    gradient, and writes fp32 gate gradients."""
    es = 2 if w.u_dtype == "bf16" else 4
    ns = 1 if w.cell == "gru" else 2
    return w.N * (w.G * es + ns * 4 + 4 + w.G * 4)


# the sources each profiled kernel is compiled from (its device code)
_COMMON = ["device_common.cuh", "pararnn_internal.h", "cells.cuh", "scan_common.cuh"]
KERNEL_SOURCES = {
    "newton_solve_ws_kernel": _COMMON + ["newton.cuh", "newton_ws.cuh"],
    "adjoint_ws_kernel": _COMMON + ["adjoint.cuh", "adjoint_ws.cuh"],
    "project_pass0_kernel": _COMMON + ["project.cuh"],
}


def source_digest(kernel: str) -> str:
    """Digest of the device sources of `kernel`; a profile summary records it,
    so that its counters are used only while the kernel is unchanged."""
    h = hashlib.sha256()
    for name in sorted(KERNEL_SOURCES[kernel]):
        with open(os.path.join(CSRC, name), "rb") as f:
            h.update(name.encode() + b"\0" + f.read())
    return h.hexdigest()[:16]


def profile_traffic(kernel: str, workload: str):
    """DRAM bytes per launch from the committed ncu summary of this kernel and
    workload, or None when there is none or the kernel's sources changed since
    the counters were taken."""
    path = os.path.join(PROFILES, f"{kernel}__{workload}.md")
    try:
        text = open(path).read()
    except OSError:
        return None
    m_t = re.search(r"^traffic_bytes_per_launch:\s*(\d+)", text, re.M)
    m_s = re.search(r"^source_digest:\s*([0-9a-f]+)", text, re.M)
    if not m_t or not m_s or m_s.group(1) != source_digest(kernel):
        return None
    return int(m_t.group(1))


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


def dist_setup():
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


def max_over_ranks(value, world, device="cuda"):
    """Max of a per-rank number over all ranks (every rank gets it); `device`
    is where the backend's tensors live (cuda for nccl, cpu for gloo)."""
    if world == 1:
        return value
    import torch.distributed as dist
    t = torch.tensor([value], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def job_value(n_per_rank, world, ms_per_step):
    """Whole-job throughput: every rank runs its own problem of n_per_rank
    token*channels per step (weak scaling); the step time is the slowest
    rank's."""
    return world * n_per_rank / (ms_per_step * 1e-3)


def barrier(world):
    if world > 1:
        import torch.distributed as dist
        dist.barrier()


class Step:
    """One pass of the hot path on device-resident inputs, through the C ABI.
    Records CUDA events on `stream` around the solve (and the adjoint)."""

    def __init__(self, w, xd, dev, stream):
        import nonlinear_rnn_newton_b200 as P
        self.P, self.w, self.x, self.stream = P, w, xd, stream
        ns = 1 if w.cell == "gru" else 2
        self.out = [torch.empty((w.B, w.L, w.D), dtype=torch.float32, device=dev) for _ in range(ns)]
        size = (P.pararnn_gru_workspace_size if w.cell == "gru" else P.pararnn_lstm_workspace_size)
        self.ws = torch.empty(size(w.B, w.L, w.D), dtype=torch.uint8, device=dev)
        self.adj = None
        if w.train:
            asize = (P.pararnn_gru_adjoint_workspace_size if w.cell == "gru"
                     else P.pararnn_lstm_adjoint_workspace_size)
            self.adj = {
                "ws": torch.empty(asize(w.B, w.L, w.D), dtype=torch.uint8, device=dev),
                "du": torch.empty((w.B, w.L, w.G, w.D), dtype=torch.float32, device=dev),
                "da": torch.empty((w.G, w.D), dtype=torch.float32, device=dev),
            }

    def solve(self):
        w, x, P = self.w, self.x, self.P
        if w.cell == "gru":
            P.pararnn_gru_solve_async(x.u, x.a, x.h0, self.out[0], self.ws, w.tol, w.max_iters, self.stream)
        else:
            P.pararnn_lstm_solve_async(x.u, x.a, x.c0, x.h0, self.out[0], self.out[1], self.ws, w.tol,
                                       w.max_iters, self.stream)

    def adjoint(self):
        w, x, P, a = self.w, self.x, self.P, self.adj
        if w.cell == "gru":
            P.pararnn_gru_adjoint(x.u, x.a, x.h0, self.out[0], x.dh, du=a["du"], da=a["da"], want_dh0=False,
                                  workspace=a["ws"], stream=self.stream)
        else:
            P.pararnn_lstm_adjoint(x.u, x.a, x.c0, x.h0, self.out[0], self.out[1], x.dh, du=a["du"],
                                   da=a["da"], want_ds0=False, workspace=a["ws"], stream=self.stream)

    def __call__(self, ev=None):
        if ev is not None:
            ev[0].record(self.stream)
        self.solve()
        if ev is not None:
            ev[1].record(self.stream)
        if self.adj is not None:
            self.adjoint()
            if ev is not None:
                ev[2].record(self.stream)

    def result(self):
        return self.P.pararnn_read_result(self.ws, self.stream)

    def pass_times(self):
        return self.P.pararnn_read_pass_times(self.ws, self.stream)


def events(n, k):
    return [[torch.cuda.Event(enable_timing=True) for _ in range(k)] for _ in range(n)]


def time_baselines(w, xd, out, stream, dev, reps=5):
    """Device time of the two GPU baselines on the same input: the naive
    sequential step kernel (one thread per channel walks L) and one pass of the
    plain diagonal linear scan."""
    import nonlinear_rnn_newton_b200 as P
    wsl = torch.empty(P.pararnn_linear_scan_workspace_size(w.B, w.L, w.D), dtype=torch.uint8, device=dev)
    es = 2 if w.u_dtype == "bf16" else 4
    res = {}
    for name, fn, nbytes in (
            ("sequential_gpu", lambda: P.pararnn_gru_sequential(xd.u, xd.a, xd.h0, out, stream=stream),
             w.N * (w.G * es + 4)),
            ("linear_scan_gpu", lambda: P.pararnn_linear_scan(xd.u, xd.h0, out, wsl, stream=stream),
             w.N * (2 * es + 4))):
        for _ in range(2):
            fn()
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        e0.record(stream)
        for _ in range(reps):
            fn()
        e1.record(stream)
        stream.synchronize()
        ms = e0.elapsed_time(e1) / reps
        res[name] = {"ms": ms, "value": w.N / (ms * 1e-3), "unit": UNIT, "gbs": nbytes / (ms * 1e-3) / 1e9}
    return res


def measure(w, dev, stream, reps=10, warmup=3, baselines=True):
    """One workload at full size: `reps` back-to-back steps after `warmup`,
    CUDA events around every solve (and adjoint), the solve's per-pass device
    timestamps, and (GRU) the two GPU baselines on the same input.  Inputs
    exceed L2 (flagged where they do not)."""
    peak, _ = hbm_peak()
    xd = W.make_inputs(w, seed=0).to(dev)
    st = Step(w, xd, dev, stream)
    for _ in range(warmup):
        st()
    nev = 3 if w.train else 2
    evs = events(reps, nev)
    for i in range(reps):
        st(evs[i])
    stream.synchronize()
    r = st.result()
    if r[0] not in (0, 1):
        raise SystemExit(f"{w.name}: solve failed: status {r[0]}")
    solve_ms = statistics.mean(e[0].elapsed_time(e[1]) for e in evs)
    step_ms = statistics.mean(e[0].elapsed_time(e[-1]) for e in evs)
    algo = solve_bytes(w, r[1])
    out = {"workload": w.name, "cell": w.cell, "B": w.B, "L": w.L, "D": w.D, "u_dtype": w.u_dtype,
           "ms_per_step": step_ms, "value": w.N / (step_ms * 1e-3), "unit": UNIT, "iters": r[1],
           "status": r[0], "residual": r[2],
           "l2_resident": solve_bytes(w, 1) < 126e6,
           "roofline": {"bound": "hbm", "kernel": "newton_solve_ws_kernel", "kernel_ms_mean": solve_ms,
                        "algorithmic_bytes_per_launch": algo, "achieved": algo / (solve_ms * 1e-3) / 1e9,
                        "peak": peak, "unit": "GB/s", "frac": algo / (solve_ms * 1e-3) / 1e9 / peak,
                        "traffic": profile_traffic("newton_solve_ws_kernel", w.name),
                        "per_pass": per_pass(w, st.pass_times(), peak)}}
    if w.train:
        adj_ms = statistics.mean(e[1].elapsed_time(e[2]) for e in evs)
        ab = adjoint_bytes(w)
        out["adjoint"] = {"kernel": "adjoint_ws_kernel", "kernel_ms_mean": adj_ms, "algorithmic_bytes_per_launch": ab,
                          "achieved": ab / (adj_ms * 1e-3) / 1e9, "frac": ab / (adj_ms * 1e-3) / 1e9 / peak,
                          "traffic": profile_traffic("adjoint_ws_kernel", w.name)}
    if baselines and w.cell == "gru":
        out["baselines"] = time_baselines(w, xd, st.out[0], stream, dev)
    del st, xd
    torch.cuda.empty_cache()
    return out


def run_projection(dev, stream, B=8, L=4096, Din=1024, D=1024, reps=10):
    """The ParaGRU solve from the layer input, x [B,L,Din] -> u = x w^T
    (bf16, fp32 accumulation) -> Newton solve: the fused path (the projection
    on the tensor cores with pass 0 in its epilogue, pararnn_gru_project_solve)
    against the projection as a cuBLAS GEMM (torch.matmul) followed by the
    solve.  Inputs: x ~ N(0,1), w ~ N(0,1/Din), no bias, a ~ U(-0.5,0.5),
    h0 ~ N(0,0.1)."""
    import nonlinear_rnn_newton_b200 as P
    xi = W.make_projection_inputs(B, L, Din, D, seed=0, bias_std=0.0).to(dev)
    u = torch.empty((B, L, 3, D), dtype=torch.bfloat16, device=dev)
    h = torch.empty((B, L, D), dtype=torch.float32, device=dev)
    ws = torch.empty(P.pararnn_gru_project_workspace_size(B, L, D, Din), dtype=torch.uint8, device=dev)
    u2 = torch.empty_like(u)
    h2 = torch.empty_like(h)
    ws2 = torch.empty(P.pararnn_gru_workspace_size(B, L, D), dtype=torch.uint8, device=dev)
    x2, w2 = xi.x.view(B * L, Din), xi.w.view(3 * D, Din)

    def fused():
        P.pararnn_gru_project_solve_async(xi.x, xi.w, None, xi.a, xi.h0, u, h, ws, stream=stream)

    def gemm():
        with torch.cuda.stream(stream):
            torch.matmul(x2, w2.t(), out=u2.view(B * L, 3 * D))

    def unfused():
        gemm()
        P.pararnn_gru_solve_async(u2, xi.a, xi.h0, h2, ws2, stream=stream)

    def timed(fn):
        for _ in range(3):
            fn()
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        e0.record(stream)
        for _ in range(reps):
            fn()
        e1.record(stream)
        stream.synchronize()
        return e0.elapsed_time(e1) / reps

    t_f, t_u, t_g = timed(fused), timed(unfused), timed(gemm)
    fused()
    passes = P.pararnn_read_pass_times(ws, stream)
    rf = P.pararnn_read_result(ws, stream)
    unfused()
    ru = P.pararnn_read_result(ws2, stream)
    flops = 2.0 * B * L * Din * 3 * D
    return {"workload": f"gru_project_B{B}_L{L}_Din{Din}_D{D}", "fused_ms": t_f, "gemm_then_solve_ms": t_u,
            "gemm_ms": t_g, "gemm_tflops": flops / (t_g * 1e-3) / 1e12,
            "fused_pass0_us": passes[0] if passes else None,
            "fused_pass0_tflops": flops / (passes[0] * 1e-6) / 1e12 if passes else None,
            "iters": [rf[1], ru[1]], "status": [rf[0], ru[0]],
            "max_abs_state_diff": float((h - h2).abs().max()),
            "u_equal_fraction": float((u == u2).float().mean())}


def run_configs(headline, dev, stream):
    """Every solve workload except the headline, one after another, and the
    solve from the layer input (the fused input projection)."""
    out = {}
    for w in (W.GRU, W.LSTM) + W.GRU_SWEEP + (W.LSTM_TRAIN, W.GRU_TRAIN):
        if w.name == headline.name:
            continue
        out[w.name] = measure(w, dev, stream)
    pr = run_projection(dev, stream)
    out[pr["workload"]] = pr
    return out


def run_decode(dev, stream, T=256, reps=5):
    """Decode steps (one recurrence step for B sequences, state updated in
    place) at the solve workloads' width D=1024, bf16 gates: T steps captured
    in one CUDA graph, timed over `reps` replays; per step one kernel launch."""
    import nonlinear_rnn_newton_b200 as P
    out = []
    for cell in ("gru", "lstm"):
        for B in (8, 256):
            w = W.custom(cell, B, T, 1024, "bf16", h0_std=0.1)
            x = W.make_inputs(w, seed=0)
            u = x.u.transpose(0, 1).contiguous().to(dev)  # [T, B, G, D]: one contiguous slab per step
            a = x.a.to(dev)
            h = torch.zeros((B, w.D), device=dev)
            c = torch.zeros((B, w.D), device=dev)

            def steps():
                for t in range(T):
                    if cell == "gru":
                        P.pararnn_gru_step(u[t], a, h, h, stream=stream)
                    else:
                        P.pararnn_lstm_step(u[t], a, c, h, c, h, stream=stream)

            with torch.cuda.stream(stream):
                steps()  # warm up outside the capture
                g = torch.cuda.CUDAGraph()
                with torch.cuda.graph(g, stream=stream):
                    steps()
                for _ in range(2):
                    g.replay()
                e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
                e0.record(stream)
                for _ in range(reps):
                    g.replay()
                e1.record(stream)
            stream.synchronize()
            us = e0.elapsed_time(e1) * 1e3 / (reps * T)
            ns = 1 if cell == "gru" else 2
            nbytes = B * w.D * (w.G * 2 + 8 * ns) + w.G * w.D * 4  # gates, state read + write, weights
            out.append({"cell": cell, "B": B, "D": w.D, "us_per_step": round(us, 3),
                        "tokens_per_s": B / (us * 1e-6), "gbs": nbytes / (us * 1e-6) / 1e9,
                        "launches_per_step": 1})
            del g, u
    return out


def run_cells(dev, stream, reps=5):
    """User-written cells (the GRU and LSTM sources of example_cells, compiled
    at run time) on the solve workloads, beside the built-in kernels."""
    import nonlinear_rnn_newton_b200 as P
    from nonlinear_rnn_newton_b200 import example_cells
    peak, _ = hbm_peak()
    out = []
    for (w, src), flags in itertools.product(((W.GRU, example_cells.GRU), (W.LSTM, example_cells.LSTM)), (0, 1)):
        ns = 1 if w.cell == "gru" else 2
        with torch.cuda.device(dev):
            cell = P.pararnn_cell_create(src, w.G, ns, flags)
        x = W.make_inputs(w, seed=0).to(dev)
        s0 = torch.zeros((ns, w.B, w.D), device=dev)
        if x.h0 is not None:
            s0[ns - 1] = x.h0
        s = torch.empty((ns, w.B, w.L, w.D), device=dev)
        ws = torch.empty(P.pararnn_cell_workspace_size(cell, x.u.dtype, w.B, w.L, w.D), dtype=torch.uint8,
                         device=dev)
        run = lambda: P.pararnn_cell_solve_async(cell, x.u, x.a, s0, s, ws, tol=w.tol, max_iters=w.max_iters,
                                                 stream=stream)
        for _ in range(3):
            run()
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        e0.record(stream)
        for _ in range(reps):
            run()
        e1.record(stream)
        stream.synchronize()
        ms = e0.elapsed_time(e1) / reps
        r = P.pararnn_read_result(ws, stream)
        gbs = solve_bytes(w, r[1]) / (ms * 1e-3) / 1e9
        out.append({"workload": w.name, "cell": f"{w.cell} (user source)", "fast_math": bool(flags),
                    "compute_warps": P.pararnn_cell_compute_warps(cell, x.u.dtype), "ms": round(ms, 4), "iters": r[1],
                    "status": r[0], "value": w.N / (ms * 1e-3), "gbs": gbs, "frac": gbs / peak})
        del cell, ws, s, x
        torch.cuda.empty_cache()
    return out


def run_segments(w, xd, dev, stream, counts, reps=3):
    """The solve with each sequence split into R segments (the multi-GPU
    sequence sharding), all R run one after another on this GPU: time per
    solve and iterations, beside the unsplit solve."""
    from nonlinear_rnn_newton_b200 import sharded as SH
    ns = 1 if w.cell == "gru" else 2
    s0 = torch.zeros((ns, w.B, w.D), device=dev)
    if xd.h0 is not None:
        s0[ns - 1] = xd.h0
    out = []
    for R in counts:
        edges = [round(i * w.L / R) for i in range(R + 1)]
        segs = [SH.Segment(w.cell, xd.u[:, edges[r]:edges[r + 1]].contiguous(), xd.a, r, stream=stream)
                for r in range(R)]
        run = lambda: SH.solve_segments(segs, SH.LocalComm(), s0, w.tol, w.max_iters)
        run()
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        e0.record(stream)
        for _ in range(reps):
            it, r, st = run()
        e1.record(stream)
        stream.synchronize()
        ms = e0.elapsed_time(e1) / reps
        out.append({"segments": R, "ms": round(ms, 3), "ms_per_segment": round(ms / R, 3), "iters": it,
                    "status": st, "residual": r})
        del segs
        torch.cuda.empty_cache()
    return out


def oracle_sample(w, x, rows, chans):
    """Sub-problem of the workload the oracle is timed on: the first `rows`
    batch rows and `chans` channels (channels are independent, so this is the
    same work per token*channel)."""
    rows, chans = min(rows, w.B), min(chans, w.D)
    u = x.u[:rows, :, :, :chans]
    a = x.a[:, :chans]
    h0 = None if x.h0 is None else x.h0[:rows, :chans]
    dh = None if x.dh is None else x.dh[:rows, :, :chans]
    return u, a, h0, dh, rows * w.L * chans


def host_cores():
    """Threads the oracle's OpenMP loops use on this host (its default: one
    per core the process may run on)."""
    import oracle
    return oracle.max_threads()


def widen(u, a, h0):
    return (u.double().numpy(), a.double().numpy(), None if h0 is None else h0.double().numpy())


def time_oracle_seq(w, x, rows, chans, threads):
    """Tokens*channels/s of the oracle's sequential stepping (the plain
    definition of the solve's result: fp64 C, OpenMP over the independent
    channels) on `threads` threads, on a sample of the workload; the fp64
    widening of the inputs happens before the clock starts."""
    import numpy as np

    import oracle
    oracle.set_threads(threads)
    u, a, h0, _, n = oracle_sample(w, x, rows, chans)
    u64, a64, h064 = widen(u, a, h0)
    t0 = time.perf_counter()
    if w.cell == "gru":
        h = oracle.gru_seq(u64, a64, h064)
    else:
        _, h = oracle.lstm_seq(u64, a64, None, h064)
    dt = time.perf_counter() - t0
    assert np.isfinite(h).all()
    desc = (f"oracle sequential stepping (fp64 C, OpenMP over channels, {threads} thread(s)) on batch rows "
            f"0..{min(rows, w.B) - 1}, channels 0..{min(chans, w.D) - 1} of the workload (B={min(rows, w.B)}, "
            f"L={w.L}, D={min(chans, w.D)}); fp64 widening of the inputs excluded")
    return n / dt, dt, desc


def time_oracle_newton(w, x, rows, chans):
    """Tokens*channels/s of the oracle's serial Newton solve (one thread: the
    oracle's Newton is one serial loop) on a sample of the workload."""
    import numpy as np

    import oracle
    oracle.set_threads(1)
    u, a, h0, _, n = oracle_sample(w, x, rows, chans)
    u64, a64, h064 = widen(u, a, h0)
    t0 = time.perf_counter()
    if w.cell == "gru":
        h, it, _, _, _ = oracle.gru_newton(u64, a64, h064, tol=w.tol, max_iters=w.max_iters)
    else:
        _, h, it, _, _, _ = oracle.lstm_newton(u64, a64, None, h064, tol=w.tol, max_iters=w.max_iters)
    dt = time.perf_counter() - t0
    assert np.isfinite(h).all()
    desc = (f"oracle serial Newton (fp64 C, 1 thread, {it} iterations) on batch row 0, channels "
            f"0..{min(chans, w.D) - 1} (B=1, L={w.L}, D={min(chans, w.D)})")
    return n / dt, dt, desc


def cpu_baselines(w, x):
    """The CPU oracle beside the GPU numbers: its sequential stepping on all
    host cores (128 channels per thread, at most 1024 channels: a few seconds
    of CPU work) and on one core (128 channels), and its serial Newton on one
    core (64 channels)."""
    cores = host_cores()
    v, secs, desc = time_oracle_seq(w, x, 1, min(w.D, 1024, 128 * cores), cores)
    v1, secs1, desc1 = time_oracle_seq(w, x, 1, 128, 1)
    vn, secsn, descn = time_oracle_newton(w, x, 1, 64)
    return {"value": v, "unit": UNIT, "cores": cores, "kind": "oracle", "sample": desc, "seconds": secs,
            "one_core": {"value": v1, "unit": UNIT, "cores": 1, "sample": desc1, "seconds": secs1},
            "serial_newton_one_core": {"value": vn, "unit": UNIT, "cores": 1, "sample": descn, "seconds": secsn}}


def run_reference(args, w):
    rank = int(os.environ.get("RANK", "0"))
    if rank != 0:
        return
    cores = host_cores()
    x = W.make_inputs(w, seed=0)
    # each step: the oracle's sequential stepping on all host cores over one
    # batch row and 32 channels per thread (at most all of them) -- a bounded
    # sample, so that the whole run stays within minutes
    chans = min(w.D, 32 * cores)
    vals, desc = [], ""
    for i in range(args.warmup + args.steps):
        v, _, desc = time_oracle_seq(w, x, 1, chans, cores)
        if i >= args.warmup:
            vals.append(v)
    value = statistics.median(vals)
    line = {
        "impl": "reference", "metric": METRIC, "value": value, "unit": UNIT, "n_gpus": args.gpus,
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": 1e3 * (w.L * chans) / value,
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f64", "data": "synthetic",
        "config": {"workload": w.name},
        "cpu_baseline": {"value": value, "unit": UNIT, "cores": cores, "kind": "oracle", "sample": desc},
        "e2e": {"value": value, "unit": UNIT, "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
    }
    print(json.dumps(line), flush=True)


def run_e2e(w, x, dev, steps, nbuf=2):
    """The metric end to end through the public API: every step copies its
    inputs from pinned host memory to the device, runs the step and copies
    the states back to pinned host memory.  Steps are pipelined over `nbuf`
    sets of device buffers and three streams (host-to-device copies, compute,
    device-to-host copies), so that step i's copies overlap the compute of its
    neighbours; every copy of every step stays inside the timed region, which
    runs from the first copy of the first step to the last copy of the last."""
    hu = x.u.pin_memory()
    ha = x.a.pin_memory()
    hh0 = None if x.h0 is None else x.h0.pin_memory()
    hdh = None if x.dh is None else x.dh.pin_memory()
    s_in, s_comp, s_out = (torch.cuda.Stream(dev) for _ in range(3))
    sets = []
    for _ in range(nbuf):
        xe = W.Inputs(u=torch.empty_like(hu, device=dev), a=torch.empty_like(ha, device=dev),
                      h0=None if hh0 is None else torch.empty_like(hh0, device=dev), c0=None,
                      dh=None if hdh is None else torch.empty_like(hdh, device=dev))
        st = Step(w, xe, dev, s_comp)
        hout = [torch.empty((w.B, w.L, w.D), dtype=torch.float32).pin_memory() for _ in st.out]
        sets.append((xe, st, hout, torch.cuda.Event(), torch.cuda.Event(), torch.cuda.Event()))
    h2d = sum(t.numel() * t.element_size() for t in (hu, ha, hh0, hdh) if t is not None)
    d2h = sum(t.numel() * t.element_size() for t in sets[0][2])

    def one(i):
        xe, st, hout, ev_in, ev_comp, ev_out = sets[i % nbuf]
        s_in.wait_event(ev_comp)  # this set's inputs are free once its last step has run
        with torch.cuda.stream(s_in):
            for d, h in ((xe.u, hu), (xe.a, ha), (xe.h0, hh0), (xe.dh, hdh)):
                if h is not None:
                    d.copy_(h, non_blocking=True)
        ev_in.record(s_in)
        s_comp.wait_event(ev_in)
        s_comp.wait_event(ev_out)  # its outputs are free once they reached the host
        st()
        ev_comp.record(s_comp)
        s_out.wait_event(ev_comp)
        with torch.cuda.stream(s_out):
            for o, ho in zip(st.out, hout):
                ho.copy_(o, non_blocking=True)
        ev_out.record(s_out)

    for i in range(nbuf):
        one(i)
    torch.cuda.synchronize(dev)
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record(s_in)
    for i in range(steps):
        one(i)
    e1.record(s_out)
    torch.cuda.synchronize(dev)
    st0 = sets[0][1].result()
    if st0[0] not in (0, 1):
        raise SystemExit(f"end-to-end solve failed: status {st0[0]}")
    return e0.elapsed_time(e1) / steps, h2d, d2h


HEADLINE = W.BY_NAME["gru_bf16_B1_L65536_D2048"]


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=20)
    ap.add_argument("--warmup", type=int, default=3)
    ap.add_argument("--impl", default="ours", choices=["ours", "reference"])
    ap.add_argument("--workload", default=HEADLINE.name, choices=sorted(W.BY_NAME))
    ap.add_argument("--no-extras", action="store_true", help="only the headline workload (the other solve "
                    "workloads run by default on one GPU)")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--e2e-steps", type=int, default=-1,
                    help="steps of the end-to-end run (-1: as many as --steps; 0: none)")
    ap.add_argument("--baselines", type=int, default=1, help="also time the sequential GPU kernel and "
                    "the plain linear scan on the headline's input (GRU workloads)")
    ap.add_argument("--decode", action="store_true", help="add the decode-step timings (CUDA graph of steps)")
    ap.add_argument("--cells", action="store_true", help="add the runtime-compiled user cells (GRU, LSTM sources)")
    ap.add_argument("--seq-segments", default="", help="comma list of R: the solve with each sequence split into "
                    "R segments (sequence sharding), run on this GPU one segment after another")
    ap.add_argument("--projection-only", action="store_true", help="only the solve from the layer input (fused "
                    "input projection against cuBLAS GEMM + solve), one JSON object; for profiling")
    args = ap.parse_args()
    args.warmup = max(args.warmup, 3)
    w = W.BY_NAME[args.workload]

    if args.impl == "reference":
        run_reference(args, w)
        return
    if args.projection_only:
        dev = torch.device("cuda", 0)
        torch.cuda.set_device(dev)
        print(json.dumps(run_projection(dev, torch.cuda.Stream(dev), reps=args.steps)), flush=True)
        return

    rank, world, local = dist_setup()
    dev = torch.device("cuda", local)
    torch.cuda.set_device(dev)
    from nonlinear_rnn_newton_b200 import capi

    x = W.make_inputs(w, seed=rank)
    xd = x.to(dev)
    stream = torch.cuda.Stream(dev)
    step = Step(w, xd, dev, stream)

    # warm-up (also validates the solve)
    for _ in range(args.warmup):
        step()
    st, iters, resid, resid0 = step.result()
    if st not in (0, 1):
        raise SystemExit(f"solve failed: status {st} ({capi.status_string(st)})")

    # timed region: K back-to-back steps on one stream, CUDA events around
    # each launch; inputs (> 126 MB) exceed L2, so no flush is needed
    nev = 3 if w.train else 2
    evs = events(args.steps, nev)
    barrier(world)
    torch.cuda.synchronize(dev)
    launches0 = capi.kernel_launch_count()
    with ClockSampler(local) as clk:
        t0 = torch.cuda.Event(enable_timing=True)
        t1 = torch.cuda.Event(enable_timing=True)
        t0.record(stream)
        for i in range(args.steps):
            step(evs[i])
        t1.record(stream)
        stream.synchronize()
    launches = capi.kernel_launch_count() - launches0
    barrier(world)
    torch.cuda.synchronize(dev)
    total_ms = max_over_ranks(t0.elapsed_time(t1), world)
    ms_per_step = total_ms / args.steps
    st2, iters2, resid2, _ = step.result()
    solve_ms = statistics.mean(e[0].elapsed_time(e[1]) for e in evs)
    adj_ms = statistics.mean(e[1].elapsed_time(e[2]) for e in evs) if w.train else None

    value = job_value(w.N, world, ms_per_step)
    peak, peak_kind = hbm_peak()
    # dominant kernel: the Newton solve (one launch per step)
    algo = solve_bytes(w, iters2)
    achieved = algo / (solve_ms * 1e-3) / 1e9
    kname = "newton_solve_ws_kernel"
    roofline = {"bound": "hbm", "achieved": achieved, "peak": peak, "unit": "GB/s", "frac": achieved / peak,
                "traffic": profile_traffic(kname, w.name), "peak_kind": peak_kind, "kernel": kname,
                "algorithmic_bytes_per_launch": algo, "kernel_ms_mean": solve_ms,
                "per_pass": per_pass(w, step.pass_times(), peak)}
    adjoint = None
    if w.train:
        ab = adjoint_bytes(w)
        adjoint = {"kernel_ms_mean": adj_ms, "algorithmic_bytes_per_launch": ab,
                   "achieved": ab / (adj_ms * 1e-3) / 1e9, "frac": ab / (adj_ms * 1e-3) / 1e9 / peak,
                   "traffic": profile_traffic("adjoint_ws_kernel", w.name)}

    e2e = None
    e2e_steps = args.steps if args.e2e_steps < 0 else args.e2e_steps
    if e2e_steps > 0:
        barrier(world)
        ems, h2d, d2h = run_e2e(w, x, dev, e2e_steps)
        ems = max_over_ranks(ems, world)
        e2e = {"value": job_value(w.N, world, ems), "unit": UNIT, "ms_per_step": ems,
               "h2d_bytes_per_step": h2d, "d2h_bytes_per_step": d2h, "steps": e2e_steps}

    baselines = None
    if args.baselines and w.cell == "gru":
        baselines = time_baselines(w, xd, step.out[0], stream, dev)
    del step, xd
    torch.cuda.empty_cache()

    # the other workloads and the CPU oracle: one GPU only (under torchrun
    # the ranks would wait for rank 0 at the process group's end)
    solo = rank == 0 and world == 1
    configs = run_configs(w, dev, stream) if (solo and not args.no_extras) else None
    decode = run_decode(dev, stream) if (args.decode and solo) else None
    cells = run_cells(dev, stream) if (args.cells and solo) else None
    segments = None
    if args.seq_segments and solo:
        xs = x.to(dev)
        segments = run_segments(w, xs, dev, stream, [int(v) for v in args.seq_segments.split(",")])
        del xs
    cpu = cpu_baselines(w, x) if (solo and not args.no_cpu_baseline) else None

    if rank == 0:
        line = {
            "metric": METRIC, "value": value, "unit": UNIT, "n_gpus": world, "steps": args.steps,
            "warmup": args.warmup, "ms_per_step": ms_per_step, "higher_is_better": True, "scaling": "weak",
            "vs_baseline": None, "dtype": "f32", "data": "synthetic",
            "config": {"workload": w.name, "cell": w.cell, "B": w.B, "L": w.L, "D": w.D, "u_dtype": w.u_dtype,
                       "state_dtype": "f32", "tol": w.tol, "max_iters": w.max_iters,
                       "step": "Newton solve" + (" + adjoint" if w.train else ""),
                       "l2": "inputs larger than L2 (gates + states > 126 MB); no flush",
                       "per_rank": "independent problem, seed = rank", "parallelism": f"replicas x{world}"},
            "iters": iters2, "residual": resid2, "status": st2,
            "roofline": roofline,
            "adjoint": adjoint,
            "gpu_launches": launches,
            "clocks": clk.summary(),
            "e2e": e2e,
            "cpu_baseline": cpu,
            "baselines": baselines,
            "configs": configs,
            "decode": decode,
            "user_cells": cells,
            "seq_segments": segments,
        }
        print(json.dumps(line), flush=True)
    if world > 1:
        import torch.distributed as dist
        dist.destroy_process_group()


if __name__ == "__main__":
    main()
