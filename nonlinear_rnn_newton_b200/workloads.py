"""Seeded synthetic inputs for the ParaGRU / ParaLSTM Newton-solve workloads.

This module only draws random numbers; it holds none of the method's
arithmetic.  It is the one module that both the CUDA path's tests/benchmark
and the CPU oracle's tests consume, so both sides see bit-identical inputs.

Recipe (all draws from one ``torch.Generator`` on the CPU, in float32, in the
order u, a, h0 (then c0), dh):
  * u  ~ N(0, 1), shape [B, L, G, D] (G = 3 gates z,r,c for the GRU, 4 gates
    i,f,o,g for the LSTM), biases folded in; rounded to bfloat16 with
    round-to-nearest-even where the workload is bf16;
  * a  ~ U(-0.5, 0.5), shape [G, D] (the diagonal recurrence weights);
  * h0 ~ N(0, 0.1) (0.1 read as the standard deviation) where the workload
    asks for it, else zeros; c0 = 0 for the LSTM workloads;
  * dh ~ N(0, 1), shape [B, L, D], float32 (upstream gradient) for training.
The pages publish no dataset for this path; these synthetic inputs are the
workloads themselves.
"""
from dataclasses import dataclass, field
from typing import Optional

import torch


@dataclass(frozen=True)
class Workload:
    name: str
    cell: str           # "gru" or "lstm"
    B: int
    L: int
    D: int
    u_dtype: str        # "f32" or "bf16"
    h0_std: float = 0.0  # 0 -> h0 = 0
    tol: float = 1e-6
    max_iters: int = 10
    train: bool = False  # draw an upstream gradient dh as well

    @property
    def G(self) -> int:
        return 3 if self.cell == "gru" else 4

    @property
    def N(self) -> int:
        return self.B * self.L * self.D


GRU_SMALL = Workload("gru_f32_B2_L256_D64", "gru", 2, 256, 64, "f32")
GRU = Workload("gru_bf16_B8_L4096_D1024", "gru", 8, 4096, 1024, "bf16", h0_std=0.1)
LSTM = Workload("lstm_bf16_B8_L4096_D1024", "lstm", 8, 4096, 1024, "bf16")
GRU_SWEEP = tuple(
    Workload(f"gru_bf16_B1_L{L}_D2048", "gru", 1, L, 2048, "bf16", h0_std=0.1)
    for L in (512, 2048, 8192, 32768, 65536))
LSTM_TRAIN = Workload("lstm_train_bf16_B4_L16384_D2048", "lstm", 4, 16384, 2048, "bf16",
                      train=True)
# the ParaGRU training step (solve plus adjoint) at the same shape
GRU_TRAIN = Workload("gru_train_bf16_B4_L16384_D2048", "gru", 4, 16384, 2048, "bf16", h0_std=0.1,
                     train=True)

# the training workloads at L/4 and D/2 (an eighth of their elements): about
# 0.5 GB on the device, still larger than L2 -- a size a full profiler
# capture of the adjoint handles
LSTM_TRAIN_SMALL = Workload("lstm_train_bf16_B4_L4096_D1024", "lstm", 4, 4096, 1024, "bf16", train=True)
GRU_TRAIN_SMALL = Workload("gru_train_bf16_B4_L4096_D1024", "gru", 4, 4096, 1024, "bf16", h0_std=0.1,
                           train=True)
ALL = (GRU_SMALL, GRU, LSTM) + GRU_SWEEP + (LSTM_TRAIN, GRU_TRAIN, LSTM_TRAIN_SMALL, GRU_TRAIN_SMALL)
BY_NAME = {w.name: w for w in ALL}


def custom(cell: str, B: int, L: int, D: int, u_dtype: str = "bf16",
           h0_std: float = 0.0, train: bool = False, tol: float = 1e-6,
           max_iters: int = 10) -> Workload:
    return Workload(f"{cell}_{u_dtype}_B{B}_L{L}_D{D}", cell, B, L, D, u_dtype,
                    h0_std=h0_std, tol=tol, max_iters=max_iters, train=train)


@dataclass
class Inputs:
    u: torch.Tensor                 # [B,L,G,D] float32 or bfloat16
    a: torch.Tensor                 # [G,D] float32
    h0: Optional[torch.Tensor]      # [B,D] float32 or None (zeros)
    c0: Optional[torch.Tensor] = None
    dh: Optional[torch.Tensor] = None
    extra: dict = field(default_factory=dict)

    def to(self, device, non_blocking=False):
        mv = lambda t: None if t is None else t.to(device, non_blocking=non_blocking)
        return Inputs(mv(self.u), mv(self.a), mv(self.h0), mv(self.c0), mv(self.dh))


def make_inputs(w: Workload, seed: int = 0, a_scale: float = 1.0) -> Inputs:
    """Draw the workload's inputs on the CPU.  ``a_scale`` multiplies the
    recurrence weights after drawing (0 gives the zero-weight special case)."""
    g = torch.Generator().manual_seed(seed)
    u = torch.randn((w.B, w.L, w.G, w.D), generator=g, dtype=torch.float32)
    if w.u_dtype == "bf16":
        u = u.to(torch.bfloat16)
    elif w.u_dtype != "f32":
        raise ValueError(f"unknown u dtype {w.u_dtype}")
    a = torch.rand((w.G, w.D), generator=g, dtype=torch.float32) - 0.5
    if a_scale != 1.0:
        a = a * a_scale
    h0 = None
    if w.h0_std > 0:
        h0 = torch.randn((w.B, w.D), generator=g, dtype=torch.float32) * w.h0_std
    c0 = None
    dh = None
    if w.train:
        dh = torch.randn((w.B, w.L, w.D), generator=g, dtype=torch.float32)
    return Inputs(u=u, a=a, h0=h0, c0=c0, dh=dh)


@dataclass
class ProjectionInputs:
    x: torch.Tensor                 # [B,L,Din] bfloat16
    w: torch.Tensor                 # [3,D,Din] bfloat16
    bias: Optional[torch.Tensor]    # [3,D] float32 or None
    a: torch.Tensor                 # [3,D] float32
    h0: Optional[torch.Tensor]      # [B,D] float32 or None

    def to(self, device):
        mv = lambda t: None if t is None else t.to(device)
        return ProjectionInputs(mv(self.x), mv(self.w), mv(self.bias), mv(self.a), mv(self.h0))


def make_projection_inputs(B: int, L: int, Din: int, D: int, seed: int = 0, h0_std: float = 0.1,
                           bias_std: float = 0.1) -> ProjectionInputs:
    """Inputs of the ParaGRU layer fed through its input projection, drawn on
    the CPU in the order x, w, bias, a, h0: x ~ N(0,1) and w ~ N(0, 1/Din),
    both rounded to bfloat16, so that the gate pre-activations x w^T are
    about N(0,1) like the solve workloads' u; bias ~ N(0, bias_std) (None if
    0); a ~ U(-0.5,0.5); h0 ~ N(0, h0_std) (None if 0)."""
    g = torch.Generator().manual_seed(seed)
    x = torch.randn((B, L, Din), generator=g, dtype=torch.float32).to(torch.bfloat16)
    w = (torch.randn((3, D, Din), generator=g, dtype=torch.float32) / Din ** 0.5).to(torch.bfloat16)
    bias = torch.randn((3, D), generator=g, dtype=torch.float32) * bias_std if bias_std > 0 else None
    a = torch.rand((3, D), generator=g, dtype=torch.float32) - 0.5
    h0 = torch.randn((B, D), generator=g, dtype=torch.float32) * h0_std if h0_std > 0 else None
    return ProjectionInputs(x, w, bias, a, h0)

