"""Seeded synthetic inputs for the ParaGRU / ParaLSTM solve.

This module holds no arithmetic of the method: it only draws the tensors the
solver and the oracle both consume, so both sides read the same bytes.

Every tensor has its own CPU ``torch.Generator`` (u -> seed 0, a -> 1,
bias -> 2, dL/dh -> 3, offset by ``seed``); values are drawn in fp32 and, for
bf16 projections, rounded to bf16 with round-to-nearest-even by ``Tensor.to``.
Shapes are those of language-model layers: u is the precomputed gate input
projection ``[B, T, G, D]`` (G = 3 for ParaGRU z,r,c; 4 for ParaLSTM i,f,g,o),
a and bias are ``[G, D]``, h0 / c0 ``[B, D]`` and dL/dh ``[B, T, D]``.
"""
from dataclasses import dataclass, replace
import math

import torch


@dataclass(frozen=True)
class Workload:
    name: str
    cell: str          # "gru" | "lstm"
    B: int
    T: int
    D: int
    u_dtype: str       # "bf16" | "f32"
    u_std: float
    a_range: float     # a ~ U(-a_range, a_range)
    bias: str          # "zero" | "normal0.1" | "forget1"
    adjoint: bool
    histogram: bool = False

    @property
    def G(self) -> int:
        return 3 if self.cell == "gru" else 4

    @property
    def tokch(self) -> int:
        return self.B * self.T * self.D

    def scaled(self, B=None, T=None, D=None) -> "Workload":
        """Same recipe at another shape (parity cases)."""
        return replace(self, B=B or self.B, T=T or self.T, D=D or self.D,
                       name=f"{self.name}@{B or self.B}x{T or self.T}x{D or self.D}")


def _cfg5_std(D: int) -> float:
    # "N(0, 1/sqrt(D)*4)": read with standard precedence as 4/sqrt(D).
    return 4.0 / math.sqrt(D)


WORKLOADS = {
    1: Workload("gru_b1_t256_d64_f32", "gru", 1, 256, 64, "f32", 1.0, 1.0,
                "zero", False),
    2: Workload("gru_b8_t4096_d1024_bf16", "gru", 8, 4096, 1024, "bf16", 1.0,
                1.0, "normal0.1", True),
    3: Workload("lstm_b8_t4096_d1024_bf16", "lstm", 8, 4096, 1024, "bf16", 1.0,
                1.0, "forget1", False),
    4: Workload("gru_b1_t65536_d2048_f32", "gru", 1, 65536, 2048, "f32", 1.0,
                0.9, "zero", False, histogram=True),
    5: Workload("lstm_b4_t2048_d4096_bf16", "lstm", 4, 2048, 4096, "bf16",
                _cfg5_std(4096), 1.0, "forget1", True),
}


def _gen(seed: int) -> torch.Generator:
    g = torch.Generator(device="cpu")
    g.manual_seed(seed)
    return g


def make_inputs(w: Workload, seed: int = 0, device="cpu",
                with_grad: bool = False) -> dict:
    """Draw u, a, bias, h0 (and c0 for LSTM) and dLdh for workload ``w``.

    Returned tensors live on ``device``; u is bf16 or fp32, the rest fp32.
    """
    G, B, T, D = w.G, w.B, w.T, w.D
    u = torch.randn((B, T, G, D), generator=_gen(seed + 0), dtype=torch.float32)
    if w.u_std != 1.0:
        u.mul_(w.u_std)
    u = u.to(torch.bfloat16) if w.u_dtype == "bf16" else u
    a = (torch.rand((G, D), generator=_gen(seed + 1), dtype=torch.float32)
         * (2.0 * w.a_range) - w.a_range)
    if w.bias == "zero":
        bias = torch.zeros((G, D), dtype=torch.float32)
    elif w.bias == "normal0.1":
        bias = torch.randn((G, D), generator=_gen(seed + 2),
                           dtype=torch.float32) * 0.1
    elif w.bias == "forget1":
        bias = torch.zeros((G, D), dtype=torch.float32)
        bias[1] = 1.0          # gate order i, f, g, o
    else:
        raise ValueError(w.bias)
    out = {"u": u, "a": a, "bias": bias,
           "h0": torch.zeros((B, D), dtype=torch.float32)}
    if w.cell == "lstm":
        out["c0"] = torch.zeros((B, D), dtype=torch.float32)
    if w.adjoint or with_grad:
        out["dLdh"] = torch.randn((B, T, D), generator=_gen(seed + 3),
                                  dtype=torch.float32)
    if device != "cpu":
        out = {k: v.to(device) for k, v in out.items()}
    return out
