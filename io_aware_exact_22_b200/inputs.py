"""Seeded synthetic workloads shared by the CUDA path's tests/bench and by the oracle's tests.

This module draws random inputs and describes workload shapes. It holds none of the
attention arithmetic, so both sides may take their inputs from it without sharing any
computation.

Recipe (one generator per workload, CPU, seed 0 unless stated):
  g = torch.Generator("cpu").manual_seed(seed)
  q, k, v (and dO for backward workloads) are drawn in that order with
  torch.randn(shape, generator=g, dtype=float32), multiplied by the workload's
  standard deviation (sqrt(3) for q and k of the long-sequence workload, whose
  distribution is N(0, 3), i.e. variance 3), then rounded to bf16.
Every consumer (GPU path and oracle) sees the same bf16 values; the oracle upcasts
them exactly to fp64.
"""
from __future__ import annotations

import math
from dataclasses import dataclass

import torch


@dataclass(frozen=True)
class Workload:
    name: str
    B: int
    H: int
    N: int
    d: int
    causal: bool
    backward: bool = False
    qk_std: float = 1.0
    seed: int = 0
    note: str = ""

    @property
    def scale(self) -> float:
        return 1.0 / math.sqrt(self.d)

    @property
    def shape(self):
        return (self.B, self.H, self.N, self.d)

    def fwd_flops(self) -> float:
        """Metric FLOPs of the forward: 4*B*H*N^2*d, halved when causal."""
        f = 4.0 * self.B * self.H * self.N * self.N * self.d
        return f / 2 if self.causal else f

    def bwd_flops(self) -> float:
        """Metric FLOPs of the backward: 2.5x the forward's."""
        return 2.5 * self.fwd_flops()

    def fwd_bytes(self) -> float:
        """Algorithmic HBM bytes of the forward: Q, K, V read and O written once
        (bf16), plus the fp32 per-row log-sum-exp."""
        n = self.B * self.H * self.N
        return 4.0 * n * self.d * 2 + n * 4

    def bwd_bytes(self) -> float:
        """Algorithmic HBM bytes of the backward: Q, K, V, O, dO read and dQ, dK, dV
        written once (bf16), plus the fp32 LSE read and the fp32 row term written and read."""
        n = self.B * self.H * self.N
        return 8.0 * n * self.d * 2 + n * 4 * 3


# The five workloads of the attention benchmark table (shapes, masks, distributions).
WORKLOADS = {
    1: Workload("single-head fwd B=1 H=1 N=256 d=64", 1, 1, 256, 64, False),
    2: Workload("multi-head fwd B=4 H=16 N=1024 d=64", 4, 16, 1024, 64, False),
    3: Workload("causal fwd B=2 H=16 N=4096 d=128", 2, 16, 4096, 128, True),
    4: Workload("long-sequence causal fwd B=1 H=32 N=16384 d=128, q,k ~ N(0,3)",
                1, 32, 16384, 128, True, qk_std=math.sqrt(3.0)),
    5: Workload("causal bwd B=2 H=16 N=4096 d=128", 2, 16, 4096, 128, True, backward=True),
}


def make_inputs(w: Workload, with_grad: bool | None = None):
    """Return bf16 CPU tensors (q, k, v[, dO]) of shape [B,H,N,d] for workload ``w``."""
    if with_grad is None:
        with_grad = w.backward
    g = torch.Generator("cpu").manual_seed(w.seed)
    shape = w.shape
    q = torch.randn(shape, generator=g, dtype=torch.float32) * w.qk_std
    k = torch.randn(shape, generator=g, dtype=torch.float32) * w.qk_std
    v = torch.randn(shape, generator=g, dtype=torch.float32)
    out = [q.to(torch.bfloat16), k.to(torch.bfloat16), v.to(torch.bfloat16)]
    if with_grad:
        do = torch.randn(shape, generator=g, dtype=torch.float32)
        out.append(do.to(torch.bfloat16))
    return tuple(out)


E4M3_MAX = 448.0  # largest finite FP8 E4M3 value


def make_fp8_inputs(w: Workload):
    """FP8 (E4M3) inputs for workload ``w``: q, k, v are drawn exactly as in make_inputs (same
    generator, order and standard deviations, in fp32), then each (b, h) slice x of each tensor
    is stored as E4M3 codes c = e4m3(x / descale) with descale = max|x| / 448, the conversion
    being torch's float8_e4m3fn cast (round to nearest even).  The slice then stands for
    c * descale.  Returns ((q8, k8, v8) uint8 code tensors [B,H,N,d],
    (descale_q, descale_k, descale_v) fp32 tensors [B,H]).  Codes and factors are the inputs
    of both the FP8 kernel and the oracle."""
    g = torch.Generator("cpu").manual_seed(w.seed)
    shape = w.shape
    xs = [torch.randn(shape, generator=g, dtype=torch.float32) * w.qk_std,
          torch.randn(shape, generator=g, dtype=torch.float32) * w.qk_std,
          torch.randn(shape, generator=g, dtype=torch.float32)]
    codes, descales = [], []
    for x in xs:
        amax = x.abs().amax(dim=(2, 3))
        ds = torch.where(amax > 0, amax / E4M3_MAX, torch.ones_like(amax))
        c = (x / ds[:, :, None, None]).to(torch.float8_e4m3fn).view(torch.uint8)
        codes.append(c)
        descales.append(ds.to(torch.float32))
    return tuple(codes), tuple(descales)


def custom(B: int, H: int, N: int, d: int, causal: bool, seed: int = 0,
           qk_std: float = 1.0, backward: bool = False) -> Workload:
    """An ad-hoc workload (used for ragged tails and edge cases in the tests)."""
    return Workload(f"custom B={B} H={H} N={N} d={d} causal={causal}", B, H, N, d, causal,
                    backward=backward, qk_std=qk_std, seed=seed)


def to_f64(t: torch.Tensor):
    """Exact upcast of a bf16 tensor to a float64 numpy array."""
    return t.to(torch.float64).numpy()
