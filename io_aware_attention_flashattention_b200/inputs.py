"""Seeded synthetic inputs and the named workloads.

This module holds no attention arithmetic: it only draws the random tensors that
both the CUDA path and the fp64 oracle consume, so that both see the same bits.

Recipe (every workload): ``torch.Generator().manual_seed(seed)`` on the CPU, then
four fp32 ``randn`` draws of shape [B, H, N, d] in the order Q, K, V, dO; Q and K
are multiplied by ``qk_gain`` (8 for the numerical-stress workload, else 1) before
the cast to the workload's dtype (round-to-nearest-even). The shapes are those of
the benchmark harness in "Flash Attention-2: acceleration principle and GPU memory
optimisation in deployment" (B=1, H=8, d=128, N from 2K to 16K) and the GPT-2
shape (N=1024, d=64) quoted in "A survey of key techniques of large language model
pre-training systems", Journal of Software 2026(1), p.218.
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
    dtype: torch.dtype
    causal: bool
    scale: float
    seed: int
    qk_gain: float = 1.0
    backward: bool = True

    @property
    def shape(self):
        return (self.B, self.H, self.N, self.d)

    def fwd_flops(self) -> float:
        """4*B*H*N^2*d, halved when causal (the counting convention of the metric)."""
        f = 4.0 * self.B * self.H * self.N * self.N * self.d
        return f / 2 if self.causal else f

    def bwd_flops(self) -> float:
        """2.5x the forward count."""
        return 2.5 * self.fwd_flops()


# The five workloads; workload k (1-based) draws with seed 1000 + k.
WORKLOADS = {
    "oracle_f32_n256_d64": Workload("oracle_f32_n256_d64", 1, 1, 256, 64, torch.float32,
                                    False, 1.0 / math.sqrt(64), 1001),
    "gpt2_causal_b8h12_n1024_d64": Workload("gpt2_causal_b8h12_n1024_d64", 8, 12, 1024, 64,
                                            torch.bfloat16, True, 1.0 / 8.0, 1002),
    "mid_b1h8_n4096_d128": Workload("mid_b1h8_n4096_d128", 1, 8, 4096, 128, torch.bfloat16,
                                    False, 1.0 / math.sqrt(128), 1003),
    "stress_causal_b2h16_n8192_d128_qk8": Workload(
        "stress_causal_b2h16_n8192_d128_qk8", 2, 16, 8192, 128, torch.bfloat16, True,
        1.0 / math.sqrt(128), 1004, qk_gain=8.0, backward=False),
    "long_b1h8_n16384_d128": Workload("long_b1h8_n16384_d128", 1, 8, 16384, 128,
                                      torch.bfloat16, False, 1.0 / math.sqrt(128), 1005),
}
WORKLOAD_ORDER = list(WORKLOADS)


def make_inputs(B: int, H: int, N: int, d: int, dtype: torch.dtype, seed: int,
                qk_gain: float = 1.0):
    """(Q, K, V, dO) as CPU tensors of ``dtype``, drawn as the module docstring says."""
    g = torch.Generator().manual_seed(int(seed))
    shape = (B, H, N, d)
    q = torch.randn(shape, generator=g, dtype=torch.float32)
    k = torch.randn(shape, generator=g, dtype=torch.float32)
    v = torch.randn(shape, generator=g, dtype=torch.float32)
    do = torch.randn(shape, generator=g, dtype=torch.float32)
    if qk_gain != 1.0:
        q = q * qk_gain
        k = k * qk_gain
    return q.to(dtype), k.to(dtype), v.to(dtype), do.to(dtype)


def make_inputs_device(B: int, H: int, N: int, d: int, dtype: torch.dtype, seed: int,
                       device="cuda"):
    """(Q, K, V, dO) drawn directly on a CUDA device, for shapes too large to stage
    in host memory: ``torch.Generator(device).manual_seed(seed)`` and four ``randn``
    draws of [B, H, N, d] in ``dtype``, in the order Q, K, V, dO. The oracle reads
    back whichever slices it checks, so both sides still see the same bits."""
    g = torch.Generator(device=device).manual_seed(int(seed))
    shape = (B, H, N, d)
    return tuple(torch.randn(shape, generator=g, dtype=dtype, device=device) for _ in range(4))


def workload_inputs(w: Workload):
    return make_inputs(w.B, w.H, w.N, w.d, w.dtype, w.seed, w.qk_gain)
