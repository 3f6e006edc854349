"""Seeded synthetic inputs for the weight-quantized matmul.

This module only draws random numbers and names workload shapes.  It holds none
of the quantization or matmul arithmetic, so both the CUDA path and the CPU
oracle may take their inputs from it.

Recipe (all tensors are drawn on the CPU with ``torch.Generator().manual_seed``):

* weights ``W``: float32 ``[N, K]`` ~ N(0, 0.02^2), seed 0 by default;
* activations ``A``: float32 ``[M, K]`` ~ N(0, 1), seed 1, then optionally
  ``round(outlier_frac * K)`` outlier channels (column indices drawn by a
  ``randperm`` with seed 2) multiplied by ``outlier_gain`` (20), then cast to
  fp16 / bf16 (round to nearest even);
* no public dataset or checkpoint is used: the Llama-7B / BitNet-3B layer
  shapes below stand in for real layers of those models.
"""
from __future__ import annotations

from dataclasses import dataclass, field

import torch


def weights(N: int, K: int, seed: int = 0, std: float = 0.02) -> torch.Tensor:
    g = torch.Generator().manual_seed(seed)
    return torch.randn(N, K, generator=g, dtype=torch.float32) * std


def outlier_channels(K: int, frac: float, seed: int = 2) -> torch.Tensor:
    count = int(round(frac * K))
    g = torch.Generator().manual_seed(seed)
    return torch.randperm(K, generator=g)[:count]


def activations(M: int, K: int, seed: int = 1, dtype: torch.dtype = torch.float16,
                outlier_frac: float = 0.0, outlier_gain: float = 20.0, outlier_seed: int = 2) -> torch.Tensor:
    g = torch.Generator().manual_seed(seed)
    a = torch.randn(M, K, generator=g, dtype=torch.float32)
    if outlier_frac > 0:
        a[:, outlier_channels(K, outlier_frac, outlier_seed)] *= outlier_gain
    return a.to(dtype)


def uniform_bytes(shape, seed: int) -> torch.Tensor:
    """Uniformly random uint8 values (any packed code pattern)."""
    g = torch.Generator().manual_seed(seed)
    return torch.randint(0, 256, tuple(shape), generator=g, dtype=torch.uint8)


# --------------------------------------------------------------------------
# Workload shapes.  mode: "a16" (fp16/bf16 activations), "a8" (int8 per-token
# activations) or "f8" (FP8 e4m3 per-token activations, with "e4m3" weights); quant: "sym4" (symmetric INT4, group scales), "asym4"
# (INT4 with group scales and zero points), "tern2" (ternary, 2-bit codes,
# one scale per tensor), "int1" (binary, 1-bit codes, one scale per tensor),
# "e2m1" (FP4 codes, group scales) or "e4m3" (FP8 codes, group scales).
# --------------------------------------------------------------------------
@dataclass(frozen=True)
class Case:
    M: int
    N: int
    K: int
    mode: str = "a16"
    quant: str = "sym4"
    a_dtype: torch.dtype = torch.float16
    group_size: int = 128
    outlier_frac: float = 0.0
    bias: bool = False

    @property
    def name(self) -> str:
        dt = {torch.float16: "f16", torch.bfloat16: "bf16"}[self.a_dtype]
        a = self.mode if self.mode in ("a8", "f8") else dt
        return f"{self.quant}-{a}-M{self.M}-N{self.N}-K{self.K}"


@dataclass(frozen=True)
class Workload:
    name: str
    description: str
    cases: tuple = field(default_factory=tuple)


LLAMA7B_NK = ((4096, 4096), (11008, 4096), (4096, 11008))
BITNET3B_NK = ((3200, 3200), (8640, 3200), (3200, 8640))
# bits per weight of each quant kind
QUANT_BITS = {"sym4": 4, "asym4": 4, "tern2": 2, "int1": 1, "e2m1": 4, "e4m3": 8}

WORKLOADS = {
    "gemv-small": Workload(
        "gemv-small", "W4A16 GEMV M=1 N=256 K=512, fp16 activations, symmetric INT4 g128",
        (Case(1, 256, 512, "a16", "sym4"),)),
    "decode-llama7b": Workload(
        "decode-llama7b",
        "W4A16 decode GEMV on Llama-7B layer shapes: M in {1,4,16}, (N,K) in "
        "{(4096,4096),(11008,4096),(4096,11008)}, fp16 activations with 1% outlier "
        "channels x20, asymmetric INT4 g128 with fp16 scale+zero",
        tuple(Case(M, N, K, "a16", "asym4", outlier_frac=0.01)
              for M in (1, 4, 16) for (N, K) in LLAMA7B_NK)),
    "w4a8": Workload(
        "w4a8", "W4A8: M in {16,128}, N=K=4096, per-token INT8 activations, symmetric INT4 g128",
        tuple(Case(M, 4096, 4096, "a8", "sym4") for M in (16, 128))),
    "prefill-llama7b": Workload(
        "prefill-llama7b",
        "W4A16 prefill GEMM: M in {512,2048}, (N,K) in {(4096,4096),(12288,4096),(11008,4096)}, "
        "bf16 activations, INT4 g128 scale+zero, bf16 out",
        tuple(Case(M, N, K, "a16", "asym4", a_dtype=torch.bfloat16)
              for M in (512, 2048) for (N, K) in ((4096, 4096), (12288, 4096), (11008, 4096)))),
    "bitnet3b": Workload(
        "bitnet3b",
        "BitNet-3B-shaped ternary sweep: 2-bit codes packed 4/byte, one scale per tensor, "
        "M in {1,128}, (N,K) in {(3200,3200),(8640,3200),(3200,8640)}, fp16 and INT8 activations",
        tuple(Case(M, N, K, mode, "tern2")
              for mode in ("a16", "a8") for M in (1, 128) for (N, K) in BITNET3B_NK)),
    "formats-decode": Workload(
        "formats-decode",
        "The other weight types at decode: FP16 x FP4 (e2m1, g128 scales), FP16 x FP8 (e4m3, g128 "
        "scales) and FP16 x INT1 (binary, one scale) at M=1 on the Llama-7B shapes, and INT8 x INT1 "
        "(M=1, N=K=4096), FP8 x FP8 (e4m3 activations per token, M=1, N=4096 and 11008, K=4096); fp16 "
        "activations with 1% outlier channels x20 (quantized inside the step on the INT8 / FP8 paths)",
        tuple(Case(1, N, K, "a16", q, outlier_frac=0.01) for q in ("e2m1", "e4m3", "int1")
              for (N, K) in LLAMA7B_NK) + (Case(1, 4096, 4096, "a8", "int1", outlier_frac=0.01),)
        + tuple(Case(1, N, 4096, "f8", "e4m3", outlier_frac=0.01) for N in (4096, 11008))),
    "formats-prefill": Workload(
        "formats-prefill",
        "The other weight types at prefill: FP16 x FP4 (e2m1), FP16 x FP8 (e4m3) and FP16 x INT1 at "
        "M=512, (N,K) in {(4096,4096),(11008,4096)}, INT8 x INT1 at M=128, N=K=4096, and FP8 x FP8 "
        "(e4m3 activations per token) at M=512 on the same two shapes",
        tuple(Case(512, N, K, "a16", q) for q in ("e2m1", "e4m3", "int1")
              for (N, K) in ((4096, 4096), (11008, 4096))) + (Case(128, 4096, 4096, "a8", "int1"),)
        + tuple(Case(512, N, 4096, "f8", "e4m3") for N in (4096, 11008))),
}
