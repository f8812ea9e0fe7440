"""Seeded synthetic inputs and workload shapes for the FP8 linear layer.

Shared by the tests, the oracle checks and ``bench.py``.  It holds no part of
the method's arithmetic (no amax, no scaling, no fp8 cast): only the shapes of
the workloads and seeded random bf16 tensors drawn with torch's CPU generator.

Seed rule: ``20261202 + 1000*config + 10*step + operand`` with operand ids
x=0, w=1, g=2, bias=3, outlier mask=4, per-step std=5.  Values are drawn in
fp32 and rounded to bf16 by torch's cast.
"""
from __future__ import annotations

import math
from dataclasses import dataclass

import torch

OP_X, OP_W, OP_G, OP_BIAS, OP_MASK, OP_STD = 0, 1, 2, 3, 4, 5


def seed_for(config: int, step: int, operand: int, extra: int = 0) -> int:
    return 20261202 + 1000 * config + 10 * step + operand + 100000 * extra


def normal(shape, std: float, seed: int, dtype=torch.bfloat16) -> torch.Tensor:
    """N(0, std^2) samples, drawn in fp32 with a seeded CPU generator, cast to dtype."""
    g = torch.Generator().manual_seed(seed)
    return (torch.randn(*shape, generator=g, dtype=torch.float32) * std).to(dtype)


def normal_with_outliers(shape, std: float, seed: int, mask_seed: int, p: float = 1e-3,
                         factor: float = 50.0, dtype=torch.bfloat16) -> torch.Tensor:
    """N(0, std^2) with a Bernoulli(p) subset of elements multiplied by factor."""
    g = torch.Generator().manual_seed(seed)
    v = torch.randn(*shape, generator=g, dtype=torch.float32) * std
    gm = torch.Generator().manual_seed(mask_seed)
    mask = torch.rand(*shape, generator=gm) < p
    v = torch.where(mask, v * factor, v)
    return v.to(dtype)


def log_uniform(lo: float, hi: float, seed: int) -> float:
    g = torch.Generator().manual_seed(seed)
    u = torch.rand(1, generator=g, dtype=torch.float64).item()
    return math.exp(math.log(lo) + u * (math.log(hi) - math.log(lo)))


@dataclass(frozen=True)
class LinearShape:
    name: str
    M: int
    K: int   # in_features
    N: int   # out_features


# Config 1: single linear, 4 delayed-scaling steps, x ~ N(0,1) * 2^step.
C1 = LinearShape("c1", 64, 128, 192)
C1_STEPS = 4

# Config 2: dim1024 transformer layer (12L/dim1024, B4xT512 -> M=2048 tokens).
C2_LAYER = (
    LinearShape("q", 2048, 1024, 1024),
    LinearShape("k", 2048, 1024, 1024),
    LinearShape("v", 2048, 1024, 1024),
    LinearShape("o", 2048, 1024, 1024),
    LinearShape("up", 2048, 1024, 4096),
    LinearShape("down", 2048, 4096, 1024),
)
C2_SHAPES = (C2_LAYER[0], C2_LAYER[4], C2_LAYER[5])

# Config 3: production 24L/dim1536/ffn6912 linears at M in {512, 2048}, fp8 bias.
C3_SHAPES = tuple(LinearShape(f"m{M}_{K}x{N}", M, K, N)
                  for M in (512, 2048) for (K, N) in ((1536, 1536), (1536, 6912), (6912, 1536)))

# Config 4: generic large shapes at M=4096, x with 0.1% outliers x50.
C4_SHAPES = tuple(LinearShape(f"m4096_{K}x{N}", 4096, K, N)
                  for (K, N) in ((4096, 11008), (11008, 4096), (4096, 4096)))

# Config 5: 20 steps over a 12-layer dim1024 stack (6 linears per layer), plus
# odd-K edge shapes.
C5_STEPS = 20
C5_LAYERS = 12
C5_LAYER = C2_LAYER
C5_EDGE = tuple(LinearShape(f"edge_m{M}_k{K}_n{N}", M, K, N)
                for K in (7, 100, 1534) for M in (3, 64, 2048) for N in (1024, 100))

HIST_LEN = 16


def weight_std(K: int) -> float:
    """w ~ N(0, 1/sqrt(K)): the std is 1/sqrt(K)."""
    return 1.0 / math.sqrt(K)


def normal_device(shape, std: float, seed: int, device, dtype=torch.bfloat16) -> torch.Tensor:
    """N(0, std^2) drawn in fp32 by a seeded generator on `device`, cast to dtype
    (for large benchmark inputs; the tests use the CPU generator above)."""
    g = torch.Generator(device=device).manual_seed(seed)
    return (torch.randn(*shape, generator=g, dtype=torch.float32, device=device) * std).to(dtype)


def normal_with_outliers_device(shape, std: float, seed: int, mask_seed: int, device, p: float = 1e-3,
                                factor: float = 50.0, dtype=torch.bfloat16) -> torch.Tensor:
    """normal_with_outliers drawn by seeded generators on `device` (for large
    benchmark inputs)."""
    g = torch.Generator(device=device).manual_seed(seed)
    v = torch.randn(*shape, generator=g, dtype=torch.float32, device=device) * std
    gm = torch.Generator(device=device).manual_seed(mask_seed)
    mask = torch.rand(*shape, generator=gm, device=device) < p
    return torch.where(mask, v * factor, v).to(dtype)


# Benchmark workload: the linears of the pages' 12L/dim1024/B4xT512 model
# (configuration 2), forward and backward, with a bf16 bias and its gradient.
BENCH_LAYERS = 12
BENCH_LAYER = C2_LAYER
BENCH_BIAS_STD = 0.01
