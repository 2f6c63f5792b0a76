"""Seeded synthetic inputs and the five workload shapes.

This module holds no part of the method's arithmetic: it only draws random
numbers (numpy PCG64) and rounds them to bf16, so that the CUDA path and the
CPU oracle see identical bytes.  Both the tests and the benchmark use it.

Recipe (shared by every consumer):
  * one PCG64 stream per tensor: seed 0 for W, 1 for A, 2 for B, 3 for X, 4 for
    dY, plus 10 * projection index;
  * draw float32 standard normals, scale in float32, round to bf16 (RNE);
  * W ~ N(0, 0.02); A, B ~ N(0, 0.02); X, dY ~ N(0, 1);
  * the outlier workload sets exactly round(0.01 * numel) positions, chosen by
    a seeded permutation, to +-0.16 (8 sigma) with a seeded random sign.
"""
from __future__ import annotations

from dataclasses import dataclass, field

import numpy as np
import torch

W_STD = 0.02
AB_STD = 0.02
OUTLIER_FRACTION = 0.01
OUTLIER_VALUE = 0.16      # 8 sigma of N(0, 0.02)

SEED_W, SEED_A, SEED_B, SEED_X, SEED_DY = 0, 1, 2, 3, 4


def _normal_bf16(seed: int, shape, std: float) -> torch.Tensor:
    rng = np.random.Generator(np.random.PCG64(seed))
    a = rng.standard_normal(size=int(np.prod(shape)), dtype=np.float32)
    if std != 1.0:
        a *= np.float32(std)
    return torch.from_numpy(a.reshape(shape)).to(torch.bfloat16)


def weight(shape, proj: int = 0, outliers: bool = False) -> torch.Tensor:
    w = _normal_bf16(SEED_W + 10 * proj, shape, W_STD)
    if outliers:
        n = w.numel()
        k = int(round(OUTLIER_FRACTION * n))
        rng = np.random.Generator(np.random.PCG64(1000 + SEED_W + 10 * proj))
        pos = rng.permutation(n)[:k]
        sign = np.where(rng.integers(0, 2, size=k) == 1, 1.0, -1.0).astype(np.float32)
        flat = w.view(-1)
        flat[torch.from_numpy(pos)] = torch.from_numpy(sign * np.float32(OUTLIER_VALUE)).to(torch.bfloat16)
    return w


def lora_a(r: int, k: int, proj: int = 0) -> torch.Tensor:
    return _normal_bf16(SEED_A + 10 * proj, (r, k), AB_STD)


def lora_b(n: int, r: int, proj: int = 0) -> torch.Tensor:
    return _normal_bf16(SEED_B + 10 * proj, (n, r), AB_STD)


def activations(m: int, k: int, proj: int = 0) -> torch.Tensor:
    return _normal_bf16(SEED_X + 10 * proj, (m, k), 1.0)


def grad_output(m: int, n: int, proj: int = 0) -> torch.Tensor:
    return _normal_bf16(SEED_DY + 10 * proj, (m, n), 1.0)


def bf16_bits(t: torch.Tensor) -> np.ndarray:
    """The uint16 bit patterns of a bf16 CPU tensor (what the oracle reads)."""
    return t.contiguous().view(torch.int16).numpy().view(np.uint16)


@dataclass
class Projection:
    name: str
    n: int      # out features (rows of W)
    k: int      # in features


@dataclass
class Workload:
    name: str
    projections: list
    m: int                  # token rows
    r: int                  # LoRA rank
    alpha: float
    outliers: bool = False
    token_counts: list = field(default_factory=list)

    @property
    def s(self) -> float:
        return self.alpha / self.r


def _llama(hidden: int, ffn: int):
    return [Projection("q", hidden, hidden), Projection("k", hidden, hidden),
            Projection("v", hidden, hidden), Projection("o", hidden, hidden),
            Projection("gate", ffn, hidden), Projection("up", ffn, hidden),
            Projection("down", hidden, ffn)]


# The five workloads: a tiny layer, a codec round-trip, LLaMA-7B projections,
# LLaMA-65B-shaped decode GEMV, one LLaMA-65B decoder layer.
TINY = Workload("tiny_256x256_m16_r8", [Projection("w", 256, 256)], m=16, r=8, alpha=16.0)
CODEC_4096 = Workload("codec_4096x4096_outliers", [Projection("w", 4096, 4096)], m=0, r=0,
                      alpha=0.0, outliers=True)
LLAMA7B = Workload("llama7b_7proj_m8192_r64", _llama(4096, 11008), m=16 * 512, r=64, alpha=16.0)
GEMV65B = Workload("llama65b_ffn_gemv_r64", [Projection("ffn_up", 22016, 8192),
                                              Projection("ffn_down", 8192, 22016)],
                   m=16, r=64, alpha=16.0, token_counts=[1, 4, 16])
LLAMA65B = Workload("llama65b_layer_m8192_r64", _llama(8192, 22016), m=16 * 512, r=64, alpha=16.0)

ALL = [TINY, CODEC_4096, LLAMA7B, GEMV65B, LLAMA65B]


def linear_flops(n: int, k: int, m: int, r: int) -> dict:
    """Algorithmic FLOPs of one projection (dense + LoRA), forward and backward."""
    fwd = 2 * m * n * k + 2 * m * r * (n + k)
    bwd = 2 * m * n * k + 4 * m * r * (n + k)
    return dict(fwd=fwd, bwd=bwd, total=fwd + bwd)
