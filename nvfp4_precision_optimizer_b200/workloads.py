"""Seeded synthetic momentum matrices for the benchmark and parity workloads.

This module only generates inputs; it holds none of the method's arithmetic.
The shapes are those of a 3B-class decoder (hidden 3072, FFN 8192): per block
Q, K, V, O are 3072 x 3072, gate and up 8192 x 3072, down 3072 x 8192.  The
values stand in for optimizer momenta (the pages' own momenta come from
pretraining runs that are not reproduced): N(0, 0.02^2), optionally with 0.1%
of entries scaled by 50 as outliers, or Student-t (nu = 3) rescaled to an
empirical RMS of exactly 0.02.
"""
from __future__ import annotations

from dataclasses import dataclass, field

import torch

MUON = (3.4445, -4.7750, 2.0315)
BLOCK_SHAPES = [(3072, 3072)] * 4 + [(8192, 3072), (8192, 3072), (3072, 8192)]
BASE_SEED = 20260705


@dataclass
class Workload:
    name: str
    shapes: list
    dist: str
    K: int = 5
    clip_k: float = 3.0
    coeffs: list = field(default_factory=list)

    def __post_init__(self):
        if not self.coeffs:
            self.coeffs = [MUON] * len(self.shapes)

    def flops_algorithmic(self) -> float:
        """Products the method takes: per iteration m(m+1)n (Gram, symmetric half),
        m(m+1)m (second Gram) and 2m^2 n (update), m = min side."""
        tot = 0.0
        for (r, c) in self.shapes:
            m, n = min(r, c), max(r, c)
            tot += self.K * (m * (m + 1) * n + m * (m + 1) * m + 2 * m * m * n)
        return tot

    def flops_dense(self) -> float:
        """The same products without exploiting symmetry: 4 m^2 n + 2 m^3 per iteration."""
        tot = 0.0
        for (r, c) in self.shapes:
            m, n = min(r, c), max(r, c)
            tot += self.K * (4 * m * m * n + 2 * m ** 3)
        return tot


WORKLOADS = {
    "single_256x256_gauss": Workload("single_256x256_gauss", [(256, 256)], "gauss"),
    "single_1024x4096_outliers": Workload("single_1024x4096_outliers", [(1024, 4096)], "outliers"),
    "3b_1block_gauss": Workload("3b_1block_gauss", BLOCK_SHAPES, "gauss"),
    "3b_4blocks_gauss": Workload("3b_4blocks_gauss", BLOCK_SHAPES * 4, "gauss"),
    "3b_28blocks_student": Workload("3b_28blocks_student", BLOCK_SHAPES * 28, "student"),
    "single_8192x8192_student": Workload("single_8192x8192_student", [(8192, 8192)], "student"),
}


def generate(shape, dist: str, seed: int, device="cpu") -> torch.Tensor:
    """One FP32 momentum matrix drawn with torch's generator on `device`."""
    g = torch.Generator(device=device)
    g.manual_seed(seed)
    if dist == "gauss":
        return torch.randn(shape, generator=g, device=device) * 0.02
    if dist == "outliers":
        x = torch.randn(shape, generator=g, device=device) * 0.02
        mask = torch.rand(shape, generator=g, device=device) < 0.001
        return torch.where(mask, x * 50.0, x)
    if dist == "student":
        z = torch.randn(shape, generator=g, device=device)
        chi = torch.zeros(shape, device=device)
        for _ in range(3):
            chi += torch.randn(shape, generator=g, device=device) ** 2
        t = z / torch.sqrt(chi / 3.0)
        rms = torch.sqrt(torch.mean(t.double() ** 2)).float()
        return t * (0.02 / rms)
    raise ValueError(f"unknown distribution {dist!r}")


def matrices(w: Workload, device="cpu", seed: int = BASE_SEED) -> list:
    """All matrices of a workload; matrix i is seeded with seed + i."""
    return [generate(s, w.dist, seed + i, device) for i, s in enumerate(w.shapes)]
