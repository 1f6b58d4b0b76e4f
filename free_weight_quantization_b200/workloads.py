"""Seeded synthetic weight matrices shaped like LLM projection weights.

This module holds input generators only (no quantization arithmetic), so that the CUDA path
and the CPU oracle can be fed the very same fp16 bytes.  The shapes follow the 4096-wide
hidden size and 11008-wide MLP of a 7B-class decoder; the page "HQQ 算法解读" runs its own
experiment on a 4096x4096 fp16 Linear (section "一个最小可复现实验").  Real checkpoints are not
used: these distributions stand in for them.

Recipe: samples drawn in float64 with numpy.random.default_rng(seed), then rounded once to
fp16 (round-to-nearest-even).
"""
from __future__ import annotations

from dataclasses import dataclass

import numpy as np


def outlier_normal(rows: int, cols: int, seed: int, sigma: float = 0.02,
                   outlier_frac: float = 0.001, lo: float = 0.2, hi: float = 1.0) -> np.ndarray:
    """N(0, sigma^2) with floor(outlier_frac*N) distinct entries replaced by +-U(lo, hi)."""
    rng = np.random.default_rng(seed)
    n = rows * cols
    w = rng.normal(0.0, sigma, n)
    k = int(np.floor(outlier_frac * n))
    pos = rng.choice(n, size=k, replace=False)
    mag = rng.uniform(lo, hi, k)
    sign = np.where(rng.random(k) < 0.5, -1.0, 1.0)
    w[pos] = sign * mag
    return w.reshape(rows, cols).astype(np.float16)


def student_t(rows: int, cols: int, seed: int, scale: float = 0.02, df: float = 4.0,
              clip: float = 1.0) -> np.ndarray:
    """scale * StudentT(df), clipped to +-clip (heavy-tailed, attention-projection-like)."""
    rng = np.random.default_rng(seed)
    w = scale * rng.standard_t(df, rows * cols)
    if clip is not None:
        w = np.clip(w, -clip, clip)
    return w.reshape(rows, cols).astype(np.float16)


def row_lognormal(rows: int, cols: int, seed: int, sigma: float = 0.015,
                  row_sigma: float = 0.3) -> np.ndarray:
    """N(0, sigma^2) times a per-row LogNormal(0, row_sigma) factor (MLP-like)."""
    rng = np.random.default_rng(seed)
    w = rng.normal(0.0, sigma, (rows, cols))
    w *= rng.lognormal(0.0, row_sigma, (rows, 1))
    return w.astype(np.float16)


@dataclass(frozen=True)
class Case:
    name: str
    rows: int
    cols: int
    nbits: int
    group_size: int
    axis: int
    gen: str          # generator name
    seed: int

    def make(self) -> np.ndarray:
        return GENERATORS[self.gen](self.rows, self.cols, self.seed)

    @property
    def n(self) -> int:
        return self.rows * self.cols


GENERATORS = {"outlier_normal": outlier_normal, "student_t": student_t,
              "row_lognormal": row_lognormal}

# The five workloads.  Each runs with iters <= 20, p = 0.7, beta = 10, kappa = 1.01.
SMALL = Case("outlier-normal 256x512 b4 g64 axis1", 256, 512, 4, 64, 1, "outlier_normal", 0)
ATTN = Case("student-t 4096x4096 b4 g64 axis1", 4096, 4096, 4, 64, 1, "student_t", 1)
MLP_B2 = Case("row-lognormal 4096x11008 b2 g16 axis1", 4096, 11008, 2, 16, 1, "row_lognormal", 2)
MLP_B3 = Case("row-lognormal 4096x11008 b3 g64 axis1", 4096, 11008, 3, 64, 1, "row_lognormal", 2)
ATTN_AX0 = Case("student-t 4096x4096 b4 g128 axis0", 4096, 4096, 4, 128, 0, "student_t", 3)
CASES = [SMALL, ATTN, MLP_B2, MLP_B3, ATTN_AX0]

# 7B-like stack: 32 layers x (4 x 4096x4096 attention + 3 x 4096x11008 MLP), b4 g64 axis1.
STACK_LAYERS = 32
STACK_SHAPES = [(4096, 4096)] * 4 + [(4096, 11008)] * 3


def stack_seed(layer: int, index: int) -> int:
    """Per-matrix seed of the 7B-like stack: layer seed 1000 + layer, then 16*that + index."""
    return (1000 + layer) * 16 + index


def stack_matrix(layer: int, index: int) -> np.ndarray:
    r, c = STACK_SHAPES[index]
    return student_t(r, c, stack_seed(layer, index))


def stack_matrix_torch(layer: int, index: int, device):
    """Same distribution as stack_matrix, drawn on a GPU with torch's Philox generator
    (host generation of 6.5 G samples takes minutes).  Not bit-identical to the numpy draw;
    tests that compare with the oracle copy these bytes back to the host."""
    import torch
    r, c = STACK_SHAPES[index]
    g = torch.Generator(device=device)
    g.manual_seed(stack_seed(layer, index))
    normal = torch.randn(r * c, generator=g, device=device, dtype=torch.float32)
    # chi-square(4) = 2 * Gamma(shape 2, scale 1); Gamma(2) = -log(U1*U2)
    u = torch.rand(2, r * c, generator=g, device=device, dtype=torch.float32)
    chi2 = -2.0 * torch.log(u[0].clamp_min(1e-30) * u[1].clamp_min(1e-30))
    t = normal / torch.sqrt(chi2 / 4.0)
    return (0.02 * t).clamp_(-1.0, 1.0).to(torch.float16).reshape(r, c)
