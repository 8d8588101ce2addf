"""Seeded synthetic layers shaped like the LLaMA/OPT workloads of the AWQ pages.

This module only draws random numbers; it holds none of the method's
arithmetic.  Both the CUDA path and the CPU oracle take their inputs from here.

Recipe (one generator per layer, ``numpy.random.Generator(PCG64(seed))``):
  1. W[N, K] ~ Normal(0, w_std^2), drawn as float32 in row-major order,
     rounded to fp16 (round to nearest even);
  2. the outlier input channels: ``choice(K, n_outliers, replace=False)``;
  3. their factors: a fixed factor, or 10 ** Uniform[log10(lo), log10(hi));
  4. X[T, K] ~ Normal(0, 1) drawn as float32, outlier columns multiplied by
     their factors, rounded to fp16.

About 1% of the input channels carry activations 10-100x larger than the rest,
which is the structure the pages describe ("Quan sát chung" of the page
"52 · AWQ, GPTQ và SmoothQuant": most channels small, a few 10-100x larger).
"""
from __future__ import annotations

from dataclasses import dataclass, asdict

import numpy as np


@dataclass(frozen=True)
class LayerConfig:
    name: str
    N: int
    K: int
    T: int
    w_std: float
    n_outliers: int
    outlier_lo: float
    outlier_hi: float       # equal to outlier_lo for a fixed factor
    bits: int
    group: int
    seed: int

    @property
    def flops_per_alpha(self) -> int:
        return 2 * self.N * self.K * self.T

    def as_dict(self):
        return asdict(self)


# The five workload families; sizes and distributions as the benchmark states them.
CONFIGS = {
    "layer512": LayerConfig("single layer 512x512, T=512, INT4 g128", 512, 512, 512,
                            0.02, 5, 20.0, 20.0, 4, 128, 0),
    "attn4096": LayerConfig("LLaMA-7B attention projection 4096x4096, T=4096, INT4 g128",
                            4096, 4096, 4096, 0.02, 41, 10.0, 100.0, 4, 128, 1),
    "mlp_gate11008": LayerConfig("LLaMA-7B MLP gate/up 11008x4096, T=4096, INT4 g128",
                                 11008, 4096, 4096, 0.02, 41, 10.0, 100.0, 4, 128, 2),
    "mlp_gateup22016": LayerConfig("LLaMA-7B MLP gate+up stacked 22016x4096 (one shared X), T=4096, INT4 g128",
                                   22016, 4096, 4096, 0.02, 41, 10.0, 100.0, 4, 128, 2),
    "mlp_down4096": LayerConfig("LLaMA-7B MLP down 4096x11008, T=4096, INT4 g128",
                                4096, 11008, 4096, 0.02, 110, 10.0, 100.0, 4, 128, 2),
    "attn4096_int3": LayerConfig("4096x4096, T=4096, INT3 g128", 4096, 4096, 4096,
                                 0.02, 41, 10.0, 100.0, 3, 128, 3),
    "attn4096_int2": LayerConfig("4096x4096, T=4096, INT2 g64", 4096, 4096, 4096,
                                 0.02, 41, 10.0, 100.0, 2, 64, 3),
    "mlp_up28672": LayerConfig("LLaMA-70B MLP up 28672x8192, T=4096, INT4 g128",
                               28672, 8192, 4096, 0.015, 82, 10.0, 100.0, 4, 128, 4),
}


def make_config(N, K, T, bits=4, group=128, seed=0, w_std=0.02, outlier_frac=0.01,
                lo=10.0, hi=100.0, name=None) -> LayerConfig:
    """An ad-hoc layer with the same distributions (used for edge-case tests)."""
    n_out = max(1, int(round(K * outlier_frac))) if outlier_frac > 0 else 0
    return LayerConfig(name or f"{N}x{K} T={T} b{bits} g{group}", N, K, T, w_std, n_out,
                       lo, hi, bits, group, seed)


def generate(cfg: LayerConfig):
    """Returns (W fp16 [N,K], X fp16 [T,K], outlier channel indices)."""
    rng = np.random.Generator(np.random.PCG64(cfg.seed))
    W = rng.standard_normal((cfg.N, cfg.K), dtype=np.float32)
    W *= np.float32(cfg.w_std)
    W16 = W.astype(np.float16)
    del W
    if cfg.n_outliers > 0:
        idx = np.sort(rng.choice(cfg.K, cfg.n_outliers, replace=False))
        if cfg.outlier_hi == cfg.outlier_lo:
            fac = np.full(cfg.n_outliers, cfg.outlier_lo, dtype=np.float64)
        else:
            u = rng.random(cfg.n_outliers)
            l0, l1 = np.log10(cfg.outlier_lo), np.log10(cfg.outlier_hi)
            fac = 10.0 ** (l0 + (l1 - l0) * u)
    else:
        idx = np.zeros(0, dtype=np.int64)
        fac = np.zeros(0)
    X = rng.standard_normal((cfg.T, cfg.K), dtype=np.float32)
    if idx.size:
        X[:, idx] *= fac.astype(np.float32)
    X16 = X.astype(np.float16)
    return W16, X16, idx


def default_alphas(n: int = 20) -> np.ndarray:
    """The grid alpha_i = RN32(i / n), i = 0..n-1 ({0, 0.05, ..., 0.95} for n = 20)."""
    return np.array([np.float32(i / n) for i in range(n)], dtype=np.float32)
