"""Seeded synthetic AQLM layers (host numpy arrays).

This module only draws random inputs; it holds none of the layer's arithmetic.
Tests, the benchmark and the smoke check use it to feed the same bytes to the
CUDA library and to the CPU oracle.

Recipe (one generator per tensor, so tensors never share a stream):
    rng = numpy Generator(PCG64(SeedSequence([seed, workload, layer, tensor, copy])))
    tensor 0  codes      uniform integers in [0, 2^B)       uint8 (B<=8) / uint16
    tensor 1  codebooks  normal(0, 0.05) -> fp16 (RNE)       [M, 2^B, g]
    tensor 2  scales     uniform(0.5, 1.5) -> fp16           [N]
    tensor 3  x          normal(0, 1) -> fp16                [batch, K]
    tensor 4  bias       normal(0, 1) -> fp16                [N] (only when asked)
    tensor 5  outliers   make_x_outliers: the outlier channels and their values
Uniform codes are the worst case for codebook locality; the pages give no code
statistics of trained checkpoints.
"""
from __future__ import annotations

from dataclasses import dataclass
from typing import Optional

import numpy as np

CODES, CODEBOOKS, SCALES, X, BIAS, OUTLIERS = range(6)


def rng(seed: int, workload: int, layer: int, tensor: int, copy: int = 0) -> np.random.Generator:
    return np.random.Generator(np.random.PCG64(np.random.SeedSequence([seed, workload, layer, tensor, copy])))


@dataclass
class LayerData:
    M: int
    B: int
    g: int
    K: int
    N: int
    codes: np.ndarray               # [N, K/g, M] uint8 / uint16
    codebooks: np.ndarray           # [M, 2^B, g] float16
    scales: np.ndarray              # [N] float16
    bias: Optional[np.ndarray]      # [N] float16 or None


def codes_dtype(B: int):
    return np.uint8 if B <= 8 else np.uint16


def make_layer(M: int, B: int, g: int, K: int, N: int, *, seed: int = 0, workload: int = 0,
               layer: int = 0, copy: int = 0, with_bias: bool = False,
               codebook_std: float = 0.05) -> LayerData:
    if K % g:
        raise ValueError("K must be a multiple of g")
    G = K // g
    dt = codes_dtype(B)
    codes = rng(seed, workload, layer, CODES, copy).integers(0, 1 << B, size=(N, G, M), dtype=dt)
    cb = rng(seed, workload, layer, CODEBOOKS, copy).normal(0.0, codebook_std, size=(M, 1 << B, g))
    sc = rng(seed, workload, layer, SCALES, copy).uniform(0.5, 1.5, size=N)
    bias = None
    if with_bias:
        bias = rng(seed, workload, layer, BIAS, copy).normal(0.0, 1.0, size=N).astype(np.float16)
    return LayerData(M, B, g, K, N, codes, cb.astype(np.float32).astype(np.float16),
                     sc.astype(np.float32).astype(np.float16), bias)


def make_x(batch: int, K: int, *, seed: int = 0, workload: int = 0, layer: int = 0,
           copy: int = 0) -> np.ndarray:
    return rng(seed, workload, layer, X, copy).normal(0.0, 1.0, size=(batch, K)).astype(
        np.float32).astype(np.float16)


def make_x_outliers(batch: int, K: int, *, sigma: float, n_outliers: int, lo: float = 500.0,
                    hi: float = 2000.0, seed: int = 0, workload: int = 0, layer: int = 0,
                    copy: int = 0) -> np.ndarray:
    """Activations with the spread of a real fp16 layer input: x ~ normal(0, sigma), and
    n_outliers channels (the same K indices in every batch row, drawn without replacement)
    whose values are uniform in [lo, hi] in magnitude with a random sign per element,
    all rounded to fp16."""
    x = rng(seed, workload, layer, X, copy).normal(0.0, sigma, size=(batch, K))
    if n_outliers:
        r = rng(seed, workload, layer, OUTLIERS, copy)
        cols = r.choice(K, size=n_outliers, replace=False)
        mag = r.uniform(lo, hi, size=(batch, n_outliers))
        sign = np.where(r.integers(0, 2, size=(batch, n_outliers)) == 1, 1.0, -1.0)
        x[:, cols] = sign * mag
    return x.astype(np.float32).astype(np.float16)
