"""Seeded synthetic inputs shared by the tests, the benchmark and the oracle checks.

This module draws random numbers and nothing else: it holds none of the
numerical method (no splitting, quantisation, normalisation or products).
Every generator takes an explicit integer seed and returns host numpy arrays,
so the CUDA path and the CPU oracle are always fed byte-identical inputs.

Distributions follow the workloads the method is evaluated on:
  * activations  ~ N(0, 1) fp32, optionally with a Bernoulli(p) fraction of
    outliers multiplied by a factor (0.1 % x 100 for the GEMM sweep);
  * weights      ~ N(0, 0.02) fp32;
  * RMSNorm gain ~ U(0.5, 1.5);
  * K/V tensors  ~ N(0, 1) x c[h, d] with a per-channel factor
    c ~ LogUniform(0.1, 10);
  * ragged KV lengths ~ U{lo..hi}; token ids ~ U{0..vocab-1}.
"""
from __future__ import annotations

import numpy as np

__all__ = [
    "rng",
    "normal",
    "uniform",
    "normal_with_outliers",
    "kv_tensor",
    "channel_scale",
    "ragged_lengths",
    "token_ids",
    "permutation",
]


def rng(seed: int, stream: int = 0) -> np.random.Generator:
    """A PCG64 generator keyed by (seed, stream) so independent tensors of one
    case never share a stream."""
    return np.random.Generator(np.random.PCG64([int(seed) & 0xFFFFFFFF, int(stream) & 0xFFFFFFFF]))


def normal(shape, seed: int, stream: int = 0, std: float = 1.0) -> np.ndarray:
    g = rng(seed, stream)
    return (g.standard_normal(size=shape) * std).astype(np.float32)


def uniform(shape, seed: int, stream: int = 0, lo: float = 0.0, hi: float = 1.0) -> np.ndarray:
    g = rng(seed, stream)
    return g.uniform(lo, hi, size=shape).astype(np.float32)


def normal_with_outliers(shape, seed: int, stream: int = 0, frac: float = 1e-3,
                         factor: float = 100.0) -> np.ndarray:
    """N(0,1) fp32 where each element independently (probability `frac`) is
    multiplied by `factor`."""
    g = rng(seed, stream)
    x = g.standard_normal(size=shape)
    hit = g.random(size=shape) < frac
    x = np.where(hit, x * factor, x)
    return x.astype(np.float32)


def channel_scale(n_heads: int, head_dim: int, seed: int, stream: int = 0,
                  lo: float = 0.1, hi: float = 10.0) -> np.ndarray:
    """Per-(head, channel) factor c ~ LogUniform(lo, hi), fp32 [n_heads, head_dim]."""
    g = rng(seed, stream)
    u = g.uniform(np.log(lo), np.log(hi), size=(n_heads, head_dim))
    return np.exp(u).astype(np.float32)


def kv_tensor(n_tokens: int, n_heads: int, head_dim: int, seed: int, stream: int = 0,
              scale: np.ndarray | None = None) -> np.ndarray:
    """fp32 [n_tokens, n_heads, head_dim] ~ N(0,1) times a per-channel factor."""
    x = normal((n_tokens, n_heads, head_dim), seed, stream).astype(np.float64)
    if scale is not None:
        x = x * scale.astype(np.float64)[None, :, :]
    return x.astype(np.float32)


def ragged_lengths(n: int, seed: int, stream: int = 0, lo: int = 128, hi: int = 8192) -> np.ndarray:
    g = rng(seed, stream)
    return g.integers(lo, hi + 1, size=n).astype(np.int32)


def token_ids(n: int, vocab: int, seed: int, stream: int = 0) -> np.ndarray:
    g = rng(seed, stream)
    return g.integers(0, vocab, size=n).astype(np.int32)


def permutation(n: int, seed: int, stream: int = 0) -> np.ndarray:
    g = rng(seed, stream)
    return g.permutation(n).astype(np.int64)
