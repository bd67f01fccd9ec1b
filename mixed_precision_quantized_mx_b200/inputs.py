"""Seeded synthetic inputs shared by the tests, the benchmark and the oracle checks.

This module draws random numbers only: it holds none of the quantization or
GEMM arithmetic, so that the CUDA path and the CPU oracle can both be fed from it
without sharing any of the method's code.  Everything is numpy on the host.

Workloads (shapes from the MixLLM paper's Llama 3.1 models and its single-linear
benchmark, section 4.3; value distributions are synthetic stand-ins for trained
weights and real activations, which are not available here):

* tiny layer: X fp32 [16, 512] ~ N(0, 1) with 4 outlier channels x20,
  W fp32 [512, 512] ~ N(0, 0.02), saliency score ~ |N(0, 1)| per output row,
  top 10% rows (51) at 8 bits, group 128.
* Llama-shaped layers: W ~ N(0, 0.02) with 0.1% of entries x10,
  X ~ N(0, 1) with 1% of channels x20 stored as fp16, 10% 8-bit rows.
"""
from __future__ import annotations

from dataclasses import dataclass

import numpy as np


def n8_for(N: int, frac: float) -> int:
    """Number of 8-bit rows for a fraction p of N: floor(p N + 1/2)."""
    return int(np.floor(frac * N + 0.5))


def saliency_mask(scores: np.ndarray, n8: int) -> np.ndarray:
    """uint8 mask of the n8 rows with the largest score; ties go to the lower row index."""
    N = scores.shape[0]
    order = np.lexsort((np.arange(N), -scores))  # primary: score descending, then index
    mask = np.zeros(N, np.uint8)
    mask[order[:n8]] = 1
    return mask


@dataclass
class Layer:
    X: np.ndarray      # [M, K] fp32 or fp16 (host)
    W: np.ndarray      # [N, K] fp32 (host)
    is8: np.ndarray    # [N] uint8
    group: int
    name: str

    @property
    def M(self) -> int:
        return self.X.shape[0]

    @property
    def K(self) -> int:
        return self.X.shape[1]

    @property
    def N(self) -> int:
        return self.W.shape[0]

    @property
    def n8(self) -> int:
        return int(self.is8.sum())


def activations(rng: np.random.Generator, M: int, K: int, n_outlier: int,
                outlier_scale: float = 20.0, dtype=np.float16) -> np.ndarray:
    """X ~ N(0, 1) with n_outlier seed-chosen channels (columns) scaled up."""
    X = rng.standard_normal((M, K), dtype=np.float32)
    if n_outlier:
        cols = rng.choice(K, size=n_outlier, replace=False)
        X[:, cols] *= outlier_scale
    return X.astype(dtype)


def weights(rng: np.random.Generator, N: int, K: int, std: float = 0.02,
            outlier_frac: float = 0.0, outlier_scale: float = 10.0) -> np.ndarray:
    """W ~ N(0, std) with a fraction of entries (uniform positions) scaled up."""
    W = rng.standard_normal((N, K), dtype=np.float32)
    W *= np.float32(std)
    n_out = int(round(outlier_frac * N * K))
    if n_out:
        idx = rng.integers(0, N * K, size=n_out, dtype=np.int64)
        W.reshape(-1)[idx] *= np.float32(outlier_scale)
    return W


def gradients(rng: np.random.Generator, N: int, K: int, std: float = 1e-3, row_sigma: float = 1.0,
              dtype=np.float32) -> np.ndarray:
    """Stand-in for the loss gradient of a weight matrix on a calibration batch:
    G ~ N(0, std) times a log-normal scale per output row (sigma row_sigma), so that
    a few rows carry most of the gradient."""
    G = rng.standard_normal((N, K), dtype=np.float32)
    G *= (np.float32(std) * np.exp(rng.standard_normal(N) * row_sigma).astype(np.float32))[:, None]
    return G.astype(dtype)


def block_codes(rng: np.random.Generator, N: int, K: int, probs=(0.25, 0.25, 0.25, 0.25),
                block_rows: int = 64, block_cols: int = 128) -> np.ndarray:
    """2-bit code (0..3) of every block of block_rows output rows x block_cols input
    columns, drawn with the given probabilities: [ceil(N / block_rows), K / block_cols]."""
    shape = ((N + block_rows - 1) // block_rows, K // block_cols)
    return rng.choice(4, size=shape, p=np.asarray(probs, np.float64)).astype(np.uint8)


def tiny_layer(seed: int = 0) -> Layer:
    """Tiny linear layer: M=16, K=N=512, g=128, 51 of 512 rows at 8 bits, fp32 X."""
    rng = np.random.default_rng(seed)
    X = activations(rng, 16, 512, 4, dtype=np.float32)
    W = weights(rng, 512, 512)
    scores = np.abs(rng.standard_normal(512))
    return Layer(X, W, saliency_mask(scores, n8_for(512, 0.10)), 128, "tiny")


def llama_layer(M: int, K: int, N: int, frac8: float = 0.10, group: int = 128,
                seed: int = 0, x_dtype=np.float16, name: str = "") -> Layer:
    """Llama-shaped layer with the value distributions described above."""
    rng = np.random.default_rng(seed)
    X = activations(rng, M, K, int(round(0.01 * K)), dtype=x_dtype)
    W = weights(rng, N, K, outlier_frac=0.001)
    scores = np.abs(rng.standard_normal(N))
    return Layer(X, W, saliency_mask(scores, n8_for(N, frac8)), group,
                 name or f"M{M}_K{K}_N{N}_p{frac8:g}_g{group}")


# Llama 3 shapes named by the workloads they come from (K -> N).
SHAPES = {
    "llama3-8b-qo": (4096, 4096),
    "llama3-8b-up": (4096, 14336),
    "llama3-8b-down": (14336, 4096),
    "llama3-70b-up": (8192, 28672),
    "llama3-70b-down": (28672, 8192),
    "sweep-8192": (8192, 8192),
}
