"""Seeded synthetic inputs for the blocked-Shampoo step.

This module only draws random numbers and arranges them into the shapes of
the five workloads; it holds none of the optimizer's arithmetic, so both the
CUDA path and the float64 checker can take their inputs from here.

Every generator returns float32 arrays (the bytes the GPU reads).  Checkers
upcast the same float32 values to float64, so both sides see identical input.

Workload recipes (shapes after "DASH: Faster Shampoo via Batched Block
Preconditioning and Efficient Inverse-Root Solvers", §4 Blocking Strategy and
§5 Experimental Results, where a transformer is blocked at B = 1024):

* tiny_dense   -- one 256x256 weight, N(0,1) gradients for 10 steps.
* lowrank_stack -- 256 blocks of 128x128, G = U diag(1/i) V^T with U, V
                   Haar-random orthogonal (fresh per block and step).
* transformer  -- 8 layers of d=1024, FFN 4096: four d x d attention weights,
                  one d x 4F and one 4F x d MLP weight; N(0, 0.02^2) entries,
                  1% of them multiplied by 50.
* spd_stack    -- 512 SPD matrices Q diag(lam) Q^T, lam log-uniform in
                  [1e-6, 1].
* large_blocks -- 32 blocks of 2048x2048, N(0,1) entries scaled per row by
                  exp(N(0,1)).
"""
from __future__ import annotations

import numpy as np

__all__ = [
    "haar_orthogonal",
    "tiny_dense_grads",
    "lowrank_stack_grads",
    "transformer_shapes",
    "transformer_grads",
    "spd_stack",
    "large_block_grads",
    "power_iteration_starts",
    "gaussian_stack",
]


def haar_orthogonal(rng: np.random.Generator, n: int, count: int = 1) -> np.ndarray:
    """`count` Haar-distributed n x n orthogonal matrices (float64).

    QR of a Gaussian matrix with the signs of R's diagonal folded into Q
    (Mezzadri, "How to generate random matrices from the classical compact
    groups", 2007), which makes the distribution exactly Haar.
    """
    z = rng.standard_normal((count, n, n))
    q, r = np.linalg.qr(z)
    d = np.sign(np.diagonal(r, axis1=1, axis2=2))
    d[d == 0] = 1.0
    return q * d[:, None, :]


def tiny_dense_grads(steps: int = 10, rows: int = 256, cols: int = 256, seed: int = 0) -> np.ndarray:
    """(steps, rows, cols) float32 gradients with i.i.d. N(0,1) entries."""
    rng = np.random.default_rng(seed)
    return rng.standard_normal((steps, rows, cols)).astype(np.float32)


def lowrank_stack_grads(steps: int = 5, blocks: int = 256, n: int = 128, seed: int = 0) -> np.ndarray:
    """(steps, blocks, n, n) float32 gradients U diag(sigma) V^T, sigma_i = 1/i.

    U and V are fresh Haar-random orthogonal matrices for every block and step.
    """
    rng = np.random.default_rng(seed)
    sigma = 1.0 / np.arange(1, n + 1, dtype=np.float64)
    out = np.empty((steps, blocks, n, n), dtype=np.float32)
    for t in range(steps):
        u = haar_orthogonal(rng, n, blocks)
        v = haar_orthogonal(rng, n, blocks)
        out[t] = np.einsum("bik,k,bjk->bij", u, sigma, v).astype(np.float32)
    return out


def transformer_shapes(n_layers: int = 8, d: int = 1024, ffn: int = 4096) -> list[tuple[int, int]]:
    """Weight shapes of a transformer stack: per layer 4 x (d,d), (d,ffn), (ffn,d)."""
    shapes: list[tuple[int, int]] = []
    for _ in range(n_layers):
        shapes += [(d, d)] * 4 + [(d, ffn), (ffn, d)]
    return shapes


def transformer_grads(shapes: list[tuple[int, int]], std: float = 0.02, outlier_frac: float = 0.01,
                      outlier_scale: float = 50.0, seed: int = 0) -> list[np.ndarray]:
    """One float32 gradient per weight: N(0, std^2), a Bernoulli(outlier_frac) mask scaled by outlier_scale."""
    rng = np.random.default_rng(seed)
    grads = []
    for (m, n) in shapes:
        g = rng.standard_normal((m, n), dtype=np.float32) * np.float32(std)
        mask = rng.random((m, n), dtype=np.float32) < outlier_frac
        g[mask] *= np.float32(outlier_scale)
        grads.append(g)
    return grads


def spd_stack(count: int = 512, n: int = 256, log10_lo: float = -6.0, log10_hi: float = 0.0,
              seed: int = 0) -> tuple[np.ndarray, np.ndarray, np.ndarray]:
    """SPD stack Q diag(lam) Q^T with lam = 10^U(lo, hi) and Haar Q.

    Returns (A32, Q, lam): the float32 matrices the GPU reads, and the float64
    factors they were built from.
    """
    rng = np.random.default_rng(seed)
    q = haar_orthogonal(rng, n, count)
    lam = 10.0 ** rng.uniform(log10_lo, log10_hi, size=(count, n))
    a = np.einsum("bik,bk,bjk->bij", q, lam, q)
    a = 0.5 * (a + np.swapaxes(a, 1, 2))
    return a.astype(np.float32), q, lam


def large_block_grads(steps: int = 3, blocks: int = 32, n: int = 2048, seed: int = 0) -> np.ndarray:
    """(steps, blocks, n, n) float32: N(0,1) entries times exp(N(0,1)) per row."""
    rng = np.random.default_rng(seed)
    out = np.empty((steps, blocks, n, n), dtype=np.float32)
    for t in range(steps):
        for b in range(blocks):
            row = np.exp(rng.standard_normal((n, 1))).astype(np.float32)
            out[t, b] = rng.standard_normal((n, n), dtype=np.float32) * row
    return out


def power_iteration_starts(n: int, vectors: int = 16, seed: int = 0) -> np.ndarray:
    """(vectors, n) float32 N(0,1) start vectors for multi-power-iteration."""
    rng = np.random.default_rng(seed + 7919)
    return rng.standard_normal((vectors, n)).astype(np.float32)


def gaussian_stack(count: int, rows: int, cols: int, seed: int = 0, scale: float = 1.0) -> np.ndarray:
    """(count, rows, cols) float32 N(0, scale^2) — generic test input."""
    rng = np.random.default_rng(seed)
    return (rng.standard_normal((count, rows, cols)) * scale).astype(np.float32)
