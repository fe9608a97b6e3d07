"""Seeded synthetic inputs for GPTQ-2D two-sided rounding.

This module only draws random numbers and assembles them into the shapes of
the workloads; it holds none of the rounding method's arithmetic.  Both the
fp64 oracle (through the tests) and the CUDA path (through the tests and the
benchmark) take their inputs from here, so the two sides always see the same
arrays.

Workloads (shapes follow the Llama-style layers the GPTQ-2D abstract quantizes
on arxivlens "GPTQ-2D: Cubic-Time Two-Sided Adaptive Rounding", Abstract):

* ``tiny``   W 64x64 fp64 ~ U(-8, 8), unit scales, no clamp; each Kronecker
             factor is X^T X / 256 + 0.01 I with X 256x64 ~ N(0, 1).
* ``small``  W 512x512 fp32 ~ N(0, 0.02^2) with 1% of columns scaled x10;
             INT4 per-row absmax scales; factors from 2048 Student-t(4)
             activation rows times a random per-channel scale U(0.1, 10),
             Gram / rows + 1% mean-diagonal damping.
* ``attn``   W 4096x4096 bf16 (used as fp32) ~ N(0, 0.02^2) with 0.5%
             heavy-tailed outlier columns; INT4; factors from 4096 rows each.
* ``mlp``    W 4096x14336, factors 4096^2 and 14336^2 from 8192 rows each.
* ``block70b`` the seven linear shapes of one 70B-class transformer block.

Activation model: Student-t with 4 degrees of freedom (heavy tails, finite
variance) times a per-channel scale drawn uniformly from [0.1, 10]; this is
the stand-in for calibration activations, which the pages do not provide.
"""
from __future__ import annotations

import dataclasses
import numpy as np

__all__ = [
    "Problem", "grid_limits", "absmax_scales", "student_t_activations",
    "damped_gram", "tiny", "small", "attn", "mlp", "block70b_shapes",
    "layer", "random_spd",
]


@dataclasses.dataclass
class Problem:
    """One rounding problem: W (m x n), H_L (m x m), H_R (n x n), scales (m)."""

    name: str
    W: np.ndarray            # m x n, fp32 or fp64 (the dtype handed to the library)
    H_L: np.ndarray          # m x m symmetric positive definite
    H_R: np.ndarray          # n x n symmetric positive definite
    scales: np.ndarray       # m, fp32, strictly positive
    bits: int                # grid width; clamp range [-2^(bits-1), 2^(bits-1)-1]
    clamp: bool

    @property
    def shape(self):
        return self.W.shape


def grid_limits(bits: int):
    """Signed integer grid of ``bits`` bits: [-2^(bits-1), 2^(bits-1) - 1]."""
    return -(1 << (bits - 1)), (1 << (bits - 1)) - 1


def absmax_scales(W: np.ndarray, bits: int) -> np.ndarray:
    """Per-row scale s_i = max_j |W_ij| / hi (hi = 7 for INT4); rows of zeros get 1."""
    _, hi = grid_limits(bits)
    s = np.max(np.abs(W.astype(np.float64)), axis=1) / hi
    s[s == 0] = 1.0
    return s.astype(np.float32)


def group_absmax_scales(W: np.ndarray, bits: int, group_size: int) -> np.ndarray:
    """Symmetric group-wise scales: s[i, g] = max |W[i, group g]| / hi, shape
    m x ceil(n / group_size); all-zero groups get 1."""
    m, n = W.shape
    _, hi = grid_limits(bits)
    ng = -(-n // group_size)
    A = np.zeros((m, ng))
    for g in range(ng):
        A[:, g] = np.max(np.abs(W[:, g * group_size:(g + 1) * group_size].astype(np.float64)), axis=1)
    s = A / hi
    s[s == 0] = 1.0
    return s.astype(np.float32)


def group_minmax_grid(W: np.ndarray, bits: int, group_size: int):
    """Asymmetric group-wise grid in the usual GPTQ convention: the range of each
    (row, group) is widened to include 0, s = (max - min) / (2^bits - 1) and the
    integer zero point z = round(-min / s) in [0, 2^bits - 1], so that code c
    stands for s (c - z).  group_size 0 means one group per row.  Returns
    (scales fp32, zeros uint8), each m x ceil(n / group_size)."""
    m, n = W.shape
    G = group_size or n
    ng = -(-n // G) if n else 0
    top = float((1 << bits) - 1)
    S = np.ones((m, ng), np.float32)
    Z = np.zeros((m, ng), np.uint8)
    for g in range(ng):
        blk = W[:, g * G:(g + 1) * G].astype(np.float64)
        lo = np.minimum(blk.min(axis=1), 0.0)
        hi = np.maximum(blk.max(axis=1), 0.0)
        sc = ((hi - lo) / top).astype(np.float32).astype(np.float64)
        sc[sc == 0] = 1.0
        S[:, g] = sc
        Z[:, g] = np.clip(np.rint(-lo / sc), 0, top).astype(np.uint8)
    return S, Z


def student_t_activations(rng: np.random.Generator, rows: int, width: int,
                          nu: float = 4.0) -> np.ndarray:
    """rows x width activations: Student-t(nu) entries times a per-column scale U(0.1, 10)."""
    X = rng.standard_t(nu, size=(rows, width))
    c = rng.uniform(0.1, 10.0, size=width)
    return X * c[None, :]


def damped_gram(X: np.ndarray, damp: float = 0.01, matmul=None) -> np.ndarray:
    """X^T X / rows + damp * mean(diag) * I, formed in fp64, returned as fp32.

    ``matmul`` lets a caller form the Gram on another device; it must return a
    float64 numpy array.  The default is numpy's fp64 product.
    """
    rows = X.shape[0]
    G = (X.T @ X) if matmul is None else matmul(X)
    G = G / rows
    G = 0.5 * (G + G.T)
    G[np.diag_indices_from(G)] += damp * float(np.mean(np.diag(G)))
    return G.astype(np.float32)


def random_spd(rng: np.random.Generator, k: int, rows: int | None = None,
               damp: float = 0.01, dtype=np.float64) -> np.ndarray:
    """Well-conditioned SPD test factor: X^T X / rows + damp I with X ~ N(0, 1)."""
    rows = rows if rows is not None else max(4 * k, 8)
    X = rng.standard_normal((rows, k))
    H = X.T @ X / rows + damp * np.eye(k)
    return (0.5 * (H + H.T)).astype(dtype)


def _bf16_round(a: np.ndarray) -> np.ndarray:
    """Round fp32 values to the nearest bf16 (ties to even) and return them as fp32."""
    u = np.ascontiguousarray(a, dtype=np.float32).view(np.uint32).astype(np.uint64)
    u = (u + 0x7FFF + ((u >> 16) & 1)) & 0xFFFF0000
    return u.astype(np.uint32).view(np.float32)


def _outlier_weight(rng: np.random.Generator, m: int, n: int, std: float,
                    frac: float, mode: str) -> np.ndarray:
    W = rng.normal(0.0, std, size=(m, n))
    k = int(np.floor(frac * n))
    if k > 0:
        cols = rng.choice(n, size=k, replace=False)
        if mode == "scale10":
            W[:, cols] *= 10.0
        else:  # heavy-tailed columns: 10x the base std, Student-t(4) shaped
            W[:, cols] = 10.0 * std * rng.standard_t(4.0, size=(m, k)) / np.sqrt(2.0)
    return W


def tiny(seed: int = 0) -> Problem:
    """64x64 fp64 case that the naive mn x mn Kronecker sweep finishes in seconds."""
    rng = np.random.default_rng(seed)
    m = n = 64
    W = rng.uniform(-8.0, 8.0, size=(m, n))
    XL = rng.standard_normal((256, m))
    XR = rng.standard_normal((256, n))
    H_L = XL.T @ XL / 256 + 0.01 * np.eye(m)
    H_R = XR.T @ XR / 256 + 0.01 * np.eye(n)
    H_L = 0.5 * (H_L + H_L.T)
    H_R = 0.5 * (H_R + H_R.T)
    return Problem("tiny64", W, H_L, H_R, np.ones(m, np.float32), 4, False)


def small(seed: int = 0, m: int = 512, n: int = 512, bits: int = 4) -> Problem:
    """512x512 fp32 layer with 1% outlier columns (x10), INT4 absmax scales."""
    rng = np.random.default_rng(seed)
    W = _outlier_weight(rng, m, n, 0.02, 0.01, "scale10").astype(np.float32)
    H_L = damped_gram(student_t_activations(rng, 2048, m))
    H_R = damped_gram(student_t_activations(rng, 2048, n))
    return Problem(f"small{m}x{n}_s{seed}", W, H_L, H_R, absmax_scales(W, bits), bits, True)


def layer(m: int, n: int, *, seed: int = 0, bits: int = 4, std: float = 0.02,
          outlier_frac: float = 0.005, rows_l: int | None = None,
          rows_r: int | None = None, matmul=None, name: str | None = None) -> Problem:
    """An LLM-shaped layer: bf16-valued W (held as fp32), heavy-tailed Grams, absmax scales."""
    rng = np.random.default_rng(seed)
    W = _bf16_round(_outlier_weight(rng, m, n, std, outlier_frac, "heavy").astype(np.float32))
    H_L = damped_gram(student_t_activations(rng, rows_l or m, m), matmul=matmul)
    H_R = damped_gram(student_t_activations(rng, rows_r or n, n), matmul=matmul)
    return Problem(name or f"layer{m}x{n}_int{bits}_s{seed}", W, H_L, H_R,
                   absmax_scales(W, bits), bits, True)


def attn(seed: int = 0, matmul=None) -> Problem:
    """4096x4096 attention projection, INT4, factors from 4096 activation rows per side."""
    return layer(4096, 4096, seed=seed, bits=4, rows_l=4096, rows_r=4096,
                 matmul=matmul, name=f"attn4096x4096_int4_s{seed}")


def mlp(seed: int = 0, bits: int = 4, matmul=None) -> Problem:
    """4096x14336 MLP projection, factors from 8192 activation rows per side."""
    return layer(4096, 14336, seed=seed, bits=bits, rows_l=8192, rows_r=8192,
                 matmul=matmul, name=f"mlp4096x14336_int{bits}_s{seed}")


def block70b_shapes():
    """(name, m, n, count) of the linear layers of one 70B-class block (q/o, k/v, gate/up, down)."""
    return [("q", 8192, 8192, 1), ("o", 8192, 8192, 1), ("k", 1024, 8192, 1),
            ("v", 1024, 8192, 1), ("gate", 8192, 28672, 1), ("up", 8192, 28672, 1),
            ("down", 28672, 8192, 1)]
