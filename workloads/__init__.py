"""Seeded synthetic workloads for the BaKron solve (inputs only).

This module holds no arithmetic of the method: it only draws W and the two
Kronecker factors A (n x n, input side) and B (m x m, output side) of the
Hessian, the way the pages' experiments would obtain them from calibration
data (Gram matrices of activation / gradient samples plus damping).  Both the
CUDA path and the oracle consume the arrays it returns.

The shapes follow the pages' benchmarks ("What carries the argument" /
"If this is right": 4096 x 4096; referee report on Table 3: 14336 x 4096) and
typical transformer projections; the value distributions are synthetic
stand-ins for the calibration data the pages use (no dataset or checkpoint is
available).  Recipes:

  tiny     W 64x128  N(0,0.02^2); A = X^T X/512, X 512x128 N(0,1) diag(u),
           u ~ U[0.5,2]; B likewise from G 512x64; damping 1% of mean diag; INT4
  tiny_bI  as tiny with B = I (two-sided solve must reduce to GPTQ)
  mid      W 1024x1024 N(0,0.02^2); A from X 4096x1024 N(0,1) with 1% of the
           channels scaled x20; B from G 4096x1024 Student-t(4); 1%; INT4
  bench    W 4096x4096 N(0,0.02^2); A, B from X = Z diag(sigma) Q^T, Z 8192x4096
           N(0,1), sigma_k^2 = 10^(-4k/(n-1)), Q Haar-orthogonal; 1%; INT4
  mlp_up   W 11008x4096 N(0,0.015^2); A from 8192 Student-t(4) activation
           samples; B from 8192 Gaussian gradient samples; 1%; INT3
  mlp_down the transposed shape 4096x11008, same recipe
  large2   W 14336x4096 N(0,0.01^2); A, B from 16384 Gaussian samples with
           0.5% outlier channels x30; damping 0.5%; INT2
  large4   as large2 with INT4

Random streams: numpy ``Generator(PCG64)`` seeded by
``SeedSequence(seed, spawn_key=(stream,))`` with independent streams for W (0),
A (1) and B (2).
"""
from __future__ import annotations

import dataclasses
import hashlib
import os

import numpy as np


@dataclasses.dataclass(frozen=True)
class Workload:
    name: str
    m: int
    n: int
    bits: int
    w_std: float
    a_recipe: str
    b_recipe: str
    a_samples: int
    b_samples: int
    damping: float
    outlier_frac: float = 0.0
    outlier_scale: float = 1.0
    seed: int = 0

    @property
    def qmax(self) -> int:
        return (1 << (self.bits - 1)) - 1

    @property
    def qmin(self) -> int:
        return -self.qmax


WORKLOADS = {
    w.name: w
    for w in [
        Workload("tiny", 64, 128, 4, 0.02, "scaled_gauss", "scaled_gauss", 512, 512, 0.01),
        Workload("tiny_bI", 64, 128, 4, 0.02, "scaled_gauss", "identity", 512, 0, 0.01),
        Workload("mid", 1024, 1024, 4, 0.02, "outlier_gauss", "student_t", 4096, 4096, 0.01,
                 outlier_frac=0.01, outlier_scale=20.0),
        Workload("bench", 4096, 4096, 4, 0.02, "decaying_spectrum", "decaying_spectrum", 8192, 8192, 0.01),
        Workload("mlp_up", 11008, 4096, 3, 0.015, "student_t", "gauss", 8192, 8192, 0.01),
        Workload("mlp_down", 4096, 11008, 3, 0.015, "student_t", "gauss", 8192, 8192, 0.01),
        Workload("large2", 14336, 4096, 2, 0.01, "outlier_gauss", "outlier_gauss", 16384, 16384, 0.005,
                 outlier_frac=0.005, outlier_scale=30.0),
        Workload("large4", 14336, 4096, 4, 0.01, "outlier_gauss", "outlier_gauss", 16384, 16384, 0.005,
                 outlier_frac=0.005, outlier_scale=30.0),
    ]
}


def rng(seed: int, stream: int) -> np.random.Generator:
    return np.random.Generator(np.random.PCG64(np.random.SeedSequence(seed, spawn_key=(stream,))))


def _samples(recipe: str, N: int, d: int, g: np.random.Generator, w: Workload) -> np.ndarray:
    """N x d float32 sample matrix for one side of the Hessian."""
    if recipe == "scaled_gauss":
        X = g.standard_normal((N, d), dtype=np.float32)
        X *= g.uniform(0.5, 2.0, size=d).astype(np.float32)[None, :]
    elif recipe == "gauss":
        X = g.standard_normal((N, d), dtype=np.float32)
    elif recipe == "outlier_gauss":
        X = g.standard_normal((N, d), dtype=np.float32)
        k = max(1, int(round(w.outlier_frac * d)))
        idx = g.choice(d, size=k, replace=False)
        X[:, idx] *= np.float32(w.outlier_scale)
    elif recipe == "student_t":
        # Student-t(4): z / sqrt(chi2_4 / 4)
        z = g.standard_normal((N, d), dtype=np.float32)
        chi = g.chisquare(4.0, size=(N, d)).astype(np.float32)
        X = z / np.sqrt(chi / np.float32(4.0))
    elif recipe == "decaying_spectrum":
        # X = Z diag(sigma) Q^T with sigma_k^2 = 10^(-4k/(d-1)), Q Haar-orthogonal
        Z = g.standard_normal((N, d), dtype=np.float32)
        G = g.standard_normal((d, d))
        Q, Rq = np.linalg.qr(G)
        Q = Q * np.sign(np.diag(Rq))[None, :]
        sigma = np.sqrt(10.0 ** (-4.0 * np.arange(d) / max(d - 1, 1)))
        X = Z @ (sigma[:, None] * Q.T).astype(np.float32)
    else:
        raise ValueError(recipe)
    return X


def _gram(recipe: str, N: int, d: int, g: np.random.Generator, w: Workload) -> np.ndarray:
    if recipe == "identity":
        return np.eye(d, dtype=np.float32)
    X = _samples(recipe, N, d, g, w)
    G = (X.T @ X).astype(np.float64) / N
    G = 0.5 * (G + G.T)
    G[np.diag_indices(d)] += w.damping * float(np.mean(np.diag(G)))
    return G.astype(np.float32)


def _cache_dir():
    d = os.environ.get("BAKRON_WORKLOAD_CACHE")
    return d if d else None


def generate(name_or_workload, seed: int | None = None):
    """Return ``(W, A, B)`` as contiguous float32 arrays for a named workload.

    If ``BAKRON_WORKLOAD_CACHE`` names a directory, arrays are cached there as
    ``.npy`` files keyed by workload and seed.
    """
    w = WORKLOADS[name_or_workload] if isinstance(name_or_workload, str) else name_or_workload
    if seed is not None:
        w = dataclasses.replace(w, seed=seed)
    cache = _cache_dir()
    key = hashlib.sha256(repr(w).encode()).hexdigest()[:16]
    if cache:
        p = os.path.join(cache, f"{w.name}_{key}.npz")
        if os.path.exists(p):
            z = np.load(p)
            return z["W"], z["A"], z["B"]
    W = (rng(w.seed, 0).standard_normal((w.m, w.n), dtype=np.float32) * np.float32(w.w_std)).astype(np.float32)
    A = _gram(w.a_recipe, w.a_samples, w.n, rng(w.seed, 1), w)
    B = _gram(w.b_recipe, w.b_samples, w.m, rng(w.seed, 2), w)
    W, A, B = (np.ascontiguousarray(x) for x in (W, A, B))
    if cache:
        os.makedirs(cache, exist_ok=True)
        tmp = os.path.join(cache, f".{w.name}_{key}.{os.getpid()}.npz")
        np.savez(tmp, W=W, A=A, B=B)
        os.replace(tmp, p)
    return W, A, B


def random_problem(m: int, n: int, seed: int, bits: int = 4, w_std: float = 0.02,
                   samples_factor: int = 4, damping: float = 0.01, cond_spread: float = 2.0):
    """Small random problem (W, A, B) for property tests: Gram factors of
    Gaussian samples with column scales in [1/cond_spread, cond_spread]."""
    g = rng(seed, 7)
    W = (g.standard_normal((m, n)) * w_std).astype(np.float32)

    def gram(d):
        N = max(samples_factor * d, 4)
        X = g.standard_normal((N, d)) * g.uniform(1.0 / cond_spread, cond_spread, size=d)[None, :]
        G = X.T @ X / N
        G = 0.5 * (G + G.T)
        G[np.diag_indices(d)] += damping * float(np.mean(np.diag(G)))
        return G.astype(np.float32)

    return W, gram(n), gram(m)
