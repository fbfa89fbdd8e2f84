"""Plain FP64 oracle for the BaKron two-sided adaptive-rounding solve.

TEST INFRASTRUCTURE ONLY.  Only ``tests/``, ``__graft_entry__.smoke()`` and the
CPU-baseline leg of ``bench.py`` may import this package.  It shares no code with
the CUDA library (``two_sided_gptq_b200``) and never imports it.

What it follows (pages: "BaKron: Efficient Quantization with Kronecker-Factored
Hessians", pith.science review of arXiv 2608.06291, and the arXiv abstract):

* proxy loss ``||vec(W)-vec(V)||_H^2`` with ``H = A (x) B`` (Appendix A.1 as quoted
  in the reference list; Corollary 3.4 writes it ``||B^{1/2}(V-W)A^{1/2}||_F^2``);
* factors: lower Cholesky factors of ``A^{-1}`` and ``B^{-1}`` ("What carries the
  argument"; the assumption list says Cholesky distributes over Kronecker
  products);
* Proposition 3.1 and Theorem 3.2: the intended output computed by
  BaKron-naive (Algorithm 2), BaKron-antidiagonal, BaKron-recursive and BaKron
  (Algorithm 6) -- see ``bakron_oracle.c``;
* one-sided GPTQ, to which the method reduces when ``B = I`` ("Load-bearing
  premise": GPTQ's Hessian is ``E[xx^T] (x) I``).

Readings where the pages are silent:
symmetric grid ``qmax = 2^(b-1)-1``, ``qmin = -qmax``; per-row step
``s_i = absmax_j |W_ij| / qmax`` in fp32 (1 for an all-zero row); ties round half
to even; the decision ``clamp(rint(Wt/s))`` is taken in fp32; clamp error is part
of the residual; "normalised" factors have unit diagonal.

Heavy dense steps use numpy/LAPACK as library primitives (Cholesky, triangular
solve, matmul); the sequential rounding loops are plain C (``bakron_oracle.c``).
"""
from __future__ import annotations

import ctypes
import os
import subprocess
import threading

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "bakron_oracle.c")
_LIB_PATH = os.path.join(_HERE, "liboracle.so")
_lib = None
_lock = threading.Lock()

CFLAGS = ["-O3", "-mavx2", "-mfma", "-fopenmp", "-fPIC", "-shared", "-std=c11"]


def build(force: bool = False) -> str:
    """Compile ``liboracle.so`` next to its source with gcc (checker build only)."""
    if force or not os.path.exists(_LIB_PATH) or os.path.getmtime(_LIB_PATH) < os.path.getmtime(_SRC):
        tmp = _LIB_PATH + f".tmp{os.getpid()}"
        subprocess.run(["gcc", *CFLAGS, "-o", tmp, _SRC, "-lm"], check=True)
        os.replace(tmp, _LIB_PATH)
    return _LIB_PATH


def _load():
    global _lib
    with _lock:
        if _lib is None:
            build()
            lib = ctypes.CDLL(_LIB_PATH)
            dp = ctypes.POINTER(ctypes.c_double)
            fp = ctypes.POINTER(ctypes.c_float)
            ip = ctypes.POINTER(ctypes.c_int32)
            c_int = ctypes.c_int
            lib.bko_pull.argtypes = [c_int, c_int, dp, dp, dp, fp, c_int, c_int, ip, ip, dp, dp, c_int]
            lib.bko_pull_order.argtypes = [c_int, c_int, dp, dp, dp, fp, c_int, c_int, ip, ip, dp]
            lib.bko_antidiag_push.argtypes = [c_int, c_int, dp, dp, dp, fp, c_int, c_int, ip, dp]
            lib.bko_recursive.argtypes = [c_int, c_int, dp, dp, dp, fp, c_int, c_int, c_int, c_int, ip, dp]
            lib.bko_rowcol.argtypes = [c_int, c_int, dp, dp, dp, fp, c_int, c_int, ip, dp]
            lib.bko_naive_vec.argtypes = [c_int, c_int, dp, dp, fp, c_int, c_int, ip, dp]
            lib.bko_brute.argtypes = [c_int, c_int, dp, dp, dp, dp, dp, fp, c_int, c_int, ip, dp, ip]
            lib.bko_brute.restype = ctypes.c_long
            lib.bko_decide.argtypes = [ctypes.c_double, ctypes.c_float, c_int, c_int]
            lib.bko_decide.restype = c_int
            lib.bko_num_threads.restype = c_int
            _lib = lib
    return _lib


def _d(a):
    a = np.ascontiguousarray(a, dtype=np.float64)
    return a, a.ctypes.data_as(ctypes.POINTER(ctypes.c_double))


def _f(a):
    a = np.ascontiguousarray(a, dtype=np.float32)
    return a, a.ctypes.data_as(ctypes.POINTER(ctypes.c_float))


def _i(a):
    a = np.ascontiguousarray(a, dtype=np.int32)
    return a, a.ctypes.data_as(ctypes.POINTER(ctypes.c_int32))


def num_threads() -> int:
    """OpenMP threads the C loops use by default on this host."""
    return int(_load().bko_num_threads())


# --------------------------------------------------------------------------
# Grid (base quantizer): fixed symmetric per-row INT-b grid.
# --------------------------------------------------------------------------
def grid(bits: int) -> tuple[int, int]:
    """Symmetric integer range for ``bits``: ``(-(2^(b-1)-1), 2^(b-1)-1)``."""
    qmax = (1 << (bits - 1)) - 1
    return -qmax, qmax


def scales(W: np.ndarray, qmax: int) -> np.ndarray:
    """Per-row step ``s_i = absmax_j |W_ij| / qmax`` in fp32 IEEE division; 1 for a zero row."""
    W32 = np.asarray(W, dtype=np.float32)
    amax = np.max(np.abs(W32), axis=1) if W32.shape[1] else np.zeros(W32.shape[0], np.float32)
    s = (amax / np.float32(qmax)).astype(np.float32)
    s[amax == 0] = np.float32(1.0)
    return s


def shrink_candidates(grid: int) -> np.ndarray:
    """The searched shrink factors ``c_k = 1 - (1/2) k / (grid - 1)``, k = 0..grid-1,
    from 1 down to 1/2 ("per-row scaling factor (shrink) up to factor 2, MSE
    search" in the review's free-parameter list), each rounded to fp32 as
    ``1 - fp32(k/2) / fp32(grid - 1)``."""
    k = np.arange(grid, dtype=np.float32)
    return (np.float32(1.0) - (np.float32(0.5) * k) / np.float32(grid - 1)).astype(np.float32)


def row_mse(W: np.ndarray, s: np.ndarray, qmin: int, qmax: int) -> np.ndarray:
    """Round-to-nearest error of each row on its grid: ``sum_j (W_ij - s_i q_ij)^2``
    with ``q = clamp(rint(fp32(W_ij / s_i)))``; the sum is taken in FP64."""
    q = decide(W, s, qmin, qmax).astype(np.float64)
    d = np.asarray(W, dtype=np.float32).astype(np.float64) - np.asarray(s, np.float32).astype(np.float64)[:, None] * q
    return np.sum(d * d, axis=1)


def scales_mse(W: np.ndarray, qmin: int, qmax: int, grid: int) -> tuple[np.ndarray, np.ndarray]:
    """Per-row step searched for the least round-to-nearest error: over the
    candidates ``s_k = fp32(fp32(c_k * absmax) / qmax)`` (``c_k`` from
    :func:`shrink_candidates`) the one with the smallest :func:`row_mse`, the
    first (largest step) on equal errors; a zero row keeps ``s = 1``.  Returns
    the steps and, per row, the relative gap between the best and the
    second-best error (where two candidates' errors differ by less than the
    FP64 summation order can, either is a valid answer)."""
    W32 = np.asarray(W, dtype=np.float32)
    amax = np.max(np.abs(W32), axis=1) if W32.shape[1] else np.zeros(W32.shape[0], np.float32)
    cands = shrink_candidates(grid)
    errs = np.empty((W32.shape[0], grid))
    steps = np.empty((W32.shape[0], grid), np.float32)
    for k, c in enumerate(cands):
        sk = ((c * amax).astype(np.float32) / np.float32(qmax)).astype(np.float32)
        sk[amax == 0] = np.float32(1.0)
        steps[:, k] = sk
        errs[:, k] = row_mse(W32, sk, qmin, qmax)
    best = np.argmin(errs, axis=1)  # first index on equal errors
    rows = np.arange(W32.shape[0])
    s = steps[rows, best]
    srt = np.sort(errs, axis=1)
    gap = (srt[:, 1] - srt[:, 0]) / np.maximum(srt[:, 0], 1e-300) if grid > 1 else np.full(W32.shape[0], np.inf)
    return s.astype(np.float32), gap

def decide(Wt: np.ndarray, s: np.ndarray, qmin: int, qmax: int) -> np.ndarray:
    """Rounding decision in fp32: ``clamp(rint(float32(Wt) / s))`` (round half to even)."""
    x = np.asarray(Wt, dtype=np.float32) / np.asarray(s, dtype=np.float32)[:, None]
    return np.clip(np.rint(x), qmin, qmax).astype(np.int32)


def gram(X: np.ndarray, damping: float = 0.0) -> np.ndarray:
    """Kronecker factor from samples (rows of ``X``): ``X^T X / N`` plus
    ``damping * mean(diag) * I`` (the pages' Gram-matrix regularisation), in
    FP64."""
    X64 = np.asarray(X, dtype=np.float64)
    A = X64.T @ X64 / X64.shape[0]
    return A + damping * np.mean(np.diag(A)) * np.eye(A.shape[0])


# --------------------------------------------------------------------------
# Factors.
# --------------------------------------------------------------------------
class NotSPD(ValueError):
    pass


def factor(A: np.ndarray) -> np.ndarray:
    """Lower Cholesky factor ``L`` of ``A^{-1}`` (``L L^T = A^{-1}``), FP64.

    Written as the definition: invert ``A`` through its own Cholesky factor,
    then take the Cholesky factor of the inverse.
    """
    import scipy.linalg as sla

    A = np.asarray(A, dtype=np.float64)
    n = A.shape[0]
    if n == 0:
        return np.zeros((0, 0))
    try:
        C = np.linalg.cholesky(A)
    except np.linalg.LinAlgError as e:
        raise NotSPD(str(e)) from e
    Cinv = sla.solve_triangular(C, np.eye(n), lower=True)
    Ainv = Cinv.T @ Cinv
    Ainv = 0.5 * (Ainv + Ainv.T)
    try:
        return np.linalg.cholesky(Ainv)
    except np.linalg.LinAlgError as e:
        raise NotSPD(str(e)) from e


def normalize(L: np.ndarray) -> np.ndarray:
    """Unit-diagonal factor ``L * diag(L)^{-1}`` (columns scaled by their pivot)."""
    L = np.asarray(L, dtype=np.float64)
    return np.tril(L / np.diag(L)[None, :])


# --------------------------------------------------------------------------
# Solvers (Theorem 3.2's four variants + GPTQ).
# --------------------------------------------------------------------------
def solve(W, LtA, LtB, s, qmin, qmax, mode="pull", T=1, leaf=1, order=None, nthreads=None):
    """Codes of the intended output, computed by one of the variants.

    mode: ``pull`` (anti-diagonal, entry by entry; main oracle), ``order``
    (pull in a given linear extension), ``push`` (literal anti-diagonal with
    rank updates), ``recursive`` (Algorithm 6 over key ranges; ``T`` = 1 for
    entry anti-diagonals, >1 for tile diagonals), ``rowcol`` (BaKron-recursive).
    Returns ``(codes int32 m x n, Wt float64 m x n)``.
    """
    lib = _load()
    W, pW = _d(W)
    m, n = W.shape
    LtA, pA = _d(LtA)
    LtB, pB = _d(LtB)
    s, ps = _f(s)
    codes = np.zeros((m, n), np.int32)
    Wt = np.zeros((m, n), np.float64)
    _, pc = _i(codes)
    _, pw = _d(Wt)
    if m == 0 or n == 0:
        return codes, Wt
    if mode == "pull":
        nt = nthreads or num_threads()
        lib.bko_pull(m, n, pW, pA, pB, ps, qmin, qmax, None, pc, pw, None, nt)
    elif mode == "order":
        o, po = _i(np.asarray(order).reshape(-1, 2))
        lib.bko_pull_order(m, n, pW, pA, pB, ps, qmin, qmax, po, pc, pw)
    elif mode == "push":
        lib.bko_antidiag_push(m, n, pW, pA, pB, ps, qmin, qmax, pc, pw)
    elif mode == "recursive":
        lib.bko_recursive(m, n, pW, pA, pB, ps, qmin, qmax, int(T), int(leaf), pc, pw)
    elif mode == "rowcol":
        lib.bko_rowcol(m, n, pW, pA, pB, ps, qmin, qmax, pc, pw)
    else:
        raise ValueError(mode)
    return codes, Wt


def naive(W, A, B, s, qmin, qmax):
    """BaKron-naive (Algorithm 2): GPTQ on column-major ``vec(W)`` with the
    lower Cholesky factor of ``(A (x) B)^{-1}``, built as an explicit
    ``mn x mn`` matrix.  Small inputs only."""
    lib = _load()
    W, pW = _d(W)
    m, n = W.shape
    H = np.kron(np.asarray(A, np.float64), np.asarray(B, np.float64))  # H[j*m+i, j'*m+i'] = A[j,j'] B[i,i']
    Lh = factor(H)
    Lh, pL = _d(Lh)
    s, ps = _f(s)
    codes = np.zeros((m, n), np.int32)
    Wt = np.zeros((m, n), np.float64)
    _, pc = _i(codes)
    _, pw = _d(Wt)
    lib.bko_naive_vec(m, n, pW, pL, ps, qmin, qmax, pc, pw)
    return codes, Wt


def gptq(W, A, s, qmin, qmax):
    """One-sided GPTQ with Hessian ``A`` on every row (column order 0..n-1).

    Uses GPTQ's own form: ``U`` = upper Cholesky factor of ``A^{-1}``; for each
    column j, quantise, ``err = (w_j - q_j) / U[j,j]``, and subtract
    ``err * U[j, j+1:]`` from the later columns.
    """
    W = np.array(W, dtype=np.float64, copy=True)
    m, n = W.shape
    Ainv = np.linalg.inv(np.asarray(A, np.float64))
    U = np.linalg.cholesky(0.5 * (Ainv + Ainv.T)).T
    codes = np.zeros((m, n), np.int32)
    s = np.asarray(s, np.float32)
    for j in range(n):
        q = decide(W[:, j:j + 1], s, qmin, qmax)[:, 0]
        codes[:, j] = q
        err = (W[:, j] - s.astype(np.float64) * q) / U[j, j]
        W[:, j + 1:] -= np.outer(err, U[j, j + 1:])
    return codes


def brute(W, A, B, LtA, LtB, s, qmin, qmax):
    """Enumerate every code matrix of a tiny (mn <= 8) problem.

    Returns ``(n_consistent, first_consistent_codes, best_loss, best_codes)``.
    """
    lib = _load()
    W, pW = _d(W)
    m, n = W.shape
    LtA, pA = _d(LtA)
    LtB, pB = _d(LtB)
    A, pAA = _d(A)
    B, pBB = _d(B)
    s, ps = _f(s)
    first = np.zeros((m, n), np.int32)
    best = np.zeros((m, n), np.int32)
    _, pf = _i(first)
    _, pb = _i(best)
    bl = ctypes.c_double(0.0)
    cnt = lib.bko_brute(m, n, pW, pA, pB, pAA, pBB, ps, qmin, qmax, pf, ctypes.byref(bl), pb)
    return int(cnt), first, float(bl.value), best


# --------------------------------------------------------------------------
# Loss and checks.
# --------------------------------------------------------------------------
def proxy_loss(W, V, A, B) -> float:
    """``tr((W-V)^T B (W-V) A) = sum_ij (B E)_ij (E A)_ij`` with ``E = W - V``, FP64."""
    E = np.asarray(W, np.float64) - np.asarray(V, np.float64)
    return float(np.sum((np.asarray(B, np.float64) @ E) * (E @ np.asarray(A, np.float64))))


def forced_check(W, LtA, LtB, s, qmin, qmax, codes, tie_eps=1e-6, nthreads=None):
    """Teacher-forced check of a candidate code matrix (e.g. the GPU's).

    Runs the anti-diagonal pull with each residual formed from the candidate's
    code, so one flipped decision does not propagate; at every entry the
    oracle's own fp32 decision on its FP64 ``Wt`` is compared with the
    candidate.  A mismatch is a *tie* when the two codes are adjacent and ``Wt``
    lies within ``tie_eps`` (absolute, weight units) of the midpoint between
    them; any other mismatch is a *failure*.
    """
    lib = _load()
    W, pW = _d(W)
    m, n = W.shape
    LtA, pA = _d(LtA)
    LtB, pB = _d(LtB)
    s32, ps = _f(s)
    cand, pcand = _i(codes)
    own = np.zeros((m, n), np.int32)
    Wt = np.zeros((m, n), np.float64)
    _, po = _i(own)
    _, pw = _d(Wt)
    if m and n:
        lib.bko_pull(m, n, pW, pA, pB, ps, qmin, qmax, pcand, po, pw, None, nthreads or num_threads())
    mis = own != cand
    idx = np.argwhere(mis)
    lo = np.minimum(own, cand)[mis]
    srow = s32.astype(np.float64)[idx[:, 0]] if len(idx) else np.zeros(0)
    dist = np.abs(Wt[mis] - srow * (lo + 0.5)) if len(idx) else np.zeros(0)
    adjacent = (np.abs(own - cand)[mis] == 1) if len(idx) else np.zeros(0, bool)
    tie = adjacent & (dist <= tie_eps)
    return {
        "entries": m * n,
        "mismatches": int(mis.sum()),
        "ties": int(tie.sum()),
        "failures": int((~tie).sum()),
        "max_fail_dist": float(dist[~tie].max()) if (~tie).any() else 0.0,
        "max_tie_dist": float(dist[tie].max()) if tie.any() else 0.0,
        "Wt": Wt,
        "own": own,
    }


def midpoint_distance(Wt, s, qmin, qmax) -> np.ndarray:
    """Distance (weight units) of each ``Wt`` to the nearest decision boundary
    of its row's grid (ignoring boundaries outside the clamp range)."""
    s64 = np.asarray(s, np.float64)[:, None]
    x = np.asarray(Wt, np.float64) / s64
    fl = np.floor(x)
    mid = fl + 0.5
    d = np.abs(x - mid)
    outside = (mid < qmin) | (mid > qmax)
    d = np.where(outside, np.inf, d)
    return d * s64
