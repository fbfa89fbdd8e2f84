"""The seeded input generator matches its documented recipes (shapes, seeds,
damping, outliers, spectrum) and is deterministic; host only, small sizes."""
import dataclasses

import numpy as np
import pytest

import workloads


def test_named_shapes_grids_and_determinism(tmp_path, monkeypatch):
    for name, (m, n, bits) in {"tiny": (64, 128, 4), "tiny_bI": (64, 128, 4), "mid": (1024, 1024, 4),
                               "bench": (4096, 4096, 4), "mlp_up": (11008, 4096, 3),
                               "mlp_down": (4096, 11008, 3), "large2": (14336, 4096, 2),
                               "large4": (14336, 4096, 4)}.items():
        w = workloads.WORKLOADS[name]
        assert (w.m, w.n, w.bits) == (m, n, bits) and w.qmax == (1 << (bits - 1)) - 1 and w.qmin == -w.qmax
    monkeypatch.delenv("BAKRON_WORKLOAD_CACHE", raising=False)
    a = workloads.generate("tiny")
    b = workloads.generate("tiny")
    assert all(np.array_equal(x, y) for x, y in zip(a, b))
    assert all(x.dtype == np.float32 and x.flags.c_contiguous for x in a)
    c = workloads.generate("tiny", seed=1)
    assert not np.array_equal(a[0], c[0])
    # the cache returns the same arrays
    monkeypatch.setenv("BAKRON_WORKLOAD_CACHE", str(tmp_path))
    d = workloads.generate("tiny")
    e = workloads.generate("tiny")
    assert all(np.array_equal(x, y) for x, y in zip(a, d)) and all(np.array_equal(x, y) for x, y in zip(a, e))


def test_tiny_factors_spd_with_damping_and_B_identity(monkeypatch):
    monkeypatch.delenv("BAKRON_WORKLOAD_CACHE", raising=False)
    W, A, B = workloads.generate("tiny")
    assert W.shape == (64, 128) and A.shape == (128, 128) and B.shape == (64, 64)
    assert abs(float(W.std()) - 0.02) < 0.002
    for F in (A, B):
        F64 = F.astype(np.float64)
        assert np.array_equal(F, F.T)
        ev = np.linalg.eigvalsh(F64)
        # damping adds 1% of the mean diagonal: no eigenvalue below ~0.99% of it
        assert ev.min() >= 0.0099 * np.mean(np.diag(F64)) / 1.01
    _, _, I = workloads.generate("tiny_bI")
    assert np.array_equal(I, np.eye(64, dtype=np.float32))


def test_outlier_channels_and_heavy_tails():
    w = dataclasses.replace(workloads.WORKLOADS["mid"], n=200)
    g = workloads.rng(3, 1)
    X = workloads._samples("outlier_gauss", 4000, 200, g, w)
    var = X.astype(np.float64).var(axis=0)
    big = var > 20.0  # scaled channels have variance ~400
    assert big.sum() == 2  # 1% of 200
    T = workloads._samples("student_t", 4000, 50, workloads.rng(4, 1), w).astype(np.float64).ravel()
    kurt = np.mean((T - T.mean()) ** 4) / np.var(T) ** 2
    assert kurt > 5.0  # Gaussian: 3; Student-t(4) has infinite kurtosis


def test_decaying_spectrum_condition_number():
    """X = Z diag(sigma) Q^T with sigma_k^2 = 10^(-4k/(d-1)): the sample Gram's
    eigenvalues span about 1e4 before damping."""
    w = workloads.WORKLOADS["bench"]
    d, N = 48, 48 * 200
    X = workloads._samples("decaying_spectrum", N, d, workloads.rng(5, 1), w).astype(np.float64)
    ev = np.linalg.eigvalsh(X.T @ X / N)
    assert 3e3 < ev.max() / ev.min() < 3e4


@pytest.mark.parametrize("shape", [(1, 1), (5, 9), (40, 17)])
def test_random_problem_is_spd_and_seeded(shape):
    m, n = shape
    W, A, B = workloads.random_problem(m, n, seed=11)
    W2, A2, B2 = workloads.random_problem(m, n, seed=11)
    assert np.array_equal(W, W2) and np.array_equal(A, A2) and np.array_equal(B, B2)
    assert W.shape == (m, n) and A.shape == (n, n) and B.shape == (m, m)
    for F in (A, B):
        assert np.linalg.eigvalsh(F.astype(np.float64)).min() > 0
