"""GPU parity of bakron_factor and bakron_proxy_loss, end-to-end solves with
GPU factors, and device-detected errors (all raised on the host side: bad
inputs are planted in the data, never a fault)."""
import numpy as np
import pytest

import oracle
import workloads
from parity import LOSS_RTOL, TIE_EPS, tie_cap

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def bk():
    import torch

    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    import two_sided_gptq_b200 as bk

    return bk


def _t(x):
    import torch

    return torch.from_numpy(np.ascontiguousarray(x, dtype=np.float32)).cuda()


def fp64_then_rounded(Lg, Lo, label):
    """The factor is computed in FP64 and rounded once to fp32: every entry
    lies within half an fp32 ulp of the oracle's FP64 value, plus the FP64
    path's own error (cond(M) * 2^-52 relative, far below 1e-9 of the largest
    entry for these damped Gram factors)."""
    excess = np.abs(Lg - Lo) - 2.0 ** -24 * np.abs(Lo) * (1 + 2.0 ** -20)
    worst = float(excess.max()) / float(np.abs(Lo).max())
    print(f"[{label}] max (|L - L_oracle| - half ulp) / max|L| = {worst:.3g}")
    assert worst <= 1e-9


@pytest.mark.parametrize("name", ["tiny", "mid"])
def test_factor_matches_oracle(bk, name):
    W, A, B = workloads.generate(name)
    LA, LB = bk.factor(_t(A), _t(B))
    for L, M in ((LA, A), (LB, B)):
        Lg = L.cpu().numpy().astype(np.float64)
        Lo = oracle.factor(M)
        rel = np.linalg.norm(Lg - Lo) / np.linalg.norm(Lo)
        resid = np.abs(Lg @ Lg.T @ M.astype(np.float64) - np.eye(M.shape[0])).max()
        print(name, "factor rel err", rel, "max |L L^T A - I|", resid)
        assert np.all(np.triu(Lg, 1) == 0) and np.all(np.diag(Lg) > 0)
        assert rel <= 1e-5
        fp64_then_rounded(Lg, Lo, f"{name} {M.shape[0]}")


@pytest.mark.slow
@pytest.mark.parametrize("name,side", [("bench", "A"), ("large4", "B")])
def test_factor_full_size_matches_oracle(bk, name, side):
    """bakron_factor at the sizes the solves use: n = 4096 (the 4096 x 4096
    workload's A, 64 panels) and m = 14336 (the 14336 x 4096 workload's B),
    against the oracle's FP64 definition (invert, then Cholesky)."""
    import torch

    _, A, B = workloads.generate(name)
    M = A if side == "A" else B
    L, _ = bk.factor(_t(M), None)
    Lg = L.cpu().numpy().astype(np.float64)
    Lo = oracle.factor(M)
    rel = np.linalg.norm(Lg - Lo) / np.linalg.norm(Lo)
    # ||L L^T M - I||, an identity that does not go through the oracle (FP64 on the device)
    Ld = torch.from_numpy(Lg).cuda()
    R = Ld @ (Ld.T @ torch.from_numpy(M.astype(np.float64)).cuda())
    R.diagonal().sub_(1.0)
    resid = float(R.abs().max())
    print(f"[{name} {side}, {M.shape[0]}] factor rel err {rel:.3g}, max |L L^T M - I| {resid:.3g}")
    assert np.all(np.triu(Lg, 1) == 0) and np.all(np.diag(Lg) > 0)
    assert rel <= 1e-5
    fp64_then_rounded(Lg, Lo, f"{name} {side} {M.shape[0]}")


# one panel, ragged panels, and sizes whose recursive inverse splits unevenly
@pytest.mark.parametrize("n", [1, 2, 63, 64, 65, 127, 129, 200, 513, 1000, 2111])
def test_factor_sizes(bk, n):
    _, A, _ = workloads.random_problem(2, n, seed=n)
    LA, _ = bk.factor(_t(A), None)
    Lg = LA.cpu().numpy().astype(np.float64)
    Lo = oracle.factor(A)
    assert np.linalg.norm(Lg - Lo) / np.linalg.norm(Lo) <= 1e-5
    assert np.all(np.triu(Lg, 1) == 0)
    fp64_then_rounded(Lg, Lo, f"n={n}")


def test_factor_not_spd(bk):
    A = np.eye(70, dtype=np.float32)
    A[40, 40] = -1.0
    with pytest.raises(bk.BakronError) as e:
        bk.factor(_t(A), None)
    assert e.value.status == bk.Status.ERR_NOT_SPD


def test_factor_nonfinite(bk):
    A = np.eye(30, dtype=np.float32)
    A[20, 3] = np.nan
    with pytest.raises(bk.BakronError) as e:
        bk.factor(_t(A), None)
    assert e.value.status in (bk.Status.ERR_NONFINITE, bk.Status.ERR_NOT_SPD)


def test_solve_device_errors(bk):
    W, A, B = workloads.random_problem(50, 60, seed=1)
    LA = oracle.factor(A).astype(np.float32)
    LB = oracle.factor(B).astype(np.float32)
    Wn = W.copy()
    Wn[3, 7] = np.inf
    with pytest.raises(bk.BakronError) as e:
        bk.solve(_t(Wn), _t(LA), _t(LB))
    assert e.value.status == bk.Status.ERR_NONFINITE
    LAz = LA.copy()
    LAz[10, 10] = 0.0
    with pytest.raises(bk.BakronError) as e:
        bk.solve(_t(W), _t(LAz), _t(LB))
    assert e.value.status == bk.Status.ERR_BAD_FACTOR
    # the status is cleared after it has been read: a good solve passes
    bk.solve(_t(W), _t(LA), _t(LB))


@pytest.mark.parametrize("name", ["tiny", "mid", (200, 333), (129, 1), (1, 130),
                                  pytest.param("bench", marks=pytest.mark.slow)])
def test_proxy_loss_matches_oracle(bk, name):
    """bakron_proxy_loss (both products on the tensor cores in 3xTF32, FP64
    dot) against the oracle's FP64 tr((W-V)^T B (W-V) A); ragged shapes pad
    every operand to whole tiles with zeros."""
    if isinstance(name, tuple):
        m, n = name
        W, A, B = workloads.random_problem(m, n, seed=m + n)
    else:
        W, A, B = workloads.generate(name)
    LA = oracle.factor(A).astype(np.float32)
    LB = oracle.factor(B).astype(np.float32)
    Wd = _t(W)
    V, codes, s = bk.solve(Wd, _t(LA), _t(LB), bits=4)
    l_gpu = bk.proxy_loss(Wd, V, _t(A), _t(B))
    l_or = oracle.proxy_loss(W, V.cpu().numpy(), A, B)
    print(name, "loss gpu", l_gpu, "oracle", l_or)
    assert abs(l_gpu - l_or) <= LOSS_RTOL * abs(l_or)
    # fixed-order reduction: repeated calls agree to the last bit
    assert all(bk.proxy_loss(Wd, V, _t(A), _t(B)) == l_gpu for _ in range(3))


@pytest.mark.parametrize("name", ["tiny", "mid", pytest.param("bench", marks=pytest.mark.slow)])
def test_end_to_end_gpu_factors(bk, name):
    """factor and solve both on the GPU, checked against the oracle running
    from its own FP64 factors: the fp32 factor rounding moves pre-rounding
    values by far less than the tie window, so the same contract holds (the
    4096 x 4096 case is the workload the benchmark times, factor included)."""
    W, A, B = workloads.generate(name)
    LA, LB = bk.factor(_t(A), _t(B))
    Wd = _t(W)
    V, codes, s = bk.solve(Wd, LA, LB, bits=4)
    qmin, qmax = oracle.grid(4)
    s_or = oracle.scales(W, qmax)
    LtA = oracle.normalize(oracle.factor(A))
    LtB = oracle.normalize(oracle.factor(B))
    r = oracle.forced_check(W, LtA, LtB, s_or, qmin, qmax, codes.cpu().numpy().astype(np.int32), tie_eps=TIE_EPS)
    print(name, "e2e mismatches", r["mismatches"], "ties", r["ties"], "failures", r["failures"],
          "max tie dist", r["max_tie_dist"])
    assert r["failures"] == 0 and r["ties"] <= tie_cap(W.size)


@pytest.mark.parametrize("shape,leaf", [((150, 270), 0), ((1000, 300), 0), ((300, 1000), 6), ((640, 384), 7),
                                        ((129, 1), 5), ((1, 257), 3)])
def test_solve_host_buffers(bk, shape, leaf):
    """bakron_solve_host (row blocks of V and codes copied back while the solve
    runs, on the library's copy stream) equals the device solve, for tall and
    wide shapes and for leaf structures whose launches cover one or two tile
    diagonals; pinned host buffers, so the copies are asynchronous."""
    import torch

    m, n = shape
    W, A, B = workloads.random_problem(m, n, seed=m + 3 * n)
    LA = oracle.factor(A).astype(np.float32)
    LB = oracle.factor(B).astype(np.float32)
    pin = lambda x: torch.from_numpy(x).pin_memory()
    Vh, ch, sh = bk.solve_host(pin(W), pin(LA), pin(LB), bits=4, leaf=leaf)
    Vd, cd, sd = bk.solve(_t(W), _t(LA), _t(LB), bits=4, leaf=leaf)
    assert np.array_equal(ch.numpy(), cd.cpu().numpy())
    assert np.array_equal(Vh.numpy(), Vd.cpu().numpy())
    assert np.array_equal(sh.numpy(), sd.cpu().numpy())


@pytest.mark.parametrize("shape", [(1000, 300), (8192, 256), (77, 130)])
def test_gram_matches_oracle(shape):
    """bakron_gram (3xTF32 tensor-core X^T X, FP32 per-chunk sums) against the
    FP64 definition: relative error per entry within 1e-5 of the diagonal scale."""
    import torch

    import two_sided_gptq_b200 as bk

    N, d = shape
    rng = np.random.default_rng(N + d)
    X = (rng.standard_normal((N, d)) * rng.uniform(0.5, 2.0, size=d)).astype(np.float32)
    A = bk.gram(torch.from_numpy(X).cuda(), 0.01).cpu().numpy()
    ref = oracle.gram(X, 0.01)
    err = np.abs(A - ref).max() / np.abs(np.diag(ref)).max()
    print(f"[gram {N}x{d}] max rel err {err:.2e}")
    assert err < 1e-5
    assert np.array_equal(A, A.T)
