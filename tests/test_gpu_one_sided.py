"""GPU parity of the one-sided path (B = I, ``LB=None``): the column-block
recursion with the one-sided leaf and the tensor-core update, against the
oracle's pull with an identity row factor (teacher-forced, the contract in
tests/parity.py) and, where no entry sits at a tie, against GPTQ's own form
(``oracle.gptq``: updates through the upper Cholesky factor of A^{-1})."""
import numpy as np
import pytest

import oracle
import workloads
from parity import check_solve, gpu_solve, oracle_factors

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def _cuda():
    import torch

    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    import two_sided_gptq_b200 as bk

    bk._lib()


def _wt_ok(r):
    # the pre-rounding values the leaf wrote match the oracle's FP64 ones
    assert r["wt_max_abs_err"] <= 1e-4 * max(1.0, r["wt_scale"]), (r["wt_max_abs_err"], r["wt_scale"])


def test_tiny_equals_gptq():
    W, A, B = workloads.generate("tiny_bI")
    LA, _ = oracle_factors(A, B)
    _, codes, s, _ = gpu_solve(W, LA, None, 4)
    qmin, qmax = oracle.grid(4)
    assert np.array_equal(codes, oracle.gptq(W, A, s, qmin, qmax))
    _wt_ok(check_solve(W, LA, None, 4, label="tiny_bI/one-sided"))


# one block, several blocks and levels, ragged in either direction, degenerate
SHAPES = [(1, 1), (1, 300), (300, 1), (31, 128), (129, 257), (200, 333), (77, 1000), (33, 1536), (256, 2048)]


@pytest.mark.parametrize("shape", SHAPES)
def test_shapes(shape):
    m, n = shape
    W, A, B = workloads.random_problem(m, n, seed=7 * m + n)
    LA, _ = oracle_factors(A, B)
    _wt_ok(check_solve(W, LA, None, 4, label=f"{m}x{n}/one-sided"))


@pytest.mark.parametrize("bits", [2, 3, 8])
def test_other_grids(bits):
    W, A, B = workloads.random_problem(96, 700, seed=bits)
    LA, _ = oracle_factors(A, B)
    check_solve(W, LA, None, bits, label=f"96x700/one-sided/{bits}b")


def test_zero_row_and_user_scales():
    W, A, B = workloads.random_problem(64, 300, seed=5)
    W[3] = 0.0
    LA, _ = oracle_factors(A, B)
    check_solve(W, LA, None, 4, label="zero row/one-sided")
    s = oracle.scales(W, oracle.grid(4)[1]) * np.float32(0.75)
    s[3] = np.float32(1.0)
    check_solve(W, LA, None, 4, row_scale=s, label="user steps/one-sided")


def test_host_buffers_and_repeat():
    """solve_host with LB=None equals the device call, and two device calls agree bit for bit."""
    import torch

    import two_sided_gptq_b200 as bk

    W, A, B = workloads.random_problem(200, 333, seed=11)
    LA, _ = oracle_factors(A, B)
    Wd, LAd = torch.from_numpy(W).cuda(), torch.from_numpy(LA).cuda()
    V1, c1, s1 = bk.solve(Wd, LAd, None, bits=4)
    V2, c2, s2 = bk.solve(Wd, LAd, None, bits=4)
    assert torch.equal(c1, c2) and torch.equal(V1, V2) and torch.equal(s1, s2)
    Vh, ch, sh = bk.solve_host(torch.from_numpy(W), torch.from_numpy(LA), None, bits=4)
    assert torch.equal(ch, c1.cpu()) and torch.equal(Vh, V1.cpu()) and torch.equal(sh, s1.cpu())


@pytest.mark.slow
@pytest.mark.parametrize("name", ["mid", "bench"])
def test_full_size(name):
    W, A, B = workloads.generate(name)
    LA, _ = oracle_factors(A, B)
    check_solve(W, LA, None, workloads.WORKLOADS[name].bits, label=f"{name}/one-sided")
