"""GPU parity of the BaKron solve against the oracle (calls the C ABI through
the Python binding).  See tests/parity.py for the contract."""
import numpy as np
import pytest

import oracle
import workloads
from parity import check_outputs, check_solve, gpu_solve, gpu_solve_canaries, oracle_factors

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def _cuda():
    import torch

    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    import two_sided_gptq_b200 as bk

    bk._lib()


_cache = {}


def named(name):
    key = "large" if name in ("large2", "large4") else name  # same inputs, two grids
    if key not in _cache:
        W, A, B = workloads.generate(name)
        LA, LB = oracle_factors(A, B)
        _cache[key] = (W, A, B, LA, LB)
    return _cache[key]


@pytest.mark.parametrize("gemm", [0, 1])
@pytest.mark.parametrize("name", ["tiny", "tiny_bI", "mid"])
def test_named_workloads(name, gemm):
    W, A, B, LA, LB = named(name)
    check_solve(W, LA, LB, workloads.WORKLOADS[name].bits, gemm=gemm, label=f"{name}/gemm{gemm}")


def test_tiny_B_identity_equals_gptq():
    """B = I: the GPU codes equal one-sided GPTQ's (oracle, GPTQ's own form)."""
    W, A, B, LA, LB = named("tiny_bI")
    _, codes, s, _ = gpu_solve(W, LA, LB, 4)
    qmin, qmax = oracle.grid(4)
    assert np.array_equal(codes, oracle.gptq(W, A, s, qmin, qmax))


# ragged shapes: several tiles and a ragged tail in either direction, plus
# degenerate single-row / single-column / single-entry problems
RAGGED = [(1, 1), (1, 300), (300, 1), (129, 257), (257, 129), (200, 333), (384, 640), (77, 1000)]


@pytest.mark.parametrize("gemm", [0, 1])
@pytest.mark.parametrize("shape", RAGGED)
def test_ragged_shapes(shape, gemm):
    m, n = shape
    W, A, B = workloads.random_problem(m, n, seed=m * 1000 + n)
    LA, LB = oracle_factors(A, B)
    check_solve(W, LA, LB, 4, gemm=gemm, label=f"{m}x{n}/gemm{gemm}")


@pytest.mark.parametrize("leaf", [3, 5, 6, 7, 8])
@pytest.mark.parametrize("shape", RAGGED)
def test_ragged_shapes_canary_write_only_their_buffers(shape, leaf):
    """Canary-padded workspace and outputs (guard zones of a known byte
    pattern before and after every buffer): no kernel of the solve writes
    outside what it was given, on every ragged shape; the codes still pass
    the oracle contract."""
    m, n = shape
    W, A, B = workloads.random_problem(m, n, seed=m * 1000 + n)
    LA, LB = oracle_factors(A, B)
    V, codes, s = gpu_solve_canaries(W, LA, LB, 4, leaf=leaf)
    check_outputs(W, LA, LB, 4, V, codes, s, label=f"{m}x{n}/canary/leaf{leaf}")


@pytest.mark.parametrize("bits", [2, 3, 8])
def test_other_grids(bits):
    W, A, B = workloads.random_problem(300, 260, seed=bits)
    LA, LB = oracle_factors(A, B)
    check_solve(W, LA, LB, bits, label=f"int{bits}")


def test_zero_row_and_user_scales():
    W, A, B = workloads.random_problem(140, 150, seed=3)
    W[5] = 0.0
    LA, LB = oracle_factors(A, B)
    r = check_solve(W, LA, LB, 4, label="zero-row")
    rs = np.full(140, 0.004, np.float32)
    check_solve(W, LA, LB, 4, row_scale=rs, label="user-scales")
    del r


def test_deterministic():
    W, A, B, LA, LB = named("mid")
    a = gpu_solve(W, LA, LB, 4)
    b = gpu_solve(W, LA, LB, 4)
    assert np.array_equal(a[1], b[1]) and np.array_equal(a[3], b[3])


def test_tensor_core_and_fp32_paths_agree():
    """The 3xTF32 tensor-core band products and the FP32 CUDA-core ones give
    pre-rounding values within FP32-level error of each other."""
    W, A, B, LA, LB = named("mid")
    _, c0, _, wt0 = gpu_solve(W, LA, LB, 4, gemm=0)
    _, c1, _, wt1 = gpu_solve(W, LA, LB, 4, gemm=1)
    err = np.abs(wt0.astype(np.float64) - wt1).max()
    print("tc vs simt max |dWt| =", err, " code mismatches =", int((c0 != c1).sum()))
    assert err < 1e-5 * np.abs(W).max() * 10


@pytest.mark.parametrize("case", ["mid", (300, 260), (129, 257), (1, 300)])
def test_leaf_variants(case):
    """The other leaf structures (one anti-diagonal sweep per 128 x 128 tile;
    4 x 4 sub-tiles of 32 swept one warp each) meet the same contract as the
    default."""
    if isinstance(case, str):
        W, A, B, LA, LB = named(case)
        label = case
    else:
        m, n = case
        W, A, B = workloads.random_problem(m, n, seed=m + 7 * n)
        LA, LB = oracle_factors(A, B)
        label = f"{m}x{n}"
    for leaf in (1, 2, 3, 4, 5, 6, 7, 8):
        check_solve(W, LA, LB, 4, leaf=leaf, label=f"{label}/leaf{leaf}")


@pytest.mark.parametrize("case", ["mid", (300, 260), (129, 1000), (1000, 129), (640, 384)])
def test_fused_node_widths(case):
    """Both band products of a node in one launch (X in tensor memory) against
    the two-launch form: the same oracle contract whether no node, the narrow
    nodes (the default) or every node runs fused."""
    if case == "mid":
        W, A, B, LA, LB = named("mid")
        label = "mid"
    else:
        m, n = case
        W, A, B = workloads.random_problem(m, n, seed=3 * m + n)
        LA, LB = oracle_factors(A, B)
        label = f"{m}x{n}"
    for fw in (1, 2, 0, 65535):
        check_solve(W, LA, LB, 4, fuse_width=fw, label=f"{label}/fuse{fw}")


@pytest.mark.slow
@pytest.mark.parametrize("name", ["bench", "large4"])
def test_two_diagonal_leaves_full_size(name):
    """Leaf structure 7 (two tile diagonals per launch, device flags, the
    width-2 nodes' updates inside the leaf) on the 4096 x 4096 and the
    14336 x 4096 workloads, every entry checked."""
    W, A, B, LA, LB = named(name)
    check_solve(W, LA, LB, workloads.WORKLOADS[name].bits, leaf=7, label=f"{name}/leaf7")


@pytest.mark.slow
def test_bench_workload_4096():
    W, A, B, LA, LB = named("bench")
    check_solve(W, LA, LB, 4, label="bench4096")


@pytest.mark.slow
@pytest.mark.parametrize("name", ["mlp_up", "mlp_down", "large2", "large4"])
def test_full_size_workloads(name):
    """The remaining full-size workloads (transformer MLP shapes at INT3 and the
    14336 x 4096 Table 3 shape at INT2 and INT4): teacher-forced check of every
    entry against the oracle."""
    W, A, B, LA, LB = named(name)
    check_solve(W, LA, LB, workloads.WORKLOADS[name].bits, label=name)
    if name != "large2":
        _cache.pop("large" if name == "large4" else name, None)


def test_tune_leaf_picks_a_measured_structure():
    """bakron_tune_leaf times every leaf structure on the problem and returns
    the fastest; its outputs meet the parity contract."""
    import torch

    import two_sided_gptq_b200 as bk

    W, A, B, LA, LB = named("mid")
    Wd, LAd, LBd = (torch.from_numpy(x).cuda() for x in (W, LA.astype(np.float32), LB.astype(np.float32)))
    leaf, ms = bk.tune_leaf(Wd, LAd, LBd, bits=4)
    assert leaf in (1, 2, 3, 4, 5, 6, 7, 8) and all(t > 0 for t in ms)
    assert ms[leaf - 1] == min(ms)
    check_solve(W, LA, LB, 4, leaf=leaf, label=f"mid/tuned-leaf{leaf}")


def test_tune_leaf_cache(tmp_path):
    """With a cache file the first call measures and stores, the second returns
    the stored measurement for the same (m, n, bits, GPU)."""
    import torch

    import two_sided_gptq_b200 as bk

    W, A, B, LA, LB = named("mid")
    Wd, LAd, LBd = (torch.from_numpy(x).cuda() for x in (W, LA.astype(np.float32), LB.astype(np.float32)))
    path = str(tmp_path / "tune.json")
    first = bk.tune_leaf(Wd, LAd, LBd, bits=4, cache=path)
    key = bk.tune_cache_key(1024, 1024, 4, torch.cuda.get_device_name(0))
    assert bk.tune_cache_get(path, key) == first
    assert bk.tune_leaf(Wd, LAd, LBd, bits=4, cache=path) == first


@pytest.mark.parametrize("case", [("mid", 4, 100), ((300, 260), 3, 64), ((129, 257), 2, 20)])
def test_mse_searched_steps(case):
    """shrink_grid: the device's searched steps equal the oracle's (a row whose
    two best candidates' errors lie within 1e-12 of each other may take either:
    FP64 summation order decides there), and the solve on those steps meets the
    parity contract."""
    import torch

    import two_sided_gptq_b200 as bk

    what, bits, grid = case
    if isinstance(what, str):
        W, A, B, LA, LB = named(what)
    else:
        W, A, B = workloads.random_problem(*what, seed=sum(what) + grid)
        LA, LB = oracle_factors(A, B)
    qmin, qmax = oracle.grid(bits)
    Wd, LAd, LBd = (torch.from_numpy(x).cuda() for x in (W, LA, LB))
    _, _, s_gpu = bk.solve(Wd, LAd, LBd, bits=bits, shrink_grid=grid)
    s_gpu = s_gpu.cpu().numpy()
    s_or, gap = oracle.scales_mse(W, qmin, qmax, grid)
    diff = s_gpu != s_or
    print(f"[mse {what}] rows {len(s_or)} differing {int(diff.sum())} shrunk {int((s_or < oracle.scales(W, qmax)).sum())}")
    assert np.all(gap[diff] < 1e-12), (np.nonzero(diff)[0][:5], gap[diff][:5])
    assert (s_or < oracle.scales(W, qmax)).any()  # the search does move some steps
    check_solve(W, LA, LB, bits, row_scale=s_gpu, label=f"{what}/mse{grid}")


def test_solve_batch_equals_single_solves():
    """bakron_solve_batch: independent solves of different shapes on two
    streams give the same results as one-at-a-time solves."""
    import torch

    import two_sided_gptq_b200 as bk

    probs = []
    for (m, n) in ((300, 260), (129, 257), (256, 512)):
        W, A, B = workloads.random_problem(m, n, seed=m * 7 + n)
        LA, LB = oracle_factors(A, B)
        probs.append(tuple(torch.from_numpy(x).cuda() for x in (W, LA, LB)))
    streams = [torch.cuda.Stream(), torch.cuda.Stream()]
    res = bk.solve_batch(probs, bits=4, streams=streams)
    torch.cuda.synchronize()
    for (W, LA, LB), (V, codes, scales) in zip(probs, res):
        V1, c1, s1 = bk.solve(W, LA, LB, bits=4)
        assert torch.equal(codes, c1) and torch.equal(scales, s1) and torch.equal(V, V1)
