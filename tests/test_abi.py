"""C-ABI checks that need no GPU: the library builds and loads, exports every
function include/bakron.h declares, and its host-only entry points behave."""
import ctypes
import os
import re
import sys

import pytest

from conftest import ROOT

HEADER = os.path.join(ROOT, "include", "bakron.h")


@pytest.fixture(scope="module")
def lib():
    from two_sided_gptq_b200 import _native, build

    build.build()
    return _native.load()


def declared_functions():
    text = open(HEADER).read()
    text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
    return sorted(set(re.findall(r"\b(bakron_[a-z_]+)\s*\(", text)))


def test_every_declared_symbol_is_exported(lib):
    from two_sided_gptq_b200 import _native

    names = declared_functions()
    assert len(names) >= 12
    for name in names:
        assert hasattr(lib, name), name
    assert set(names) == set(_native.SIGNATURES), "binding signatures must mirror the header"


def test_library_is_sm100a_build():
    from two_sided_gptq_b200 import build

    assert "arch=compute_100a,code=sm_100a" in " ".join(build.FLAGS)


def test_host_only_queries(lib):
    from two_sided_gptq_b200 import _native

    assert lib.bakron_version().decode().startswith("bakron-b200")
    assert lib.bakron_status_string(3).decode().startswith("matrix is not")
    assert lib.bakron_solve_workspace_size(0, 5, None) == 0
    ws = lib.bakron_solve_workspace_size(4096, 4096, None)
    # Wt, D hi/lo, X^T hi/lo (5 x m n) + three copies of each factor
    assert ws >= 4 * (5 * 4096 * 4096 + 6 * 4096 * 4096)
    assert lib.bakron_solve_host_workspace_size(100, 70, None) > lib.bakron_solve_workspace_size(100, 70, None)
    assert lib.bakron_factor_workspace_size(300, 200) >= 2 * 300 * 300 * 8
    # status block; E, E^T, B, A hi / lo and the two products, each padded to
    # 128-multiples; 592 FP64 partial sums (1024-byte aligned)
    assert lib.bakron_proxy_loss_workspace_size(3, 4) == 1024 + 10 * 128 * 128 * 4 + 5120
    assert lib.bakron_proxy_loss_workspace_size(4096, 4096) == 1024 + 10 * 4096 * 4096 * 4 + 5120
    assert lib.bakron_proxy_loss_workspace_size(200, 300) == 1024 + (6 * 256 * 384 + 2 * 256 * 256 + 2 * 384 * 384) * 4 + 5120
    bad = _native.Config(64, 0, 0, 0, None)  # unsupported tile
    assert lib.bakron_solve_workspace_size(10, 10, ctypes.byref(bad)) == 0


def test_argument_errors_return_before_any_device_work(lib):
    from two_sided_gptq_b200 import _native

    q = _native.Quantizer(4, 0, 0, None)
    fake = 1 << 20  # aligned, never dereferenced: validation fails first
    args = lambda W=fake, m=8, n=8, ws=fake, wsb=1 << 30: (W, m, n, fake, fake, ctypes.byref(q), fake, fake, fake,
                                                           ws, wsb, None, None)
    assert lib.bakron_solve(*args(m=0)) == _native.Status.ERR_INVALID_ARG
    assert lib.bakron_solve(*args(n=-3)) == _native.Status.ERR_INVALID_ARG
    assert lib.bakron_solve(*args(W=None)) == _native.Status.ERR_INVALID_ARG
    assert lib.bakron_solve(*args(ws=None)) == _native.Status.ERR_WORKSPACE
    assert lib.bakron_solve(*args(W=fake + 4)) == _native.Status.ERR_ALIGNMENT
    assert lib.bakron_solve(*args(wsb=100)) == _native.Status.ERR_WORKSPACE
    q_bad = _native.Quantizer(9, 0, 0, None)
    a = list(args())
    a[5] = ctypes.byref(q_bad)
    assert lib.bakron_solve(*a) == _native.Status.ERR_INVALID_ARG
    q_bad = _native.Quantizer(4, 3, -3, None)
    a[5] = ctypes.byref(q_bad)
    assert lib.bakron_solve(*a) == _native.Status.ERR_INVALID_ARG
    for grid in (1, -2, 1025):  # the step search takes 2..1024 candidates
        q_bad = _native.Quantizer(4, 0, 0, None, grid)
        a[5] = ctypes.byref(q_bad)
        assert lib.bakron_solve(*a) == _native.Status.ERR_INVALID_ARG
    cfg = _native.Config(0, 5, 0, 0, None)
    a = list(args())
    a[11] = ctypes.byref(cfg)
    assert lib.bakron_solve(*a) == _native.Status.ERR_INVALID_ARG
    # use_graph is 0 or 1, and not with per-launch profiling
    for bad in (_native.Config(0, 0, 2, 0, None), _native.Config(0, 0, 1, 0, None, 1)):
        a[11] = ctypes.byref(bad)
        assert lib.bakron_solve(*a) == _native.Status.ERR_INVALID_ARG
    # b_identity is 0 or 1; LB may be NULL only on the one-sided path
    cfg = _native.Config(0, 0, 0, 0, None, 0, 0, 2)
    a[11] = ctypes.byref(cfg)
    assert lib.bakron_solve(*a) == _native.Status.ERR_INVALID_ARG
    # fuse_width is 0 (default), 1 (never) or a width up to 65535
    for fw in (-1, 65536):
        cfg = _native.Config(0, 0, 0, 0, None, 0, 0, 0, fw)
        a[11] = ctypes.byref(cfg)
        assert lib.bakron_solve(*a) == _native.Status.ERR_INVALID_ARG
    a = list(args())
    a[4] = None
    assert lib.bakron_solve(*a) == _native.Status.ERR_INVALID_ARG
    cfg = _native.Config(0, 0, 0, 0, None, 0, 0, 1)
    a[11] = ctypes.byref(cfg)
    a[0] = fake + 4  # with LB = NULL accepted, validation goes on to the next check
    assert lib.bakron_solve(*a) == _native.Status.ERR_ALIGNMENT
    # the bounded-wait self-test validates before it launches anything
    assert lib.bakron_selftest_wait_timeout(0, fake, 256, None) == _native.Status.ERR_INVALID_ARG
    assert lib.bakron_selftest_wait_timeout(10001, fake, 256, None) == _native.Status.ERR_INVALID_ARG
    assert lib.bakron_selftest_wait_timeout(5, None, 256, None) == _native.Status.ERR_WORKSPACE
    assert lib.bakron_selftest_wait_timeout(5, fake, 255, None) == _native.Status.ERR_WORKSPACE
    assert lib.bakron_selftest_wait_timeout(5, fake + 8, 256, None) == _native.Status.ERR_ALIGNMENT
    need = lib.bakron_selftest_band_abort_workspace_size()
    assert need >= 256 + 6 * 256 * 256 * 4
    assert lib.bakron_selftest_band_abort(0, fake, need, None) == _native.Status.ERR_INVALID_ARG
    assert lib.bakron_selftest_band_abort(5, None, need, None) == _native.Status.ERR_WORKSPACE
    assert lib.bakron_selftest_band_abort(5, fake, need - 1, None) == _native.Status.ERR_WORKSPACE
    assert lib.bakron_selftest_band_abort(5, fake + 8, need, None) == _native.Status.ERR_ALIGNMENT
    assert lib.bakron_factor(fake, -1, fake, 4, fake, fake, fake, 1 << 30, None) == _native.Status.ERR_INVALID_ARG
    assert lib.bakron_factor(fake, 4, fake, 4, fake + 8, fake, fake, 1 << 30, None) == _native.Status.ERR_ALIGNMENT
    assert lib.bakron_factor(fake, 4, fake, 4, fake, fake, fake, 16, None) == _native.Status.ERR_WORKSPACE
    assert lib.bakron_proxy_loss(fake, fake, fake, fake, 0, 4, fake, None, fake, 256, None) == \
        _native.Status.ERR_INVALID_ARG
    assert lib.bakron_proxy_loss(fake, fake, fake, fake, 4, 4, fake, None, fake, 1031, None) == \
        _native.Status.ERR_WORKSPACE


def _brute_schedule_flops(Mt, Nt, T=128):
    """Independent count of the tile-cut schedule's band-product FLOPs.

    For every node of the midpoint recursion over tile diagonals, enumerate
    all (source tile, target tile) pairs with source <= target; X(I, J') is
    needed when some pair links row I to column J'; stage 1 costs one tile
    product per source tile (I, J) with J <= J' for every needed X(I, J');
    stage 2 one per needed X(I, J') with I <= I' for every target (I', J')."""
    tiles = [(I, J) for I in range(Mt) for J in range(Nt)]
    total = [0.0, 0.0]
    diag = [0, 0]  # products whose factor tile is on the diagonal (lower triangular)

    def rec(k, l):
        if l <= 1:
            return
        h = l // 2
        rec(k, h)
        src = [(I, J) for (I, J) in tiles if k <= I + J < k + h]
        tgt = [(I, J) for (I, J) in tiles if k + h <= I + J < k + l]
        need = set()
        for (I, J) in src:
            for (I2, J2) in tgt:
                if I <= I2 and J <= J2:
                    need.add((I, J2))
        for (I, J2) in need:
            total[0] += sum(1 for (a, b) in src if a == I and b <= J2)
            diag[0] += sum(1 for (a, b) in src if a == I and b == J2)
        for (I2, J2) in tgt:
            total[1] += sum(1 for (I, Jx) in need if Jx == J2 and I <= I2)
            diag[1] += sum(1 for (I, Jx) in need if Jx == J2 and I == I2)
        rec(k + h, l - h)

    rec(0, Mt + Nt - 1)
    f = 2.0 * T ** 3
    structural = (total[0] + total[1] - diag[0] - diag[1]) * f + (diag[0] + diag[1]) * T * T * (T + 1)
    return total[0] * f, total[1] * f, structural


@pytest.mark.parametrize("shape", [(1, 1), (1, 5), (4, 1), (3, 3), (5, 8), (9, 4), (7, 11)])
def test_plan_stats_matches_bruteforce_count(lib, shape):
    from two_sided_gptq_b200 import _native

    Mt, Nt = shape
    s = _native.PlanStats()
    assert lib.bakron_plan_stats(Mt * 128, Nt * 128, None, ctypes.byref(s)) == 0
    f1, f2, fs = _brute_schedule_flops(Mt, Nt)
    assert s.tiles_m == Mt and s.tiles_n == Nt and s.tile_diagonals == Mt + Nt - 1
    assert s.leaves == Mt + Nt - 1 and s.nodes == Mt + Nt - 2
    assert s.stage1_flops == pytest.approx(f1, rel=0, abs=0)
    assert s.stage2_flops == pytest.approx(f2, rel=0, abs=0)
    assert s.structural_flops == pytest.approx(fs, rel=0, abs=0)


@pytest.mark.parametrize("shape", [(3, 3), (5, 8), (9, 4), (32, 32)])
def test_plan_stats_two_diagonal_leaves(lib, shape):
    """Leaf structure 7: the width-2 ranges of the recursion become single
    launches whose updates move into the leaf (two T^3 products per
    neighbour); every other node is counted as before."""
    from two_sided_gptq_b200 import _native

    Mt, Nt = shape
    T = 128
    base, pair = _native.PlanStats(), _native.PlanStats()
    cfg = _native.Config(0, 0, 0, 0, None, 0, 7)
    assert lib.bakron_plan_stats(Mt * T, Nt * T, None, ctypes.byref(base)) == 0
    assert lib.bakron_plan_stats(Mt * T, Nt * T, ctypes.byref(cfg), ctypes.byref(pair)) == 0

    def width2_ranges(k, l, out):
        if l <= 1:
            return
        if l == 2:
            out.append(k)
            return
        h = l // 2
        width2_ranges(k, h, out)
        width2_ranges(k + h, l - h, out)

    ks = []
    width2_ranges(0, Mt + Nt - 1, ks)
    assert pair.nodes == base.nodes - len(ks)
    assert pair.leaves == base.leaves - len(ks)
    neighbours = sum((J >= 1) + (I >= 1) for k in ks for I in range(Mt) for J in [k + 1 - I] if 0 <= J < Nt)
    assert pair.leaf_update_flops == 2.0 * T ** 3 * neighbours
    assert pair.update_flops < base.update_flops


def test_plan_stats_4096_cubic_work(lib):
    """O(mn(m+n)) work: the update FLOPs at 4096^2 lie between the
    mn(m+n) pull-form count and twice it, and grow ~8x per size doubling
    (the pages' falsification test: cubic, not m^2 n^2)."""
    from two_sided_gptq_b200 import _native

    def flops(m, n):
        s = _native.PlanStats()
        assert lib.bakron_plan_stats(m, n, None, ctypes.byref(s)) == 0
        return s.update_flops

    f = flops(4096, 4096)
    assert 4096 ** 2 * 8192 < f < 2 * 4096 ** 2 * 8192
    r = flops(8192, 8192) / f
    assert 7.0 < r < 9.0, r


def test_solve_batch_argument_errors_before_device_work(lib):
    """bakron_solve_batch checks every item before it enqueues anything."""
    from two_sided_gptq_b200 import _native

    q = _native.Quantizer(4, 0, 0, None)
    fake = 1 << 20
    st = (ctypes.c_void_p * 1)(None)
    assert lib.bakron_solve_batch(None, 0, ctypes.byref(q), None, st, 1) == _native.Status.OK  # nothing to do
    assert lib.bakron_solve_batch(None, -1, ctypes.byref(q), None, st, 1) == _native.Status.ERR_INVALID_ARG
    items = (_native.BatchItem * 2)()
    good = _native.BatchItem(fake, 8, 8, fake, fake, fake, fake, fake, fake, 1 << 30)
    items[0] = good
    items[1] = _native.BatchItem(fake, 0, 8, fake, fake, fake, fake, fake, fake, 1 << 30)  # m = 0
    assert lib.bakron_solve_batch(items, 2, ctypes.byref(q), None, st, 1) == _native.Status.ERR_INVALID_ARG
    items[1] = _native.BatchItem(fake + 4, 8, 8, fake, fake, fake, fake, fake, fake, 1 << 30)  # misaligned W
    assert lib.bakron_solve_batch(items, 2, ctypes.byref(q), None, st, 1) == _native.Status.ERR_ALIGNMENT
    items[1] = _native.BatchItem(fake, 8, 8, fake, fake, fake, fake, fake, fake, 16)  # short workspace
    assert lib.bakron_solve_batch(items, 2, ctypes.byref(q), None, st, 1) == _native.Status.ERR_WORKSPACE
    assert lib.bakron_solve_batch(items, 2, ctypes.byref(q), None, st, 0) == _native.Status.ERR_INVALID_ARG



@pytest.mark.parametrize("shape", [(1, 1), (300, 260), (4096, 4096), (14336, 4096), (100, 1000)])
def test_plan_stats_one_sided_closed_form(lib, shape):
    """B = I schedule over Nt column blocks: Nt leaves, Nt - 1 nodes, and every
    pair of blocks J < J' costs one 128^3 tile product per row tile, so the
    update FLOPs are 2 T^3 Mt Nt (Nt - 1) / 2 (stage 2 empty)."""
    from two_sided_gptq_b200 import _native

    m, n = shape
    T = 128
    Mt, Nt = -(-m // T), -(-n // T)
    s = _native.PlanStats()
    cfg = _native.Config(0, 0, 0, 0, None, 0, 0, 1)
    assert lib.bakron_plan_stats(m, n, ctypes.byref(cfg), ctypes.byref(s)) == 0
    assert (s.leaves, s.nodes) == (Nt, Nt - 1)
    assert s.stage2_flops == 0
    assert s.update_flops == s.stage1_flops == T ** 3 * Mt * Nt * (Nt - 1)


def _plan_status_under_env(env):
    import subprocess

    code = ("import ctypes, sys; sys.path.insert(0, %r); from two_sided_gptq_b200 import _native; "
            "lib = _native.load(); s = _native.PlanStats(); "
            "print(lib.bakron_plan_stats(256, 256, None, ctypes.byref(s)))") % ROOT
    e = dict(os.environ)
    e.update(env)
    out = subprocess.run([sys.executable, "-c", code], env=e, capture_output=True, text=True, timeout=120)
    assert out.returncode == 0, out.stderr
    return int(out.stdout.strip())


def test_environment_overrides_are_validated():
    """BAKRON_LEAF / _GEMM / _TIMEOUT_MS / _GRAPH / _FUSE change defaults; a malformed
    or out-of-range value makes config-reading calls fail with INVALID_ARG."""
    from two_sided_gptq_b200 import _native

    ok, bad = _native.Status.OK, _native.Status.ERR_INVALID_ARG
    assert _plan_status_under_env({"BAKRON_LEAF": "8", "BAKRON_GEMM": "1", "BAKRON_TIMEOUT_MS": "50",
                                   "BAKRON_GRAPH": "1", "BAKRON_FUSE": "8"}) == ok
    for env in ({"BAKRON_LEAF": "9"}, {"BAKRON_GEMM": "2"}, {"BAKRON_TIMEOUT_MS": "0"},
                {"BAKRON_TIMEOUT_MS": "12ms"}, {"BAKRON_GRAPH": "-1"}, {"BAKRON_FUSE": "0"},
                {"BAKRON_FUSE": "65536"}):
        assert _plan_status_under_env(env) == bad, env


@pytest.mark.parametrize("shape", [(3, 3), (5, 8), (32, 32)])
def test_plan_stats_strip_sweep_leaf_keeps_the_schedule(lib, shape):
    """Leaf structure 8 changes only how a tile diagonal is swept: the
    recursion, its leaves, nodes and update FLOPs are those of the default."""
    from two_sided_gptq_b200 import _native

    Mt, Nt = shape
    base, wave = _native.PlanStats(), _native.PlanStats()
    cfg = _native.Config(0, 0, 0, 0, None, 0, 8)
    assert lib.bakron_plan_stats(Mt * 128, Nt * 128, None, ctypes.byref(base)) == 0
    assert lib.bakron_plan_stats(Mt * 128, Nt * 128, ctypes.byref(cfg), ctypes.byref(wave)) == 0
    for f, _ in _native.PlanStats._fields_:
        assert getattr(wave, f) == getattr(base, f), f
