"""Failure detection on the GPU without a fault: a device wait that nothing
completes gives up at its deadline, records BAKRON_ERR_DEVICE_TIMEOUT in the
status word, and leaves the context usable for the next solve."""
import numpy as np
import pytest

import workloads
from parity import check_solve, oracle_factors

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def _cuda():
    import torch

    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    import two_sided_gptq_b200 as bk

    bk._lib()


def test_bounded_wait_gives_up_and_context_stays_usable():
    import torch

    import two_sided_gptq_b200 as bk

    ws = bk.workspace(256)
    for timeout_ms in (5, 40):
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        e0.record()
        bk.selftest_wait_timeout(timeout_ms, ws)
        e1.record()
        assert bk.get_status(ws) == bk.Status.ERR_DEVICE_TIMEOUT
        ms = e0.elapsed_time(e1)
        assert timeout_ms * 0.9 <= ms < timeout_ms + 500, (timeout_ms, ms)
        assert bk.get_status(ws) == bk.Status.OK  # reading clears it
    # the context is intact: a solve right after runs and matches the oracle
    W, A, B = workloads.random_problem(129, 257, seed=3)
    LA, LB = oracle_factors(A, B)
    check_solve(W, LA, LB, 4, label="after timeout")


def test_band_kernel_abort_path_records_timeout_and_context_stays_usable():
    """The band-product kernel itself (tcgen05 MMAs, TMEM, TMA pipeline) with
    its copy-issuing thread told to issue nothing: the MMA issuer's and the
    epilogue's bounded waits run out with nothing in flight; the kernel records
    the timeout with the waiting role, frees its tensor memory and exits."""
    import torch

    import two_sided_gptq_b200 as bk

    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record()
    ws = bk.selftest_band_abort(5)
    e1.record()
    torch.cuda.synchronize()
    code, where = (int(x) for x in ws[:8].view(torch.int32).cpu())
    assert code == int(bk.Status.ERR_DEVICE_TIMEOUT)
    assert where in (2001, 3001), where  # the MMA issuer or the epilogue gave up
    assert bk.get_status(ws) == bk.Status.ERR_DEVICE_TIMEOUT
    assert bk.get_status(ws) == bk.Status.OK
    assert 4.5 <= e0.elapsed_time(e1) < 500
    # tensor memory was released and the context is intact: a full solve with
    # tensor-core band products right after matches the oracle
    W, A, B = workloads.random_problem(300, 390, seed=5)
    LA, LB = oracle_factors(A, B)
    check_solve(W, LA, LB, 4, label="after band abort")


def test_two_diagonal_leaf_waits_run_out_when_a_flag_never_comes():
    """Leaf structure 7 with one first-diagonal tile told never to raise its
    flag (a host-made failure: no kernel faults or hangs): its neighbours on
    the second diagonal give up after the deadline, the solve completes and
    reports BAKRON_ERR_DEVICE_TIMEOUT with the waiting CTA (4000 + its row
    block); a normal solve right after matches the oracle."""
    import torch

    import two_sided_gptq_b200 as bk

    # 3 x 4 tiles, tile diagonals 0..5; the recursion's width-2 ranges are
    # (1, 2) and (4, 5), so tile (0, 1) (row-major index 1) on diagonal 1 is a
    # producer whose neighbours (0, 2) and (1, 1) on diagonal 2 wait for it
    m, n = 384, 512
    W, A, B = workloads.random_problem(m, n, seed=17)
    LA, LB = oracle_factors(A, B)
    Wd, LAd, LBd = (torch.from_numpy(x).cuda() for x in (W, LA, LB))
    ws = bk.workspace(bk.solve_workspace_size(m, n))
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record()
    bk.solve(Wd, LAd, LBd, bits=4, ws=ws, leaf=7, timeout_ms=5, self_test_omit=0 * 4 + 1 + 1, check_status=False)
    e1.record()
    torch.cuda.synchronize()
    code, where = (int(x) for x in ws[:8].view(torch.int32).cpu())
    assert code == int(bk.Status.ERR_DEVICE_TIMEOUT)
    assert 4000 <= where < 4004, where
    assert bk.get_status(ws) == bk.Status.ERR_DEVICE_TIMEOUT
    assert e0.elapsed_time(e1) < 2000
    check_solve(W, LA, LB, 4, leaf=7, label="after a flag that never came")
