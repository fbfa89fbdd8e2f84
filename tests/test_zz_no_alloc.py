"""bakron_solve_noalloc: the solve for callers that may not allocate device
memory when they need it (plug-in execution hooks that must not allocate,
services that fix their memory footprint at start-up).  It runs the same
kernels as bakron_solve with its workspace in a device array the library
declares, so its results must equal bakron_solve's, and once its first call
on the device has done the set-up it must take no device memory, even when
the environment asks for the CUDA graph mode (whose capture allocates).

Collected last on purpose (file name), so a run that stops at the first
failure has already run every other test; it also passes alone in a fresh
process.
"""
import ctypes

import numpy as np
import pytest

import workloads
from parity import check_outputs, oracle_factors

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def env():
    import torch

    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    import two_sided_gptq_b200 as bk
    from two_sided_gptq_b200 import _native

    return torch, bk, _native, _native.load()


def _outputs(torch, m, n):
    V = torch.empty((m, n), dtype=torch.float32, device="cuda")
    codes = torch.empty((m, n), dtype=torch.int8, device="cuda")
    scales = torch.empty((m,), dtype=torch.float32, device="cuda")
    return V, codes, scales


def _noalloc_into(env, W, LA, LB, bits, V, codes, scales, status=True):
    torch, bk, _native, lib = env
    m, n = W.shape
    q = _native.Quantizer(bits, 0, 0, None)
    dev_status = ctypes.c_int32(-1)
    stream = ctypes.c_void_p(torch.cuda.current_stream().cuda_stream)
    rc = lib.bakron_solve_noalloc(W.data_ptr(), m, n, LA.data_ptr(), LB.data_ptr(), ctypes.byref(q),
                                  V.data_ptr(), codes.data_ptr(), scales.data_ptr(), None, stream,
                                  ctypes.byref(dev_status) if status else None)
    return rc, dev_status.value


def _noalloc(env, W, LA, LB, bits):
    V, codes, scales = _outputs(env[0], *W.shape)
    rc, st = _noalloc_into(env, W, LA, LB, bits, V, codes, scales)
    return rc, st, V, codes, scales


def _problem(env, m, n, seed):
    torch = env[0]
    W, A, B = workloads.random_problem(m, n, seed=seed)
    LA, LB = oracle_factors(A, B)
    return (W, LA, LB), tuple(torch.from_numpy(x).cuda() for x in (W, LA, LB))


def test_noalloc_matches_bakron_solve_on_two_calls_in_a_row(env):
    torch, bk = env[0], env[1]
    # two different problems back to back: the second call reuses the array
    # the first one left behind, so anything not cleared would show up here
    for (m, n, seed, bits) in ((300, 260, 11, 4), (260, 390, 12, 3)):
        _, (W, LA, LB) = _problem(env, m, n, seed)
        rc, st, V, codes, scales = _noalloc(env, W, LA, LB, bits)
        assert rc == 0 and st == 0, (rc, st)
        V_ref, codes_ref, scales_ref = bk.solve(W, LA, LB, bits=bits)
        torch.cuda.synchronize()
        # identical kernels on identical inputs: the codes and steps agree
        # exactly, V within the parity tolerance of the other tests (1e-4)
        assert torch.equal(codes, codes_ref)
        assert torch.equal(scales, scales_ref)
        rel = float(torch.linalg.norm(V - V_ref) / torch.linalg.norm(V_ref))
        assert rel <= 1e-4


def test_noalloc_takes_no_device_memory_even_in_graph_mode(env, monkeypatch):
    torch = env[0]
    (Wh, LAh, LBh), (W, LA, LB) = _problem(env, 257, 300, 21)
    V, codes, scales = _outputs(torch, *Wh.shape)
    # the first call on the device does the set-up (address look-up, module load)
    rc, st = _noalloc_into(env, W, LA, LB, 4, V, codes, scales)
    assert rc == 0 and st == 0, (rc, st)
    torch.cuda.synchronize()
    # BAKRON_GRAPH=1 would send bakron_solve through graph capture, which
    # allocates; this entry point must launch directly all the same
    monkeypatch.setenv("BAKRON_GRAPH", "1")
    free_before = torch.cuda.mem_get_info()[0]
    for _ in range(2):
        rc, st = _noalloc_into(env, W, LA, LB, 4, V, codes, scales)
        assert rc == 0 and st == 0, (rc, st)
    torch.cuda.synchronize()
    assert torch.cuda.mem_get_info()[0] == free_before
    # and the result is the solve's: teacher-forced against the oracle
    check_outputs(Wh, LAh, LBh, 4, V.cpu().numpy(), codes.cpu().numpy(), scales.cpu().numpy(),
                  label="noalloc, BAKRON_GRAPH=1")


def test_noalloc_refuses_a_status_read_inside_stream_capture(env):
    torch, bk, _native, lib = env
    _, (W, LA, LB) = _problem(env, 64, 96, 31)
    V, codes, scales = _outputs(torch, 64, 96)
    rc, _ = _noalloc_into(env, W, LA, LB, 4, V, codes, scales)  # set-up outside the capture
    assert rc == 0
    torch.cuda.synchronize()
    s = torch.cuda.Stream()
    g = torch.cuda.CUDAGraph()
    with torch.cuda.stream(s):
        g.capture_begin()
        try:
            rc, st = _noalloc_into(env, W, LA, LB, 4, V, codes, scales, status=True)
        finally:
            g.capture_end()
    assert rc == _native.Status.ERR_INVALID_ARG and st == -1


def test_noalloc_rejects_problems_beyond_the_array(env):
    torch, bk, _native, lib = env
    limit = 16 << 20
    m = n = 1024  # workspace of about 44 MB > 16 MiB
    assert lib.bakron_solve_workspace_size(m, n, None) > limit
    W = torch.zeros((m, n), device="cuda")
    L = torch.eye(n, device="cuda")
    rc, st, *_ = _noalloc(env, W, L, L, 4)
    assert rc == _native.Status.ERR_WORKSPACE and st == -1
