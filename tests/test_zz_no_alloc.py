"""bakron_solve_noalloc: the solve for callers that may not allocate device
memory when they need it (plug-in execution hooks that must not allocate,
services that fix their memory footprint at start-up).  It runs the same
kernels as bakron_solve with its workspace in a device array the library
declares, so its results must equal bakron_solve's.

Collected last on purpose (file name), so a run that stops at the first
failure has already run every other test; it also passes alone in a fresh
process.
"""
import ctypes

import numpy as np
import pytest

import workloads
from parity import oracle_factors

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def env():
    import torch

    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    import two_sided_gptq_b200 as bk
    from two_sided_gptq_b200 import _native

    return torch, bk, _native, _native.load()


def _noalloc(env, W, LA, LB, bits):
    torch, bk, _native, lib = env
    m, n = W.shape
    V = torch.empty((m, n), dtype=torch.float32, device="cuda")
    codes = torch.empty((m, n), dtype=torch.int8, device="cuda")
    scales = torch.empty((m,), dtype=torch.float32, device="cuda")
    q = _native.Quantizer(bits, 0, 0, None)
    dev_status = ctypes.c_int32(-1)
    stream = ctypes.c_void_p(torch.cuda.current_stream().cuda_stream)
    rc = lib.bakron_solve_noalloc(W.data_ptr(), m, n, LA.data_ptr(), LB.data_ptr(), ctypes.byref(q),
                                  V.data_ptr(), codes.data_ptr(), scales.data_ptr(), None, stream,
                                  ctypes.byref(dev_status))
    return rc, dev_status.value, V, codes, scales


def _problem(env, m, n, seed):
    torch = env[0]
    W, A, B = workloads.random_problem(m, n, seed=seed)
    LA, LB = oracle_factors(A, B)
    return tuple(torch.from_numpy(x).cuda() for x in (W, LA, LB))


def test_noalloc_matches_bakron_solve_on_two_calls_in_a_row(env):
    torch, bk = env[0], env[1]
    # two different problems back to back: the second call reuses the array
    # the first one left behind, so anything not cleared would show up here
    for (m, n, seed, bits) in ((300, 260, 11, 4), (260, 390, 12, 3)):
        W, LA, LB = _problem(env, m, n, seed)
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


def test_noalloc_rejects_problems_beyond_the_array(env):
    torch, bk, _native, lib = env
    limit = 16 << 20
    m = n = 1024  # workspace of about 44 MB > 16 MiB
    assert lib.bakron_solve_workspace_size(m, n, None) > limit
    W = torch.zeros((m, n), device="cuda")
    L = torch.eye(n, device="cuda")
    rc, st, *_ = _noalloc(env, W, L, L, 4)
    assert rc == _native.Status.ERR_WORKSPACE and st == -1
