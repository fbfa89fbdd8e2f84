"""CUDA graph mode (cfg.use_graph): the captured-and-replayed solve gives the
same bits as direct launches, and a replay reads the buffers' current
contents."""
import numpy as np
import pytest

import workloads
from parity import oracle_factors

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def _cuda():
    import torch

    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    import two_sided_gptq_b200 as bk

    bk._lib()


@pytest.mark.parametrize("one_sided", [False, True])
@pytest.mark.parametrize("shape", [(300, 260), (129, 1000)])
def test_graph_replay_equals_direct(shape, one_sided):
    import torch

    import two_sided_gptq_b200 as bk

    m, n = shape
    W, A, B = workloads.random_problem(m, n, seed=m + 7 * n)
    LA, LB = oracle_factors(A, B)
    Wd, LAd = torch.from_numpy(W).cuda(), torch.from_numpy(LA).cuda()
    LBd = None if one_sided else torch.from_numpy(LB).cuda()
    ws = bk.workspace(bk.solve_workspace_size(m, n))
    out = (torch.empty((m, n), dtype=torch.float32, device="cuda"),
           torch.empty((m, n), dtype=torch.int8, device="cuda"), torch.empty((m,), dtype=torch.float32, device="cuda"))
    for trial in range(3):
        if trial == 2:  # new contents in the same buffer: the replay must see them
            Wd.copy_(torch.from_numpy(workloads.random_problem(m, n, seed=99)[0]))
        V0, c0, s0 = (t.clone() for t in bk.solve(Wd, LAd, LBd, bits=4))
        V1, c1, s1 = bk.solve(Wd, LAd, LBd, bits=4, ws=ws, out=out, graph=True)
        assert torch.equal(c1, c0) and torch.equal(V1, V0) and torch.equal(s1, s0), trial
