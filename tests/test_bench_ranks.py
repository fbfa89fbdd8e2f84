"""bench.py's multi-rank host logic (replicas: one matrix per rank, no
data-path collective) on two CPU processes over gloo: the timing reduction is
the max over ranks, the whole-job rate counts every rank's matrix, rank 0
generates the shared inputs before the others read them, and the reference
arm runs on rank 0 only."""
import contextlib
import io
import multiprocessing as mp
import os
import socket
import sys
import time

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _rank_main(rank, world, port, cache, q):
    try:
        os.environ.update({"RANK": str(rank), "LOCAL_RANK": str(rank), "WORLD_SIZE": str(world),
                           "MASTER_ADDR": "127.0.0.1", "MASTER_PORT": str(port),
                           "BAKRON_WORKLOAD_CACHE": cache})
        sys.path.insert(0, ROOT)
        import hashlib

        import bench

        r, ws, local, dist = bench.dist_setup("gloo", timeout_s=60)
        out = {"rank": r, "world": ws, "local": local}
        # max over ranks of a per-rank figure
        out["max"] = bench.max_over_ranks(1.5 + r, dist)
        # a timed region bracketed by barriers: each rank sleeps its own time,
        # the reported time is the slowest rank's
        dist.barrier()
        t0 = time.perf_counter()
        time.sleep(0.05 + 0.15 * r)
        dt = time.perf_counter() - t0
        dist.barrier()
        out["own_dt"] = dt
        out["job_dt"] = bench.max_over_ranks(dt, dist)
        # inputs: rank 0 generates (and caches) first, the others read after
        W, A, B = bench.load_inputs("tiny", r, dist)
        out["digest"] = hashlib.sha256(W.tobytes() + A.tobytes() + B.tobytes()).hexdigest()
        # the reference arm prints on rank 0 only; other ranks do no work
        if r != 0:
            args = type("Args", (), {"steps": 1, "warmup": 3, "gpus": ws, "workload": "tiny"})()
            buf = io.StringIO()
            with contextlib.redirect_stdout(buf):
                rc = bench.run_reference(args)
            out["ref_rc"], out["ref_out"] = rc, buf.getvalue()
        dist.barrier()
        dist.destroy_process_group()
        q.put(out)
    except Exception as e:  # reported to the parent
        q.put({"rank": rank, "error": repr(e)})


def test_two_gloo_ranks(tmp_path):
    world = 2
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_rank_main, args=(r, world, port, str(tmp_path), q)) for r in range(world)]
    for p in procs:
        p.start()
    res = {}
    try:
        for _ in range(world):
            o = q.get(timeout=240)
            res[o["rank"]] = o
    finally:
        for p in procs:
            p.join(timeout=60)
            if p.is_alive():
                p.kill()
    for r in range(world):
        assert "error" not in res[r], res[r]
        assert res[r]["world"] == world and res[r]["local"] == r
        assert res[r]["max"] == pytest.approx(1.5 + world - 1)
        # every rank reports the same job time, at least the slowest rank's own
        assert res[r]["job_dt"] == max(res[k]["own_dt"] for k in range(world))
        assert res[r]["job_dt"] >= 0.05 + 0.15 * (world - 1)
    assert res[0]["digest"] == res[1]["digest"]
    assert res[1]["ref_rc"] == 0 and res[1]["ref_out"] == ""


def test_aggregate_rate_counts_every_rank():
    sys.path.insert(0, ROOT)
    import bench

    one = bench.aggregate_rate(1, 4096, 4096, 10.0)
    assert one == pytest.approx(4096 * 4096 / 0.010)
    assert bench.aggregate_rate(8, 4096, 4096, 10.0) == pytest.approx(8 * one)
    assert bench.max_over_ranks(3.25, None) == 3.25


def test_working_set_matches_the_library_layout():
    """bench.py's working-set note uses the same workspace size as the library
    (bakron_solve_workspace_size, a host-only query) and says whether a step's
    data exceeds the L2."""
    sys.path.insert(0, ROOT)
    import bench
    import workloads

    import two_sided_gptq_b200 as bk

    lib = bk._lib()
    for m, n in ((4096, 4096), (64, 128), (14336, 4096), (300, 260)):
        ws = bench.working_set_bytes(m, n)[2]
        assert abs(ws - lib.bakron_solve_workspace_size(m, n, None)) <= 4096, (m, n)
    args = type("Args", (), {"gpus": 1})()
    assert "exceeds" in bench.config_block(workloads.WORKLOADS["bench"], args)["l2"]
    assert "fits" in bench.config_block(workloads.WORKLOADS["tiny"], args)["l2"]
