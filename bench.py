#!/usr/bin/env python
"""Throughput of the BaKron two-sided adaptive-rounding solve on B200.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl ours|reference]

A step is one full solve (grid steps and normalised factors, every leaf sweep,
every band product of the tile-diagonal recursion) of the 4096 x 4096 INT4
workload with inputs resident in HBM; the Cholesky factors are computed once
before timing (their time is reported separately as ``factor_ms``).  With N > 1
(launched by torchrun) every rank solves its own matrix: replicas of an
independent per-matrix problem, weak scaling, no data-path collective.

``--impl reference`` times the FP64 CPU oracle (the anti-diagonal pull solver)
on the host cores instead, each step a bounded sample of the same workload.
"""
from __future__ import annotations

import argparse
import json
import os
import statistics
import subprocess
import sys
import tempfile
import time

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

METRIC = "quantized weights/sec for 4096×4096 INT4 BaKron solve; % tensor-pipe roofline"
TF32_PER_BF16 = 1.1 / 2.25  # nominal dense TF32 : BF16 tensor peak ratio
FALLBACK_BF16_TFLOPS = 1590.0
LEAF_BYTES_PER_WEIGHT = 25  # read Wt 4 + diagonal factor blocks 8; write code 1, V 4, D hi/lo 8
LEAF_KERNELS = {1: ("leaf_nested_kernel", 3 * 127), 2: ("leaf_single_kernel", 255), 3: ("leaf_warp_kernel", 7 * 63),
                4: ("leaf_wide_kernel", 3 * 127), 5: ("leaf_cluster_kernel<false, false>", 7 * 63),
                6: ("leaf_cluster_kernel<true, false>", 7 * 63), 7: ("leaf_cluster_kernel<true, true>", 7 * 63),
                8: ("leaf_wave_kernel", 3 * 48 + 159)}
# DRAM traffic of the band products from an ncu capture of one solve's 93
# band launches (profiles/band_4096_dram.md); reported only while the band
# kernel sources hash to the value the capture was taken with.
BAND_TRAFFIC = {"sources_sha256": "ef9d3f34d5ea8c96364dcc2839be8f96ecc32f72ca91e2e1a88046a0f5183436",
                "bytes_per_launch": 36.80e6, "profile": "profiles/band_4096_dram.md"}
BAND_SOURCES = ("two_sided_gptq_b200/csrc/band_tc.cu", "two_sided_gptq_b200/csrc/band_fused.cu",
                "two_sided_gptq_b200/csrc/tcgen05.cuh", "two_sided_gptq_b200/csrc/common.cuh",
                "two_sided_gptq_b200/csrc/kernels.cuh")


def band_sources_sha256():
    import hashlib

    h = hashlib.sha256()
    for f in BAND_SOURCES:
        h.update(open(os.path.join(ROOT, f), "rb").read())
    return h.hexdigest()


def peaks():
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(p):
        d = json.load(open(p))
        return d.get("bf16_tflops", FALLBACK_BF16_TFLOPS), d.get("hbm_gbs", 6650.0), "measured"
    return FALLBACK_BF16_TFLOPS, 6650.0, "fallback"


class ClockSampler:
    """nvidia-smi samples of SM clock and throttle reasons during the timed region."""

    FIELDS = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, gpu_index: int):
        self.gpu = gpu_index
        self.proc = None
        self.path = None

    def __enter__(self):
        fd, self.path = tempfile.mkstemp(suffix=".csv")
        os.close(fd)
        try:
            self.proc = subprocess.Popen(["nvidia-smi", "-i", str(self.gpu), f"--query-gpu={self.FIELDS}",
                                          "--format=csv,noheader,nounits", "-lms", "200"],
                                         stdout=open(self.path, "w"), stderr=subprocess.DEVNULL)
        except OSError:
            self.proc = None
        time.sleep(0.3)
        return self

    def __exit__(self, *a):
        if self.proc is not None:
            time.sleep(0.25)
            self.proc.terminate()
            try:
                self.proc.wait(timeout=5)
            except subprocess.TimeoutExpired:
                self.proc.kill()

    def summary(self):
        rows = []
        if self.path and os.path.exists(self.path):
            for line in open(self.path):
                parts = [x.strip() for x in line.split(",")]
                if len(parts) >= 9:
                    rows.append(parts)
            os.unlink(self.path)
        if not rows:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["nvidia-smi unavailable"], "samples": 0}
        sm = [float(r[1]) for r in rows if r[1].replace(".", "").isdigit()]
        mx = [float(r[2]) for r in rows if r[2].replace(".", "").isdigit()]
        pw = [float(r[3]) for r in rows if r[3].replace(".", "").isdigit()]
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        reasons = sorted({names[k] for r in rows for k in range(4) if r[5 + k].lower() == "active"})
        # median over samples taken under load (power above the idle floor)
        load = [s for s, p in zip(sm, pw) if p > 250] or sm
        return {"sm_mhz": statistics.median(load) if load else None, "sm_max_mhz": max(mx) if mx else None,
                "reasons": reasons, "samples": len(rows), "power_w_max": max(pw) if pw else None}


def dist_setup(backend="nccl", timeout_s=300):
    """One process per GPU (torchrun env): returns rank, world size, local rank
    and the torch.distributed module (None when running alone).  The only
    collectives are the timing barriers and the max-over-ranks reductions:
    each rank solves its own matrix."""
    ws = int(os.environ.get("WORLD_SIZE", "1"))
    if ws <= 1:
        return 0, 1, 0, None
    import datetime

    import torch
    import torch.distributed as dist

    rank, local = int(os.environ["RANK"]), int(os.environ.get("LOCAL_RANK", "0"))
    kw = {}
    if backend == "nccl":
        torch.cuda.set_device(local)
        kw["device_id"] = torch.device("cuda", local)
    dist.init_process_group(backend, timeout=datetime.timedelta(seconds=timeout_s), **kw)
    return rank, ws, local, dist


def max_over_ranks(x, dist, device="cpu"):
    """Max of a per-rank float over all ranks (identity when running alone)."""
    if dist is None:
        return float(x)
    import torch

    t = torch.tensor([float(x)], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def aggregate_rate(world, m, n, ms_per_step):
    """Whole-job weights/s: every rank solves one m x n matrix per step."""
    return world * m * n / (ms_per_step / 1e3)


def load_inputs(name, rank, dist):
    import workloads

    os.environ.setdefault("BAKRON_WORKLOAD_CACHE", os.path.join(tempfile.gettempdir(), "bakron_workloads"))
    if dist is not None and rank != 0:
        dist.barrier()
    W, A, B = workloads.generate(name)
    if dist is not None and rank == 0:
        dist.barrier()
    return W, A, B


FP64_PEAK_NOMINAL = 37.0  # TFLOP/s, nominal B200 FP64


def factor_flops(d):
    """Flops of chol(M^-1) for a d x d factor as the path computes it: the
    Cholesky factorisation (d^3 / 6 multiply-adds) and the triangular inverse
    (d^3 / 6 multiply-adds), two flops per multiply-add."""
    return 2 * (d ** 3 / 6 + d ** 3 / 6)


def oracle_factors(A, B):
    """The oracle's normalised FP64 factors (computed once per run)."""
    import oracle

    return oracle.normalize(oracle.factor(A)), oracle.normalize(oracle.factor(B))


def cpu_baseline(W, A, B, bits, target_s=15.0, single_thread=False, factors=None, rows=None):
    """Oracle (FP64 anti-diagonal pull, OpenMP over each diagonal) timed on a
    bounded sample: the top r rows, a closed sub-problem (rows < r never depend
    on later rows), with r chosen for about ``target_s`` of work (or given as
    ``rows``; r = m is the whole matrix and needs no scaling); a partial time
    is scaled to the full matrix by the ratio of multiply-adds
    r n (r+n) : m n (m+n)."""
    import numpy as np

    import oracle

    m, n = W.shape
    qmin, qmax = oracle.grid(bits)
    s = oracle.scales(W, qmax)
    LtA, LtB = factors if factors is not None else oracle_factors(A, B)
    threads = oracle.num_threads()

    def run(r):
        t0 = time.perf_counter()
        oracle.solve(W[:r], LtA, np.ascontiguousarray(LtB[:r, :r]), s[:r], qmin, qmax, mode="pull", nthreads=threads)
        return time.perf_counter() - t0

    work = lambda r: r * n * (r + n)
    if rows is not None:
        r = min(m, rows)
        t = run(r)
    else:
        r0 = min(m, 128)
        t0 = run(r0)
        r = r0
        while r < m and t0 * work(min(m, 2 * r)) / work(r0) <= target_s:
            r = min(m, 2 * r)
        t = run(r) if r != r0 else t0
    t_full = t * work(m) / work(r)
    sample = (f"the whole {m}x{n} workload, {t:.2f} s measured" if r == m else
              f"top {r} of {m} rows of the {m}x{n} workload (closed sub-problem), {t:.2f} s measured, "
              f"scaled x{work(m) / work(r):.2f} by multiply-add count to the whole matrix")
    out = {"value": m * n / t_full, "unit": "weights/s", "cores": threads, "kind": "oracle",
           "sample": sample, "sample_seconds": t, "nproc": os.cpu_count()}
    if single_thread and threads > 1:
        r1 = min(m, 64)
        t1 = time.perf_counter()
        oracle.solve(W[:r1], LtA, np.ascontiguousarray(LtB[:r1, :r1]), s[:r1], qmin, qmax, mode="pull", nthreads=1)
        t1 = time.perf_counter() - t1
        out["single_thread_value"] = m * n / (t1 * work(m) / work(r1))
        out["single_thread_sample"] = f"top {r1} rows, 1 thread, {t1:.2f} s measured, scaled by multiply-add count"
    return out


def band_levels(launches):
    """Band-product time and tensor-pipe fraction per recursion level (node
    width l in tile diagonals; separate or fused stage launches), medians over
    the profiled steps.  FLOPs are the structurally non-zero ones."""
    by = {}
    for step in launches:
        acc = {}
        for r in step:
            if r["kind"] in ("stage1", "stage2", "fused"):
                a = acc.setdefault(r["l"], [0.0, 0.0, 0])
                a[0] += r["ms"]
                a[1] += r["structural_flops"]
                a[2] += 1
        for l, a in acc.items():
            by.setdefault(l, []).append(a)
    bf16, _, _ = peaks()
    peak = bf16 * TF32_PER_BF16
    out = []
    for l in sorted(by, reverse=True):
        ms = statistics.median(a[0] for a in by[l])
        fl = by[l][0][1]
        tf = 3.0 * fl / (ms / 1e3) / 1e12 if ms > 0 else 0.0
        out.append({"l": l, "launches": by[l][0][2], "ms": ms, "flops": fl, "tflops": tf, "frac": tf / peak})
    return out


def run_reference(args):
    """--impl reference: the oracle on the host cores, same metric and config."""
    rank = int(os.environ.get("RANK", "0"))
    if rank != 0:
        return 0
    import workloads

    w = workloads.WORKLOADS[args.workload]
    os.environ.setdefault("BAKRON_WORKLOAD_CACHE", os.path.join(tempfile.gettempdir(), "bakron_workloads"))
    W, A, B = workloads.generate(args.workload)
    factors = oracle_factors(A, B)
    # Every step solves the whole matrix when (steps + warm-up) such solves fit
    # the budget (the run must end within a few minutes); otherwise each step
    # takes the largest top-rows sub-problem that does, scaled (stated in the
    # line's sample).
    budget_s = 200.0
    probe = cpu_baseline(W, A, B, w.bits, factors=factors, rows=min(w.m, 256))
    full_s = w.m * w.n / probe["value"]
    rows = None
    if full_s * (args.steps + args.warmup) <= budget_s:
        rows = w.m
    else:
        per_step = budget_s / (args.steps + args.warmup)
        rows = min(w.m, 256)
        while rows < w.m and full_s * (2 * rows) * w.n * (2 * rows + w.n) / (w.m * w.n * (w.m + w.n)) <= per_step:
            rows = min(w.m, 2 * rows)
    for _ in range(args.warmup):
        cpu_baseline(W, A, B, w.bits, factors=factors, rows=rows)
    vals = [cpu_baseline(W, A, B, w.bits, factors=factors, rows=rows) for _ in range(args.steps)]
    v = statistics.median(x["value"] for x in vals)
    ms = w.m * w.n / v * 1e3
    cb = dict(vals[-1])
    cb["value"] = v
    line = {"impl": "reference", "metric": METRIC, "value": v, "unit": "weights/s", "n_gpus": args.gpus,
            "steps": args.steps, "warmup": args.warmup, "ms_per_step": ms, "higher_is_better": True,
            "scaling": "weak", "vs_baseline": None, "dtype": "f64", "data": "synthetic",
            "config": config_block(w, args), "cpu_baseline": cb,
            "e2e": {"value": v, "unit": "weights/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}}
    print(json.dumps(line), flush=True)
    return 0


L2_BYTES = 126e6


def working_set_bytes(m, n, T=128):
    """Inputs (W, LA, LB), outputs (V, codes, steps) and the solve workspace
    (Wt, Delta hi/lo, X^T hi/lo and the exported in-tile R on the padded grid;
    both normalised factors with their hi/lo parts; per-tile flags) touched by
    one solve."""
    Mp, Np = -(-m // T) * T, -(-n // T) * T
    inputs = 4 * (m * n + n * n + m * m)
    outputs = 4 * m * n + m * n + 4 * m
    workspace = 4 * (6 * Mp * Np + 3 * Np * Np + 3 * Mp * Mp) + 4 * ((Mp // T) * (Np // T) + (Mp + Np) // T)
    return inputs, outputs, workspace


def config_block(w, args):
    inputs, outputs, workspace = working_set_bytes(w.m, w.n)
    total = inputs + outputs + workspace
    l2 = (f"no flush: the per-step working set (inputs {inputs / 1e6:.0f} MB + outputs {outputs / 1e6:.0f} MB + "
          f"workspace {workspace / 1e6:.0f} MB) exceeds the 126 MB L2" if total > L2_BYTES else
          f"no flush: the per-step working set ({total / 1e6:.1f} MB) fits in the 126 MB L2, so steps run L2-warm")
    return {"workload": f"{w.name}: W {w.m}x{w.n} fp32 N(0,{w.w_std}^2), INT{w.bits} symmetric per-row grid, "
                        f"A,B {w.a_recipe}/{w.b_recipe} Gram factors, {w.damping:.1%} damping",
            "m": w.m, "n": w.n, "bits": w.bits, "tile": 128, "band_products": "tcgen05 3xTF32",
            "parallelism": f"replicas x{args.gpus}", "l2": l2}


def extra_measurements(args, bk, w, Wd, LA, LB, W, codes, ws, stream, dev, dist, leaf, fw, n_batch):
    """End to end through the host-buffer entry point, several matrices at
    once, and the one-sided path: (e2e ms, batch ms, one-sided ms) per step."""
    import numpy as np
    import torch

    m, n = W.shape
    # e2e through the host-buffer entry point: H2D of W, LA, LB and D2H of V,
    # codes, scales inside the timed region, every step
    Wh = torch.from_numpy(W).pin_memory()
    LAh, LBh = LA.cpu().pin_memory(), LB.cpu().pin_memory()
    Vh = torch.empty((m, n), dtype=torch.float32).pin_memory()
    ch = torch.empty((m, n), dtype=torch.int8).pin_memory()
    sh = torch.empty((m,), dtype=torch.float32).pin_memory()
    wsh = bk.workspace(bk.solve_host_workspace_size(m, n), dev)
    for _ in range(2):
        bk.solve_host(Wh, LAh, LBh, bits=w.bits, V=Vh, codes=ch, scales=sh, ws=wsh, stream=stream, leaf=leaf,
                      fuse_width=fw)
    torch.cuda.synchronize()
    h0, h1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e2e_steps = max(3, args.steps // 2)
    h0.record(stream)
    for _ in range(e2e_steps):
        bk.solve_host(Wh, LAh, LBh, bits=w.bits, V=Vh, codes=ch, scales=sh, ws=wsh, stream=stream, synchronize=False,
                      leaf=leaf, fuse_width=fw)
    h1.record(stream)
    torch.cuda.synchronize()
    e2e_ms = max_over_ranks(h0.elapsed_time(h1) / e2e_steps, dist, dev)
    assert np.array_equal(ch.numpy(), codes.cpu().numpy()), "host-buffer solve disagrees with device solve"

    # several matrices at once (bakron_solve_batch on separate streams): one
    # solve keeps few SMs busy during its leaf sweeps, so solves overlap
    n_batch = 4
    bstreams = [torch.cuda.Stream(device=dev) for _ in range(n_batch)]
    bouts = [(torch.empty((m, n), dtype=torch.float32, device=dev), torch.empty((m, n), dtype=torch.int8, device=dev),
              torch.empty((m,), dtype=torch.float32, device=dev)) for _ in range(n_batch)]
    bws = [bk.workspace(bk.solve_workspace_size(m, n), dev) for _ in range(n_batch)]
    probs = [(Wd, LA, LB)] * n_batch

    def batch_step():
        start = torch.cuda.Event()
        start.record(stream)
        for bs in bstreams:
            bs.wait_event(start)
        bk.solve_batch(probs, bits=w.bits, streams=bstreams, outs=bouts, workspaces=bws, leaf=leaf,
                       check_status=False, fuse_width=fw)
        for bs in bstreams:
            done = torch.cuda.Event()
            done.record(bs)
            stream.wait_event(done)

    for _ in range(2):
        batch_step()
    torch.cuda.synchronize()
    b0, b1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    b_steps = 3
    b0.record(stream)
    for _ in range(b_steps):
        batch_step()
    b1.record(stream)
    torch.cuda.synchronize()
    batch_ms = max_over_ranks(b0.elapsed_time(b1) / b_steps, dist, dev)
    assert torch.equal(bouts[-1][1], codes), "batched solve disagrees with the single solve"
    del bws, bouts

    # the one-sided path (B = I: GPTQ with Hessian A) on the same W and A
    o_out = (torch.empty_like(Wd), torch.empty((m, n), dtype=torch.int8, device=dev),
             torch.empty((m,), dtype=torch.float32, device=dev))
    for _ in range(2):
        bk.solve(Wd, LA, None, bits=w.bits, ws=ws, out=o_out, stream=stream)
    torch.cuda.synchronize()
    o0, o1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    o_steps = 5
    o0.record(stream)
    for _ in range(o_steps):
        bk.solve(Wd, LA, None, bits=w.bits, ws=ws, out=o_out, stream=stream, check_status=False)
    o1.record(stream)
    torch.cuda.synchronize()
    one_ms = max_over_ranks(o0.elapsed_time(o1) / o_steps, dist, dev)
    del o_out

    return e2e_ms, batch_ms, one_ms


def proxy_loss_timing(bk, Wd, V, Ad, Bd, stream, dist, dev):
    """bakron_proxy_loss of the solve's V (its result is copied to the host,
    so each call ends synchronised): value and ms per call (CUDA events on the
    stream, median of five after one warm-up), max over ranks."""
    import torch

    m, n = Wd.shape
    value = bk.proxy_loss(Wd, V, Ad, Bd, stream=stream)
    times = []
    for _ in range(5):
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        e0.record(stream)
        bk.proxy_loss(Wd, V, Ad, Bd, stream=stream)
        e1.record(stream)
        torch.cuda.synchronize()
        times.append(e0.elapsed_time(e1))
    ms = max_over_ranks(statistics.median(times), dist, dev)
    flops = 2.0 * m * n * (m + n)
    return {"value": value, "ms": ms, "flops": flops, "tflops": flops / (ms / 1e3) / 1e12,
            "note": "tr((W-V)^T B (W-V) A): the products B(W-V) and (W-V)A on the tcgen05 tensor cores in "
                    "3xTF32, the elementwise dot in FP64 with a fixed order; outside the metric"}


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=10)
    ap.add_argument("--warmup", type=int, default=3)
    ap.add_argument("--impl", default="ours", choices=["ours", "reference"])
    ap.add_argument("--workload", default="bench")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--profile-steps", type=int, default=3)
    ap.add_argument("--leaf", type=int, default=0,
                    help="leaf structure (bakron_config_t.leaf); 0 picks it by measurement (bakron_tune_leaf)")
    ap.add_argument("--fuse-width", type=int, default=0, help="bakron_config_t.fuse_width (0 = library default)")
    ap.add_argument("--no-extras", action="store_true",
                    help="profiling runs: skip the host-buffer, batched and one-sided measurements")
    args = ap.parse_args()
    if args.warmup < 3:
        args.warmup = 3
    if args.impl == "reference":
        return run_reference(args)

    import numpy as np
    import torch

    import two_sided_gptq_b200 as bk
    import workloads

    rank, world, local, dist = dist_setup("nccl")
    w = workloads.WORKLOADS[args.workload]
    W, A, B = load_inputs(args.workload, rank, dist)
    dev = torch.device("cuda", local)
    torch.cuda.set_device(dev)
    m, n = W.shape
    Wd, Ad, Bd = (torch.from_numpy(x).to(dev) for x in (W, A, B))

    # factor (a0): timed separately
    LA, LB = bk.factor(Ad, Bd)
    torch.cuda.synchronize()
    fe0, fe1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    fe0.record()
    LA, LB = bk.factor(Ad, Bd, check_status=False)
    fe1.record()
    torch.cuda.synchronize()
    factor_ms = fe0.elapsed_time(fe1)

    ws = bk.workspace(bk.solve_workspace_size(m, n), dev)
    V = torch.empty((m, n), dtype=torch.float32, device=dev)
    codes = torch.empty((m, n), dtype=torch.int8, device=dev)
    scales = torch.empty((m,), dtype=torch.float32, device=dev)
    out = (V, codes, scales)
    stream = torch.cuda.current_stream()

    # the schedule's leaf structure, picked by measurement on this problem
    fw = args.fuse_width
    if args.leaf > 0:
        leaf, leaf_tune_ms = args.leaf, None
    else:
        leaf, leaf_tune_ms = bk.tune_leaf(Wd, LA, LB, bits=w.bits, ws=ws, out=out, stream=stream)

    def step():
        bk.solve(Wd, LA, LB, bits=w.bits, ws=ws, out=out, check_status=False, stream=stream, leaf=leaf,
                 fuse_width=fw)

    for _ in range(args.warmup):
        step()
    torch.cuda.synchronize()
    if bk.get_status(ws) != bk.Status.OK:
        raise RuntimeError("device status not OK after warm-up")

    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    with ClockSampler(local) as clk:
        if dist is not None:
            dist.barrier()
        torch.cuda.synchronize()
        e0.record(stream)
        for _ in range(args.steps):
            step()
        e1.record(stream)
        torch.cuda.synchronize()
        if dist is not None:
            dist.barrier()
    elapsed = max_over_ranks(e0.elapsed_time(e1), dist, dev)
    status = bk.get_status(ws)
    ms_per_step = elapsed / args.steps
    value = aggregate_rate(world, m, n, ms_per_step)

    # per-kernel-class device times (separate profiled steps, events on the launch stream)
    prof, launches = [], []
    for _ in range(max(1, args.profile_steps)):
        bk.solve(Wd, LA, LB, bits=w.bits, ws=ws, out=out, check_status=False, stream=stream, profile=True,
                 leaf=leaf, fuse_width=fw)
        prof.append(bk.last_profile())
        launches.append(bk.last_profile_launches())
    pr = {k: statistics.median(p[k] for p in prof) for k in prof[0]}
    levels = band_levels(launches)
    plan = bk.plan_stats(m, n, leaf=leaf)
    bf16, hbm, src = peaks()
    tf32_peak = bf16 * TF32_PER_BF16
    gemm_ms = pr["stage1_ms"] + pr["stage2_ms"] + pr["fused_ms"]
    # a one-tile-diagonal problem (m, n <= 128) has no band products
    achieved = 3.0 * plan["structural_flops"] / (gemm_ms / 1e3) / 1e12 if gemm_ms > 0 else 0.0
    leaf_bytes = LEAF_BYTES_PER_WEIGHT * m * n
    launches_per_step = int(pr["prep_launches"] + pr["leaf_launches"] + pr["stage1_launches"] +
                            pr["stage2_launches"] + pr["fused_launches"])

    e2e_ms = batch_ms = one_ms = None
    n_batch = 4
    if not args.no_extras:
        e2e_ms, batch_ms, one_ms = extra_measurements(args, bk, w, Wd, LA, LB, W, codes, ws, stream, dev, dist,
                                                      leaf, fw, n_batch)
    loss = proxy_loss_timing(bk, Wd, V, Ad, Bd, stream, dist, dev)

    line = None
    if rank == 0:
        cb = None
        if world == 1 and not args.no_cpu_baseline:
            cb = cpu_baseline(W, A, B, w.bits, single_thread=True)
        line = {
            "metric": METRIC, "value": value, "unit": "weights/s", "n_gpus": world, "steps": args.steps,
            "warmup": args.warmup, "ms_per_step": ms_per_step, "higher_is_better": True, "scaling": "weak",
            "vs_baseline": None, "dtype": "f32", "data": "synthetic", "config": config_block(w, args),
            "roofline": {
                "bound": "tensor",
                "kernel": "band products: band_tc_kernel (stage 1, stage 2) and band_fused_kernel (both stages)",
                "achieved": achieved, "peak": tf32_peak, "unit": "TFLOP/s", "frac": achieved / tf32_peak,
                "traffic": (BAND_TRAFFIC["bytes_per_launch"]
                            if BAND_TRAFFIC["sources_sha256"] == band_sources_sha256() else None),
                "traffic_source": BAND_TRAFFIC["profile"],
                "peak_source": f"{src} bf16 {bf16:.1f} TFLOP/s x {TF32_PER_BF16:.4f} (nominal TF32:BF16), burst",
                "flops_per_step": 3.0 * plan["structural_flops"],
                "flops_note": "3 TF32 MMAs per multiply-add (3xTF32) x the structurally non-zero multiply-adds of "
                              "the schedule's band products (2 per multiply-add)",
                "flops_issued_per_step": 3.0 * plan["update_flops"],
                "flops_issued_note": "tile-dense: the zero upper triangles of the diagonal factor tiles included",
                "band_ms_per_step": gemm_ms,
                "fused_nodes_per_step": int(pr["fused_launches"])},
            "band_levels": levels,
            "leaf": {"kernel": LEAF_KERNELS[leaf][0], "structure": leaf, "tune_ms": None if leaf_tune_ms is None else dict(zip(bk.LEAF_STRUCTURES, leaf_tune_ms)),
                     "ms_per_step": pr["leaf_ms"],
                     "launches_per_step": pr["leaf_launches"],
                     "achieved_gbs": leaf_bytes / (pr["leaf_ms"] / 1e3) / 1e9, "hbm_peak_gbs": hbm,
                     "bytes_per_step": leaf_bytes, "bound": "latency (dependent rounding steps)",
                     "sequential_steps_per_tile_diagonal": LEAF_KERNELS[leaf][1],
                     "ns_per_sequential_step": pr["leaf_ms"] * 1e6 / (plan["tile_diagonals"] * LEAF_KERNELS[leaf][1]),
                     "dependent_steps_per_solve": {str(k): plan["tile_diagonals"] * v[1] for k, v in LEAF_KERNELS.items()},
                     "dependent_steps_minimum": m + n - 1,
                     "share_of_profiled_step": pr["leaf_ms"] / pr["total_ms"]},
            "profile_ms": pr,
            "factor_ms": factor_ms,
            "proxy_loss": loss,
            "factor": {"ms": factor_ms, "flops": factor_flops(n) + factor_flops(m),
                       "fp64_tflops": (factor_flops(n) + factor_flops(m)) / (factor_ms / 1e3) / 1e12,
                       "fp64_peak_tflops_nominal": FP64_PEAK_NOMINAL,
                       "note": "chol(A^-1) and chol(B^-1) in FP64 (Cholesky d^3/6 + triangular inverse "
                               "d^3/6 multiply-adds, 2 flops each, per factor); outside the metric"},
            "cpu_baseline": cb,
            "e2e": None if e2e_ms is None else {
                "value": aggregate_rate(world, m, n, e2e_ms), "unit": "weights/s",
                "h2d_bytes_per_step": 4 * (m * n + n * n + m * m),
                "d2h_bytes_per_step": 4 * m * n + m * n + 4 * m},
            "batch": None if batch_ms is None else {
                "matrices_per_step": n_batch, "streams": n_batch, "ms_per_step": batch_ms,
                "value": aggregate_rate(world, m, n, batch_ms / n_batch), "unit": "weights/s",
                "note": "bakron_solve_batch of the same workload on separate streams (not the headline)"},
            "one_sided": None if one_ms is None else {
                "ms_per_step": one_ms, "value": aggregate_rate(world, m, n, one_ms), "unit": "weights/s",
                "note": "B = I path (one-sided GPTQ with Hessian A, column-block recursion) on the same W and A "
                        "(not the headline)"},
            "gpu_launches": launches_per_step * args.steps,
            "clocks": clk.summary(),
            "device_status": status.name,
        }
        print(json.dumps(line), flush=True)
    if dist is not None:
        dist.barrier()
        dist.destroy_process_group()
    return 0


if __name__ == "__main__":
    sys.exit(main())
