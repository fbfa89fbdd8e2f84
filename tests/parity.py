"""Helpers shared by the GPU parity tests: run the CUDA path and check it
against the oracle on the same seeded inputs.

Tolerances (the solve's contract):
  * codes: bit-exact except at rounding ties -- a disagreement is allowed only
    where the oracle's FP64 pre-rounding value lies within TIE_EPS = 1e-6
    (absolute, weight units) of the midpoint between the two codes, and such
    ties are capped at 1e-5 of the entries, counted in whole entries
    (ceil(1e-5 mn): an entry closer to a midpoint than fp32 can resolve is
    undecidable in the kernel's precision even in a small matrix); anything
    else is a failure.  Checked teacher-forced (the oracle adopts the GPU's
    code at every entry), so one tie flip cannot cascade.
  * steps s_i: bit-exact (same fp32 division on both sides).
  * V: V = s_i * code exactly in fp32 on the GPU; relative Frobenius error
    against the oracle's V <= 1e-4, over the entries whose code is unique
    (at a tie both codes are valid, so there the GPU's code is taken).
  * proxy loss: relative error <= 1e-4.
"""
from __future__ import annotations

import math

import numpy as np

import oracle

TIE_EPS = 1e-6
TIE_FRAC = 1e-5
V_RTOL = 1e-4
LOSS_RTOL = 1e-4


def tie_cap(entries: int) -> int:
    return math.ceil(TIE_FRAC * entries)


def oracle_factors(A, B):
    """FP64 oracle factors, rounded to fp32 (the form the GPU solve consumes)."""
    LA = oracle.factor(A).astype(np.float32)
    LB = oracle.factor(B).astype(np.float32)
    return LA, LB


def gpu_solve(W, LA32, LB32, bits, gemm=0, row_scale=None, leaf=0, fuse_width=0):
    import torch

    import two_sided_gptq_b200 as bk

    dev = "cuda"
    Wd = torch.from_numpy(np.ascontiguousarray(W)).to(dev)
    LAd = torch.from_numpy(np.ascontiguousarray(LA32)).to(dev)
    LBd = None if LB32 is None else torch.from_numpy(np.ascontiguousarray(LB32)).to(dev)  # None: B = I
    wt = torch.empty_like(Wd)
    rs = None if row_scale is None else torch.from_numpy(np.asarray(row_scale, np.float32)).to(dev)
    V, codes, scales = bk.solve(Wd, LAd, LBd, bits=bits, gemm=gemm, wt_out=wt, row_scale=rs, leaf=leaf,
                                fuse_width=fuse_width)
    torch.cuda.synchronize()
    return V.cpu().numpy(), codes.cpu().numpy().astype(np.int32), scales.cpu().numpy(), wt.cpu().numpy()


CANARY = 0xA5  # guard byte around every buffer of a canary-checked solve
GUARD = 4096  # guard bytes on each side (a multiple of 256 keeps 16-byte alignment)


def gpu_solve_canaries(W, LA32, LB32, bits, leaf=0, fuse_width=0, gemm=0):
    """The GPU solve with its workspace and outputs (V, codes, steps) carved
    out of larger buffers whose guard zones, and the gap after the
    workspace's 256-byte status block (the next buffer starts 1 KiB in), hold
    CANARY bytes: a substitute for an out-of-bounds checker.  Asserts that no
    guard byte changed; returns host arrays like gpu_solve (no pre-rounding
    values)."""
    import torch

    import two_sided_gptq_b200 as bk

    m, n = W.shape

    def guarded(nbytes):
        raw = torch.full((nbytes + 2 * GUARD,), CANARY, dtype=torch.uint8, device="cuda")
        return raw, raw[GUARD:GUARD + nbytes]

    ws_bytes = bk.solve_workspace_size(m, n, gemm)
    raw_ws, ws = guarded(ws_bytes)
    raw_v, v = guarded(4 * m * n)
    raw_c, c = guarded(m * n)
    raw_s, sc = guarded(4 * m)
    V = v.view(torch.float32).view(m, n)
    codes = c.view(torch.int8).view(m, n)
    scales = sc.view(torch.float32)
    Wd = torch.from_numpy(np.ascontiguousarray(W)).cuda()
    LAd = torch.from_numpy(np.ascontiguousarray(LA32)).cuda()
    LBd = None if LB32 is None else torch.from_numpy(np.ascontiguousarray(LB32)).cuda()
    bk.solve(Wd, LAd, LBd, bits=bits, gemm=gemm, ws=ws, out=(V, codes, scales), leaf=leaf, fuse_width=fuse_width)
    torch.cuda.synchronize()
    for name, raw, size in (("workspace", raw_ws, ws_bytes), ("V", raw_v, 4 * m * n), ("codes", raw_c, m * n),
                            ("steps", raw_s, 4 * m)):
        h = raw.cpu().numpy()
        assert np.all(h[:GUARD] == CANARY), f"write before the {name} buffer"
        assert np.all(h[GUARD + size:] == CANARY), f"write after the {name} buffer"
    gap = raw_ws[GUARD + 256:GUARD + 1024].cpu().numpy()
    assert np.all(gap == CANARY), "write into the gap after the status block"
    return V.cpu().numpy(), codes.cpu().numpy().astype(np.int32), scales.cpu().numpy()


def check_solve(W, LA32, LB32, bits, gemm=0, row_scale=None, label="", leaf=0, fuse_width=0):
    """Run the GPU solve on (W, LA32, LB32) and check it teacher-forced
    against the oracle using the same fp32 factors (widened to FP64).
    Returns the report dict (asserts the contract)."""
    V, codes, s_gpu, wt_gpu = gpu_solve(W, LA32, LB32, bits, gemm, row_scale, leaf, fuse_width)
    return check_outputs(W, LA32, LB32, bits, V, codes, s_gpu, wt_gpu, row_scale, label)


def check_outputs(W, LA32, LB32, bits, V, codes, s_gpu, wt_gpu=None, row_scale=None, label=""):
    """Check one solve's outputs (host arrays: V fp32, codes int, steps fp32,
    optionally the pre-rounding values) teacher-forced against the oracle on
    the same fp32 factors.  LB32 None means B = I.  Returns the report dict
    (asserts the contract)."""
    qmin, qmax = oracle.grid(bits)
    codes = np.asarray(codes).astype(np.int32)
    s = oracle.scales(W, qmax) if row_scale is None else np.asarray(row_scale, np.float32)
    assert np.array_equal(np.asarray(s_gpu, np.float32).view(np.uint32), s.view(np.uint32)), f"{label}: steps differ"
    LtA = oracle.normalize(LA32.astype(np.float64))
    # B = I (the one-sided path): the pull with an identity row factor
    LtB = np.eye(W.shape[0]) if LB32 is None else oracle.normalize(LB32.astype(np.float64))
    r = oracle.forced_check(W, LtA, LtB, s, qmin, qmax, codes, tie_eps=TIE_EPS)
    m, n = W.shape
    r["label"] = label
    if wt_gpu is not None:
        r["wt_max_abs_err"] = float(np.abs(wt_gpu.astype(np.float64) - r["Wt"]).max())
    else:
        r["wt_max_abs_err"] = float("nan")
    r["wt_scale"] = float(np.abs(r["Wt"]).max())
    # codes within the grid, V = s * code exactly in fp32
    assert codes.min() >= qmin and codes.max() <= qmax
    assert np.array_equal(V, (s[:, None] * codes.astype(np.float32)).astype(np.float32))
    own = r["own"].copy()
    tie_mask = (own != codes)
    if r["ties"] and not r["failures"]:
        own[tie_mask] = codes[tie_mask]
    V_or = s.astype(np.float64)[:, None] * own
    r["v_rel_err"] = float(np.linalg.norm(V - V_or) / max(np.linalg.norm(V_or), 1e-300))
    print(f"[{label}] m={m} n={n} mismatches={r['mismatches']} ties={r['ties']} failures={r['failures']} "
          f"max_fail_dist={r['max_fail_dist']:.3g} max_tie_dist={r['max_tie_dist']:.3g} wt_err={r['wt_max_abs_err']:.3g} (|Wt|max {r['wt_scale']:.3g}) "
          f"v_rel={r['v_rel_err']:.3g}")
    assert r["failures"] == 0, f"{label}: {r['failures']} code failures (max dist {r['max_fail_dist']})"
    assert r["ties"] <= tie_cap(m * n), f"{label}: {r['ties']} tie disagreements > {TIE_FRAC} of {m * n}"
    assert r["v_rel_err"] <= V_RTOL
    return r
