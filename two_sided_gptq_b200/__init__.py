"""B200-native BaKron two-sided adaptive-rounding solver (Python binding).

Thin marshalling layer over the C ABI in ``include/bakron.h``: every step of
the computation runs in the library's CUDA kernels.  PyTorch supplies device
memory and streams only.

    LA, LB = factor(A, B)                       # chol(A^-1), chol(B^-1), FP64 inside
    V, codes, scales = solve(W, LA, LB, bits=4) # BaKron (Algorithm 6)
    loss = proxy_loss(W, V, A, B)               # tr((W-V)^T B (W-V) A)

Method: "BaKron: Efficient Quantization with Kronecker-Factored Hessians"
(arXiv 2608.06291).
"""
from __future__ import annotations

import ctypes

from . import _native
from ._native import BakronError, BatchItem, Config, PlanStats, Profile, ProfileLaunch, Quantizer, Status, check

__all__ = ["factor", "solve", "solve_host", "proxy_loss", "plan_stats", "last_profile",
           "last_profile_launches", "tune_leaf", "tune_cache_key", "tune_cache_get", "tune_cache_put",
           "solve_batch", "gram", "selftest_wait_timeout", "selftest_band_abort", "workspace", "get_status",
           "BakronError", "Status", "version", "library_path"]


# bakron_config_t.leaf values bakron_tune_leaf times (one ms_out entry each)
LEAF_STRUCTURES = (1, 2, 3, 4, 5, 6, 7, 8)


def _lib():
    return _native.load()


def library_path() -> str:
    return _native.LIB_PATH


def version() -> str:
    return _lib().bakron_version().decode()


def _torch():
    import torch

    return torch


def _ptr(t) -> int:
    return t.data_ptr() if t is not None else 0


def _stream(stream):
    torch = _torch()
    if stream is None:
        stream = torch.cuda.current_stream()
    return ctypes.c_void_p(stream.cuda_stream)


def _dev_f32(x, name):
    torch = _torch()
    if not isinstance(x, torch.Tensor) or not x.is_cuda or x.dtype != torch.float32 or not x.is_contiguous():
        raise TypeError(f"{name} must be a contiguous float32 CUDA tensor")
    return x


def _config(gemm=0, timeout_ms=0, wt_out=None, profile=False, leaf=0, b_identity=False, graph=False, fuse_width=0,
            self_test_omit=0):
    return Config(0, int(gemm), 1 if graph else 0, int(timeout_ms), _ptr(wt_out), 1 if profile else 0, int(leaf),
                  1 if b_identity else 0, int(fuse_width), int(self_test_omit))


def workspace(nbytes: int, device=None):
    """A device byte buffer usable as a workspace (torch owns the memory)."""
    torch = _torch()
    return torch.empty(max(int(nbytes), 256), dtype=torch.uint8, device=device or "cuda")


def get_status(ws, stream=None) -> Status:
    """Synchronise and return (and clear) the device status recorded in ``ws``."""
    return Status(_lib().bakron_get_status(_ptr(ws), ws.numel(), _stream(stream)))


def selftest_wait_timeout(timeout_ms: int, ws, stream=None) -> None:
    """Launch the bounded-wait self-test (``bakron_selftest_wait_timeout``): a
    device wait that nothing completes gives up after ``timeout_ms`` and records
    ``Status.ERR_DEVICE_TIMEOUT`` in ``ws``; read it with :func:`get_status`."""
    check(_lib().bakron_selftest_wait_timeout(int(timeout_ms), _ptr(ws), ws.numel(), _stream(stream)),
          "bakron_selftest_wait_timeout")


def selftest_band_abort(timeout_ms: int, ws=None, stream=None):
    """Launch the band kernel's abort-path self-test (``bakron_selftest_band_abort``):
    the stage-1 band kernel with no copies issued, whose bounded waits run out
    after ``timeout_ms``.  Returns the workspace; its status word then reads
    ``Status.ERR_DEVICE_TIMEOUT`` (read it with :func:`get_status`)."""
    need = _lib().bakron_selftest_band_abort_workspace_size()
    if ws is None:
        ws = workspace(need)
    check(_lib().bakron_selftest_band_abort(int(timeout_ms), _ptr(ws), ws.numel(), _stream(stream)),
          "bakron_selftest_band_abort")
    return ws


def factor(A, B=None, *, stream=None, ws=None, check_status=True):
    """``(LA, LB)`` with ``LA LA^T = A^{-1}``, ``LB LB^T = B^{-1}`` (lower, fp32)."""
    torch = _torch()
    lib = _lib()
    n = 0 if A is None else A.shape[0]
    m = 0 if B is None else B.shape[0]
    if A is not None:
        _dev_f32(A, "A")
    if B is not None:
        _dev_f32(B, "B")
    dev = (A if A is not None else B).device
    LA = torch.empty((n, n), dtype=torch.float32, device=dev) if n else None
    LB = torch.empty((m, m), dtype=torch.float32, device=dev) if m else None
    need = lib.bakron_factor_workspace_size(n, m)
    if ws is None:
        ws = workspace(need, dev)
    st = _stream(stream)
    check(lib.bakron_factor(_ptr(A), n, _ptr(B), m, _ptr(LA), _ptr(LB), _ptr(ws), ws.numel(), st), "bakron_factor")
    if check_status:
        check(lib.bakron_get_status(_ptr(ws), ws.numel(), st), "bakron_factor (device)")
    return LA, LB


def solve_workspace_size(m: int, n: int, gemm: int = 0) -> int:
    return int(_lib().bakron_solve_workspace_size(m, n, ctypes.byref(_config(gemm))))


def solve(W, LA, LB, bits=4, *, qmin=0, qmax=0, row_scale=None, gemm=0, ws=None, out=None, stream=None,
          wt_out=None, check_status=True, timeout_ms=0, profile=False, leaf=0, shrink_grid=0, graph=False,
          fuse_width=0, self_test_omit=0):
    """BaKron solve on device tensors.  Returns ``(V, codes, scales)``.

    ``LB=None`` selects the one-sided path (B = I: GPTQ with Hessian A, over
    128-column blocks).

    ``gemm=0`` uses the tcgen05 3xTF32 band products, ``gemm=1`` the FP32
    CUDA-core ones; ``shrink_grid`` > 1 searches each row's step for the least
    round-to-nearest error over that many shrink factors in [1/2, 1]; ``leaf``
    selects the leaf sweep structure (0 default (6),
    1 two-level CTA-wide, 2 single-level, 3 three warps per 32 x 32
    sub-tile, 4 six warps per 64 x 64 sub-tile, 5 as 3 with each tile on a
    cluster of four CTAs, 6 as 5 with the older product terms formed during
    the sweeps, 7 as 6 with two tile diagonals per launch (device flags, the
    width-2 nodes' updates inside the leaf), 8 continuous strip sweeps, one
    per CTA, staggered by 48 steps; :func:`tune_leaf` picks one by
    measurement).  ``self_test_omit`` is a self-test hook of structure 7.  ``fuse_width`` (0 default, 1 never) runs the two band
    products of recursion nodes at most that many tile diagonals wide as one
    launch per target tile.  ``graph=True`` captures the solve's launches for this
    argument set into a CUDA graph on the first call and replays it on later
    calls with the same buffers.  ``out`` may supply ``(V, codes, scales)`` buffers and
    ``ws`` a workspace; ``check_status=False`` skips the synchronising status
    read (for timing).
    """
    torch = _torch()
    lib = _lib()
    one_sided = LB is None
    _dev_f32(W, "W"), _dev_f32(LA, "LA")
    if not one_sided:
        _dev_f32(LB, "LB")
    m, n = W.shape
    if LA.shape != (n, n) or (not one_sided and LB.shape != (m, m)):
        raise ValueError("LA must be n x n and LB m x m")
    cfg = _config(gemm, timeout_ms, wt_out, profile, leaf, one_sided, graph, fuse_width, self_test_omit)
    if out is None:
        V = torch.empty((m, n), dtype=torch.float32, device=W.device)
        codes = torch.empty((m, n), dtype=torch.int8, device=W.device)
        scales = torch.empty((m,), dtype=torch.float32, device=W.device)
    else:
        V, codes, scales = out
    if ws is None:
        ws = workspace(lib.bakron_solve_workspace_size(m, n, ctypes.byref(cfg)), W.device)
    q = Quantizer(int(bits), int(qmin), int(qmax), _ptr(row_scale), int(shrink_grid))
    st = _stream(stream)
    check(lib.bakron_solve(_ptr(W), m, n, _ptr(LA), _ptr(LB), ctypes.byref(q), _ptr(V), _ptr(codes), _ptr(scales),
                           _ptr(ws), ws.numel(), ctypes.byref(cfg), st), "bakron_solve")
    if check_status:
        check(lib.bakron_get_status(_ptr(ws), ws.numel(), st), "bakron_solve (device)")
    return V, codes, scales


def tune_cache_key(m: int, n: int, bits: int, device_name: str) -> str:
    """Key of a leaf-structure measurement in the autotune cache (the library
    version is part of it: a new build re-measures)."""
    return f"{int(m)}x{int(n)}/int{int(bits)}/{device_name}/{version()}"


def tune_cache_get(path: str, key: str):
    """``(leaf, ms_list)`` stored under ``key`` in the JSON file ``path``, or None."""
    import json
    import os

    if not path or not os.path.exists(path):
        return None
    try:
        with open(path) as f:
            entry = json.load(f).get(key)
    except (OSError, ValueError):
        return None
    if not isinstance(entry, dict) or entry.get("leaf") not in LEAF_STRUCTURES:
        return None
    return int(entry["leaf"]), [float(x) for x in entry.get("ms", [])]


def tune_cache_put(path: str, key: str, leaf: int, ms) -> None:
    """Store a measurement under ``key`` in the JSON file ``path`` (written to a
    temporary file and renamed, so readers never see a partial file)."""
    import json
    import os
    import tempfile

    data = {}
    if os.path.exists(path):
        try:
            with open(path) as f:
                data = json.load(f)
        except (OSError, ValueError):
            data = {}
    data[key] = {"leaf": int(leaf), "ms": [float(x) for x in ms]}
    d = os.path.dirname(os.path.abspath(path))
    fd, tmp = tempfile.mkstemp(dir=d, prefix=".bakron_tune_")
    with os.fdopen(fd, "w") as f:
        json.dump(data, f, indent=1, sort_keys=True)
    os.replace(tmp, path)


def tune_leaf(W, LA, LB, bits=4, *, ws=None, out=None, stream=None, gemm=0, timeout_ms=0, cache=None):
    """Leaf structure chosen by measurement (``bakron_tune_leaf``): one timed
    solve per structure on this problem.  Returns ``(leaf, [ms_leaf1, ...,
    ms_leaf8])``; pass ``leaf`` to :func:`solve`.

    ``cache`` (or the ``BAKRON_TUNE_CACHE`` environment variable) names a JSON
    file keyed by (m, n, bits, GPU name): a stored measurement is returned
    without timing, a new one is stored."""
    import os

    torch = _torch()
    lib = _lib()
    _dev_f32(W, "W"), _dev_f32(LA, "LA"), _dev_f32(LB, "LB")
    m, n = W.shape
    cache = cache or os.environ.get("BAKRON_TUNE_CACHE")
    key = tune_cache_key(m, n, bits, torch.cuda.get_device_name(W.device)) if cache else None
    if cache:
        hit = tune_cache_get(cache, key)
        if hit is not None:
            return hit
    cfg = _config(gemm, timeout_ms)
    if out is None:
        out = (torch.empty((m, n), dtype=torch.float32, device=W.device),
               torch.empty((m, n), dtype=torch.int8, device=W.device),
               torch.empty((m,), dtype=torch.float32, device=W.device))
    V, codes, scales = out
    if ws is None:
        ws = workspace(lib.bakron_solve_workspace_size(m, n, ctypes.byref(cfg)), W.device)
    q = Quantizer(int(bits), 0, 0, None)
    leaf = ctypes.c_int32(0)
    ms = (ctypes.c_double * len(LEAF_STRUCTURES))()
    st = _stream(stream)
    check(lib.bakron_tune_leaf(_ptr(W), m, n, _ptr(LA), _ptr(LB), ctypes.byref(q), _ptr(V), _ptr(codes),
                               _ptr(scales), _ptr(ws), ws.numel(), ctypes.byref(cfg), st, ctypes.byref(leaf), ms),
          "bakron_tune_leaf")
    check(lib.bakron_get_status(_ptr(ws), ws.numel(), st), "bakron_tune_leaf (device)")
    result = int(leaf.value), [float(x) for x in ms]
    if cache:
        tune_cache_put(cache, key, *result)
    return result


def solve_batch(problems, bits=4, *, streams, outs=None, workspaces=None, gemm=0, leaf=0, shrink_grid=0,
                check_status=True, fuse_width=0):
    """Independent solves through ``bakron_solve_batch``: ``problems`` is a list
    of ``(W, LA, LB)`` device tensors, solve i runs on ``streams[i %
    len(streams)]`` (torch streams).  ``outs`` / ``workspaces`` may supply the
    ``(V, codes, scales)`` buffers and workspaces.  Returns the list of
    ``(V, codes, scales)``."""
    torch = _torch()
    lib = _lib()
    cfg = _config(gemm, leaf=leaf, fuse_width=fuse_width)
    items = (BatchItem * max(1, len(problems)))()
    res, wss = [], []
    for i, (W, LA, LB) in enumerate(problems):
        _dev_f32(W, "W"), _dev_f32(LA, "LA"), _dev_f32(LB, "LB")
        m, n = W.shape
        if outs is None:
            o = (torch.empty((m, n), dtype=torch.float32, device=W.device),
                 torch.empty((m, n), dtype=torch.int8, device=W.device),
                 torch.empty((m,), dtype=torch.float32, device=W.device))
        else:
            o = outs[i]
        ws = workspaces[i] if workspaces is not None else workspace(
            lib.bakron_solve_workspace_size(m, n, ctypes.byref(cfg)), W.device)
        items[i] = BatchItem(_ptr(W), m, n, _ptr(LA), _ptr(LB), _ptr(o[0]), _ptr(o[1]), _ptr(o[2]), _ptr(ws),
                             ws.numel())
        res.append(o)
        wss.append(ws)
    st = (ctypes.c_void_p * len(streams))(*[s.cuda_stream for s in streams])
    q = Quantizer(int(bits), 0, 0, None, int(shrink_grid))
    check(lib.bakron_solve_batch(items, len(problems), ctypes.byref(q), ctypes.byref(cfg), st, len(streams)),
          "bakron_solve_batch")
    if check_status:
        for i, ws in enumerate(wss):
            check(lib.bakron_get_status(_ptr(ws), ws.numel(), _stream(streams[i % len(streams)])),
                  f"bakron_solve_batch item {i} (device)")
    return res


def gram(X, damping=0.0, *, ws=None, out=None, stream=None, check_status=True):
    """Kronecker factor ``X^T X / N + damping * mean(diag) * I`` from samples
    ``X`` (N x d device tensor) on the tensor cores (``bakron_gram``)."""
    torch = _torch()
    lib = _lib()
    _dev_f32(X, "X")
    N, d = X.shape
    A = torch.empty((d, d), dtype=torch.float32, device=X.device) if out is None else out
    if ws is None:
        ws = workspace(lib.bakron_gram_workspace_size(N, d), X.device)
    st = _stream(stream)
    check(lib.bakron_gram(_ptr(X), N, d, float(damping), _ptr(A), _ptr(ws), ws.numel(), st), "bakron_gram")
    if check_status:
        check(lib.bakron_get_status(_ptr(ws), ws.numel(), st), "bakron_gram (device)")
    return A


def solve_host_workspace_size(m: int, n: int, gemm: int = 0) -> int:
    return int(_lib().bakron_solve_host_workspace_size(m, n, ctypes.byref(_config(gemm))))


def solve_host(W, LA, LB, bits=4, *, V=None, codes=None, scales=None, gemm=0, ws=None, stream=None,
               synchronize=True, leaf=0, fuse_width=0):
    """BaKron solve on HOST buffers (torch CPU tensors, ideally pinned): the
    library stages them through ``ws`` on the device and copies the results
    back.  Returns ``(V, codes, scales)`` host tensors."""
    torch = _torch()
    lib = _lib()
    m, n = W.shape
    for t, name in ((W, "W"), (LA, "LA"), (LB, "LB")):
        if t is None and name == "LB":
            continue  # B = I: the one-sided path
        if t.is_cuda or t.dtype != torch.float32 or not t.is_contiguous():
            raise TypeError(f"{name} must be a contiguous float32 CPU tensor")
    V = torch.empty((m, n), dtype=torch.float32, pin_memory=True) if V is None else V
    codes = torch.empty((m, n), dtype=torch.int8, pin_memory=True) if codes is None else codes
    scales = torch.empty((m,), dtype=torch.float32, pin_memory=True) if scales is None else scales
    cfg = _config(gemm, leaf=leaf, b_identity=int(LB is None), fuse_width=fuse_width)
    if ws is None:
        ws = workspace(lib.bakron_solve_host_workspace_size(m, n, ctypes.byref(cfg)))
    q = Quantizer(int(bits), 0, 0, 0)
    st = _stream(stream)
    check(lib.bakron_solve_host(_ptr(W), m, n, _ptr(LA), _ptr(LB), ctypes.byref(q), _ptr(V), _ptr(codes),
                                _ptr(scales), _ptr(ws), ws.numel(), ctypes.byref(cfg), st), "bakron_solve_host")
    if synchronize:
        check(lib.bakron_get_status(_ptr(ws), ws.numel(), st), "bakron_solve_host (device)")
    return V, codes, scales


def proxy_loss(W, V, A, B, *, stream=None) -> float:
    """``tr((W-V)^T B (W-V) A)`` computed on the device (both products on the
    tensor cores in 3xTF32, the elementwise dot in FP64 in a fixed order)."""
    torch = _torch()
    lib = _lib()
    m, n = W.shape
    out = torch.zeros((1,), dtype=torch.float64, device=W.device)
    ws = workspace(lib.bakron_proxy_loss_workspace_size(m, n), W.device)
    host = ctypes.c_double(0.0)
    check(lib.bakron_proxy_loss(_ptr(W), _ptr(V), _ptr(A), _ptr(B), m, n, _ptr(out), ctypes.byref(host), _ptr(ws),
                                ws.numel(), _stream(stream)), "bakron_proxy_loss")
    return float(host.value)


def last_profile() -> dict:
    """Per-kernel-class device times (ms) of the latest ``solve(..., profile=True)``
    on this thread."""
    pr = Profile()
    check(_lib().bakron_get_profile(ctypes.byref(pr)), "bakron_get_profile")
    return {f: getattr(pr, f) for f, _ in Profile._fields_}


def last_profile_launches() -> list:
    """Every launch of the latest ``solve(..., profile=True)`` on this thread, in
    launch order: dicts with kind ("prep", "leaf", "stage1", "stage2", "fused":
    both band products of a node in one launch), the recursion node (k, h, l)
    in tile diagonals, ms, FLOPs (tile-dense) and structural FLOPs (without
    the zero upper triangles of the diagonal factor tiles)."""
    lib = _lib()
    n = lib.bakron_get_profile_launches(None, 0)
    buf = (ProfileLaunch * max(1, n))()
    lib.bakron_get_profile_launches(buf, n)
    kinds = ("prep", "leaf", "stage1", "stage2", "fused")
    return [{"kind": kinds[r.kind], "k": r.k, "h": r.h, "l": r.l, "ms": r.ms, "flops": r.flops,
             "structural_flops": r.structural_flops} for r in buf[:n]]


def plan_stats(m: int, n: int, one_sided: bool = False, leaf: int = 0) -> dict:
    """Schedule statistics of an m x n solve (host only); ``one_sided`` for
    the B = I schedule over column blocks; ``leaf`` the leaf structure (7
    moves the width-2 nodes' products into the leaf launches)."""
    s = PlanStats()
    cfg = _config(b_identity=int(one_sided), leaf=leaf)
    check(_lib().bakron_plan_stats(m, n, ctypes.byref(cfg), ctypes.byref(s)), "bakron_plan_stats")
    return {f: getattr(s, f) for f, _ in PlanStats._fields_}
