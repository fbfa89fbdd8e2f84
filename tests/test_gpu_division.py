"""The rounding decisions divide by the grid step without a divide
instruction (Markstein's correction from the correctly rounded reciprocal,
div_rn_recip in csrc/common.cuh).  This test builds tests/cuda/div_check.cu and
compares it with CUDA's IEEE division on about 8e8 pairs with steps in
[2^-60, 2^60] (the range the kernels use it for): quotients a few ulps from
half-integers for every significand of the step, random normal-range pairs
and weight-like magnitudes.  Quotients agree bit for bit when |a| >= 2^-100,
and rint(quotient) -- the rounding decision -- agrees on every pair."""
import os
import subprocess

import pytest

pytestmark = pytest.mark.gpu

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def test_division_matches_ieee(tmp_path):
    import torch

    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    exe = str(tmp_path / "div_check")
    nvcc = os.environ.get("NVCC", "/usr/local/cuda/bin/nvcc")
    subprocess.run([nvcc, "-gencode", "arch=compute_100a,code=sm_100a", "-O3", "-std=c++17",
                    "-I", os.path.join(ROOT, "two_sided_gptq_b200", "csrc"), "-I", os.path.join(ROOT, "include"),
                    "-o", exe, os.path.join(ROOT, "tests", "cuda", "div_check.cu")], check=True)
    r = subprocess.run([exe], capture_output=True, text=True, timeout=300)
    print(r.stdout)
    assert r.returncode == 0, r.stdout + r.stderr
    lines = [l for l in r.stdout.splitlines() if l.startswith("mode")]
    assert len(lines) == 3 and all(" mismatches 0 decision_mismatches 0" in l for l in lines), r.stdout
