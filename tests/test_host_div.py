"""The launch-time divisor constants of the few-token product kernels
(Granlund-Montgomery multiply-high and shift, make_div_u31 in few_token.cuh)
against exact integer division, on the host: a small program built with nvcc
from the library's own header (no GPU needed)."""

import os
import subprocess

import pytest

from conftest import ROOT


def test_div_u31_constants(tmp_path):
    from bit_nf4_quantized_02_b200 import build
    csrc = os.path.join(ROOT, "bit_nf4_quantized_02_b200", "csrc")
    exe = str(tmp_path / "div_u31_check")
    cmd = [build.nvcc_path(), "-O2", "-std=c++17", "-gencode", "arch=compute_100a,code=sm_100a",
           "-I", os.path.join(ROOT, "include"), "-I", csrc, "-o", exe,
           os.path.join(ROOT, "tests", "host", "div_u31_check.cu")]
    res = subprocess.run(cmd, capture_output=True, text=True)
    if res.returncode != 0:
        pytest.fail("nvcc failed:\n" + res.stderr[-2000:])
    run = subprocess.run([exe], capture_output=True, text=True, timeout=300)
    assert run.returncode == 0, run.stdout + run.stderr
    assert " 0 wrong" in run.stdout
