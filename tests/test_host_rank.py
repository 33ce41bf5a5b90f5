"""The grouped rank-r kernel's schedule on the host: the split planner, the
launch order and the kernel's own unit decoding and boustrophedon walk
(rank_gemm.cuh), replayed for every CTA over the backward groups of LLaMA-7B
and -65B, ragged shapes and random problem lists (a small program built with
nvcc from the library's header; no GPU needed)."""

import os
import subprocess

import pytest

from conftest import ROOT


def test_rank_walk(tmp_path):
    from bit_nf4_quantized_02_b200 import build
    csrc = os.path.join(ROOT, "bit_nf4_quantized_02_b200", "csrc")
    exe = str(tmp_path / "rank_walk_check")
    cmd = [build.nvcc_path(), "-O2", "-std=c++17", "-gencode", "arch=compute_100a,code=sm_100a",
           "-I", os.path.join(ROOT, "include"), "-I", csrc, "-o", exe,
           os.path.join(ROOT, "tests", "host", "rank_walk_check.cu")]
    res = subprocess.run(cmd, capture_output=True, text=True)
    if res.returncode != 0:
        pytest.fail("nvcc failed:\n" + res.stderr[-2000:])
    run = subprocess.run([exe], capture_output=True, text=True, timeout=600)
    assert run.returncode == 0, run.stdout + run.stderr
    assert " 0 wrong" in run.stdout
