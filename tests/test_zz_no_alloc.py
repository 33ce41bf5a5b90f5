"""The no-allocation quantizer entry point gives the same result as the regular one.

Some callers cannot allocate device memory where they quantize (a framework
that owns every device byte through its own pool, or latency-critical code that
cannot afford cudaMalloc's implicit synchronization), so the library offers
qlora_quantize_nf4_dq_noalloc, whose scratch is a fixed static device array.
This test calls it through the C ABI twice in a row, with different inputs
(the second smaller, so stale scratch from the first call would show), and
compares every output with the regular entry point's, bit for bit.  It lives in
a file of its own that pytest collects last.
"""

import ctypes

import numpy as np
import pytest
import torch

from synth import inputs

pytestmark = pytest.mark.gpu

qlora = pytest.importorskip("bit_nf4_quantized_02_b200")


def _noalloc(lib, W: torch.Tensor):
    from bit_nf4_quantized_02_b200 import _lib
    n_out, k_in = W.shape
    numel = n_out * k_in
    nblk = (numel + 63) // 64
    dev = W.device
    codes = torch.empty((numel + 1) // 2, dtype=torch.uint8, device=dev)
    c2_fp8 = torch.empty(nblk, dtype=torch.uint8, device=dev)
    c1 = torch.empty((nblk + 255) // 256, dtype=torch.float32, device=dev)
    mu = torch.empty(1, dtype=torch.float32, device=dev)
    dt = _lib.QLORA_DTYPE_F32 if W.dtype == torch.float32 else _lib.QLORA_DTYPE_BF16
    rc = lib.qlora_quantize_nf4_dq_noalloc(W.data_ptr(), dt, n_out, k_in, codes.data_ptr(), c2_fp8.data_ptr(),
                                           c1.data_ptr(), mu.data_ptr(), torch.cuda.current_stream().cuda_stream)
    assert rc == _lib.QLORA_OK, lib.qlora_status_str(rc)
    return codes, c2_fp8, c1, mu


def test_noalloc_matches_regular_entry_on_two_calls():
    from bit_nf4_quantized_02_b200 import _lib
    lib = _lib.load()
    cases = [((1024, 4096), torch.float32, 61), ((300, 1000), torch.bfloat16, 62)]  # 2nd: smaller, tail blocks
    for shape, dtype, seed in cases:
        W = torch.from_numpy(inputs.normal_f32(inputs.rng(seed), shape, 0.02)).to(dtype).cuda()
        ref = qlora.quantize_nf4_dq(W)
        got = _noalloc(lib, W)
        torch.cuda.synchronize()
        for a, b in zip(got, (ref.codes, ref.c2_fp8, ref.c1, ref.c2_mean)):
            assert torch.equal(a.view(torch.uint8), b.view(torch.uint8))
    assert qlora.last_device_error() == 0


def test_noalloc_rejects_sizes_beyond_its_scratch():
    from bit_nf4_quantized_02_b200 import _lib
    lib = _lib.load()
    too_big = _lib.QLORA_NOALLOC_MAX_NUMEL // 4096 + 1
    rc = lib.qlora_quantize_nf4_dq_noalloc(None, _lib.QLORA_DTYPE_F32, too_big, 4096, None, None, None, None, None)
    assert rc == _lib.QLORA_ERR_SCRATCH_LIMIT
    assert b"scratch" in lib.qlora_status_str(rc)
