"""The boundary's stream and error rules on the GPU.

* The first library call in a fresh process enqueues its work and returns
  while another stream's kernel is still running (no device-wide
  synchronization on first use), and its result is bit-exact.
* A bounded wait inside a kernel that runs out is reported once by
  qlora_get_last_device_error as QLORA_ERR_DEVICE_TIMEOUT; the next call
  reports QLORA_OK, and a linear run afterwards is still within tolerance.
  The wait runs out on a barrier that nothing completes, under a 1 ms limit:
  no fault, no trap, nothing left in flight.
"""

import json
import os
import subprocess
import sys

import numpy as np
import pytest
import torch

from conftest import ROOT
from parity import assert_close, bf16_to_np, oracle_bwd, oracle_fwd, oracle_quant, oracle_w_hat
from synth import inputs

pytestmark = pytest.mark.gpu

qlora = pytest.importorskip("bit_nf4_quantized_02_b200")

# The child process: load the library before CUDA starts, put a ~2 s spin
# kernel on one stream, then make the library's first call (the quantizer) on
# another stream and record how long the call took on the host and whether
# the spin kernel was still running when it returned and when the quantizer's
# stream had finished.  CUDA_MODULE_LOADING is EAGER in the child so that the
# library's kernels are loaded with the context: under lazy loading the CUDA
# runtime loads a kernel at its first launch and may wait for the device to
# do so, for any library's kernels, which is not the library's doing.
_CHILD = r"""
import json, sys, time
import numpy as np
sys.path.insert(0, sys.argv[1])
from bit_nf4_quantized_02_b200 import _lib
lib = _lib.load()
import torch
from synth import inputs
from oracle import nf4dq
g = inputs.rng(4321)
W_cpu = torch.from_numpy(inputs.normal_f32(g, (96, 4096), 0.02))
W = W_cpu.cuda()
numel = W.numel()
nblk = (numel + 63) // 64
codes = torch.empty((numel + 1) // 2, dtype=torch.uint8, device="cuda")
c2_fp8 = torch.empty(nblk, dtype=torch.uint8, device="cuda")
c1 = torch.empty((nblk + 255) // 256, dtype=torch.float32, device="cuda")
mu = torch.empty(1, dtype=torch.float32, device="cuda")
ws_bytes = lib.qlora_quantize_workspace_size(numel)
ws = torch.empty(ws_bytes, dtype=torch.uint8, device="cuda")
side, main = torch.cuda.Stream(), torch.cuda.Stream()
torch.cuda.synchronize()
with torch.cuda.stream(side):
    torch.cuda._sleep(4_000_000_000)     # ~2 s at 1.9 GHz
    done = torch.cuda.Event()
    done.record()
t0 = time.perf_counter()
rc = lib.qlora_quantize_nf4_dq(W.data_ptr(), _lib.QLORA_DTYPE_F32, W.shape[0], W.shape[1], codes.data_ptr(),
                               c2_fp8.data_ptr(), c1.data_ptr(), mu.data_ptr(), ws.data_ptr(), ws_bytes,
                               main.cuda_stream)
call_s = time.perf_counter() - t0
side_busy = not done.query()
main.synchronize()
main_done_s = time.perf_counter() - t0
side_busy_after_main = not done.query()
torch.cuda.synchronize()
oq = nf4dq.quantize_nf4_dq(W_cpu.numpy())
exact = (np.array_equal(codes.cpu().numpy(), oq["packed"]) and np.array_equal(c2_fp8.cpu().numpy(), oq["c2_fp8"])
         and np.array_equal(c1.cpu().numpy().view(np.uint32), oq["c1"].view(np.uint32))
         and float(mu.cpu()[0]) == float(oq["mu"]))
print(json.dumps({"rc": rc, "call_s": call_s, "side_busy": side_busy, "main_done_s": main_done_s,
                  "side_busy_after_main": side_busy_after_main, "exact": bool(exact)}))
"""


def test_first_call_does_not_synchronize_the_device():
    env = dict(os.environ, CUDA_MODULE_LOADING="EAGER", PYTHONPATH=ROOT)
    out = subprocess.run([sys.executable, "-c", _CHILD, ROOT], capture_output=True, text=True, env=env,
                         timeout=600)
    assert out.returncode == 0, out.stderr[-3000:]
    res = json.loads(out.stdout.strip().splitlines()[-1])
    assert res["rc"] == 0
    # the call returned while the other stream's kernel was still running,
    # and the quantizer finished on its own stream before that kernel ended
    assert res["side_busy"], res
    assert res["call_s"] < 0.5, res
    assert res["side_busy_after_main"], res
    assert res["exact"], res


def _lib():
    from bit_nf4_quantized_02_b200 import _lib as L
    return L, L.load()


def test_set_wait_limit_rejects_too_long():
    L, lib = _lib()
    st = torch.cuda.current_stream().cuda_stream
    assert lib.qlora_set_wait_limit_ns(L.QLORA_MAX_WAIT_LIMIT_NS + 1, st) == L.QLORA_ERR_INVALID_ARG


def _small_linear_checked(seed: int):
    M, N, K, r, s = 200, 264, 320, 16, 1.0
    g = inputs.rng(seed)
    W = torch.from_numpy(inputs.weight_f32(g, N, K))
    X = inputs.normal_bf16(g, (M, K))
    L1, L2 = inputs.lora_factors(g, K, N, r)
    dY = inputs.normal_bf16(g, (M, N))
    q = qlora.quantize_nf4_dq(W.cuda())
    Xd, L1d, L2d, dYd = X.cuda(), L1.cuda(), L2.cuda(), dY.cuda()
    Y, T = qlora.linear_fwd(Xd, q, L1d, L2d, s)
    dX, dL1, dL2 = qlora.linear_bwd(dYd, Xd, T, q, L1d, L2d, s)
    torch.cuda.synchronize()
    w_hat = oracle_w_hat(oracle_quant(W))
    Y_ref, _ = oracle_fwd(X, w_hat, L1, L2, s)
    dX_ref, dL1_ref, dL2_ref = oracle_bwd(dY, X, w_hat, L1, L2, s)
    assert_close(bf16_to_np(Y), Y_ref, "Y")
    assert_close(bf16_to_np(dX), dX_ref, "dX")
    assert_close(dL1.float().cpu().numpy(), dL1_ref, "dL1")
    assert_close(dL2.float().cpu().numpy(), dL2_ref, "dL2")


def test_expired_wait_is_reported_then_cleared():
    L, lib = _lib()
    stream = torch.cuda.current_stream()
    st = stream.cuda_stream
    assert lib.qlora_get_last_device_error(st) == L.QLORA_OK      # start from a clear word
    limit_ns = 1_000_000                                           # 1 ms
    try:
        assert lib.qlora_set_wait_limit_ns(limit_ns, st) == L.QLORA_OK
        t0, t1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        t0.record(stream)
        assert lib.qlora_diag_expired_wait(st) == L.QLORA_OK
        t1.record(stream)
        assert lib.qlora_get_last_device_error(st) == L.QLORA_ERR_DEVICE_TIMEOUT
        waited_ms = t0.elapsed_time(t1)
        assert 0.9 * limit_ns / 1e6 <= waited_ms < 1000.0, waited_ms
        # reported once: the word was cleared by the read
        assert lib.qlora_get_last_device_error(st) == L.QLORA_OK
    finally:
        assert lib.qlora_set_wait_limit_ns(0, st) == L.QLORA_OK     # back to the default
    # the context is intact: the library's normal path still meets the tolerance
    _small_linear_checked(seed=91)
    assert lib.qlora_get_last_device_error(st) == L.QLORA_OK
