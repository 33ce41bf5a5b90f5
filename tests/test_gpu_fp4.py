"""GPU parity of the FP4 (E2M1) code table, the 4-bit float the paper compares
NF4 against (§4, Tables 2-4): bit-exact quantizer and doubleDequant against
the oracle with the FP4 table, and the linear's forward and backward (every
token-count path) within the stated tolerances."""

import numpy as np
import pytest
import torch

from oracle import nf4dq, qlora_linear
from parity import assert_close, bf16_to_np, gpu_quant_to_np
from synth import inputs

pytestmark = pytest.mark.gpu

qlora = pytest.importorskip("bit_nf4_quantized_02_b200")
FP4 = nf4dq.FP4_VALUES


def _check_fp4_bit_exact(W_cpu: torch.Tensor):
    q = qlora.quantize_nf4_dq(W_cpu.cuda(), table="fp4")
    got = gpu_quant_to_np(q)
    oq = nf4dq.quantize_nf4_dq(W_cpu.float().numpy(), FP4)
    assert got["mu"] == oq["mu"]
    assert np.array_equal(got["packed"], oq["packed"])
    assert np.array_equal(got["c2_fp8"], oq["c2_fp8"])
    assert np.array_equal(got["c1"].view(np.uint32), oq["c1"].view(np.uint32))
    w_hat = qlora.dequant(q)
    ref = nf4dq.double_dequant_bits(oq["codes"], oq["c2_fp8"], oq["c1"], oq["mu"], oq["shape"], FP4)
    assert np.array_equal(w_hat.cpu().view(torch.int16).numpy().view(np.uint16), ref)
    assert qlora.last_device_error() == 0
    return q, oq


@pytest.mark.parametrize("shape", [(1, 64), (3, 100), (7, 333), (64, 4096), (257, 64 * 257)])
@pytest.mark.parametrize("dtype", [torch.float32, torch.bfloat16])
def test_fp4_quantize_dequant_bit_exact(shape, dtype):
    g = inputs.rng(300 + shape[0] + shape[1])
    _check_fp4_bit_exact(torch.from_numpy(inputs.normal_f32(g, shape, 0.02)).to(dtype))


def test_fp4_special_values_and_thresholds():
    W = torch.zeros(4, 512, dtype=torch.float32)
    W[1, :64] = torch.linspace(-1, 1, 64)
    W[2, 64:128] = -3.0
    mids = nf4dq.midpoints(FP4).astype(np.float32)
    # every threshold, a few ulps either side, scaled by two absmax values
    row = []
    for m in mids:
        u = d = np.float32(m)
        row.append(u)
        for _ in range(3):
            u = np.nextafter(u, np.float32(2), dtype=np.float32)
            d = np.nextafter(d, np.float32(-2), dtype=np.float32)
            row += [u, d]
    row = np.clip(np.array(row, np.float32), -1, 1)
    W[3, 0] = 1.0
    W[3, 1:1 + min(63, row.size)] = torch.from_numpy(row[:63])
    W[3, 64] = -0.37
    W[3, 65:65 + min(63, row.size - 63)] = torch.from_numpy((row[63:126] * np.float32(0.37)).astype(np.float32))
    W[0, 200] = 1e-38
    _check_fp4_bit_exact(W)


def _weights(N, K, seed):
    return torch.from_numpy(inputs.weight_f32(inputs.rng(seed), N, K))


@pytest.mark.parametrize("M", [8, 16, 24, 48, 100, 200])
def test_fp4_linear_forward_every_path(M):
    """1-128 tokens (weight decoded into TMEM for tcgen05), above (dequant + GEMM)."""
    N, K, r, s = 256, 512, 16, 1.0
    g = inputs.rng(900 + M)
    W = _weights(N, K, 901 + M)
    X = inputs.normal_bf16(g, (M, K))
    L1, L2 = inputs.lora_factors(g, K, N, r)
    q = qlora.quantize_nf4_dq(W.cuda(), table="fp4")
    Y, T = qlora.linear_fwd(X.cuda(), q, L1.cuda(), L2.cuda(), s)
    torch.cuda.synchronize()
    assert qlora.last_device_error() == 0
    w_hat = nf4dq.dequantize(nf4dq.quantize_nf4_dq(W.numpy(), FP4))
    Y_ref, T_ref = qlora_linear.forward(bf16_to_np(X), w_hat, bf16_to_np(L1), bf16_to_np(L2), s)
    assert_close(bf16_to_np(Y), Y_ref, f"Y M={M}")
    assert_close(bf16_to_np(qlora.t_value(T)), T_ref, f"T M={M}")


def test_fp4_linear_backward():
    M, N, K, r, s = 300, 264, 320, 16, 0.5
    g = inputs.rng(950)
    W = _weights(N, K, 951)
    X = inputs.normal_bf16(g, (M, K))
    L1, L2 = inputs.lora_factors(g, K, N, r)
    dY = inputs.normal_bf16(g, (M, N))
    q = qlora.quantize_nf4_dq(W.cuda(), table="fp4")
    Y, T = qlora.linear_fwd(X.cuda(), q, L1.cuda(), L2.cuda(), s)
    dX, dL1, dL2 = qlora.linear_bwd(dY.cuda(), X.cuda(), T, q, L1.cuda(), L2.cuda(), s, grad_dtype=torch.float32)
    torch.cuda.synchronize()
    assert qlora.last_device_error() == 0
    w_hat = nf4dq.dequantize(nf4dq.quantize_nf4_dq(W.numpy(), FP4))
    dX_ref, dL1_ref, dL2_ref = qlora_linear.backward(bf16_to_np(dY), bf16_to_np(X), w_hat, bf16_to_np(L1),
                                                     bf16_to_np(L2), s)
    assert_close(bf16_to_np(dX), dX_ref, "dX")
    assert_close(dL1.cpu().numpy(), dL1_ref, "dL1")
    assert_close(dL2.cpu().numpy(), dL2_ref, "dL2")


def test_fp4_reconstruction_error_exceeds_nf4_on_gpu():
    """The comparison of §4 on the GPU's own outputs: N(0, 0.02^2) weights
    dequantized from each table, RMS error against the original."""
    W = inputs.device_normal((1024, 4096), 0.02, 77, "cuda")
    err = {}
    for t in ("nf4", "fp4"):
        wh = qlora.dequant(qlora.quantize_nf4_dq(W, table=t)).float()
        err[t] = float((wh - W).square().mean().sqrt())
    assert err["nf4"] < 0.95 * err["fp4"], err


def test_unknown_table_is_rejected():
    with pytest.raises(ValueError):
        qlora.quantize_nf4_dq(torch.zeros(4, 64, device="cuda"), table="int4")
