"""GPU parity of the QLoRA linear forward and backward against the float64
oracle, element by element, at sizes spanning several tiles with ragged
tails, plus special cases and sampled checks at a full LLaMA-7B layer size."""

import numpy as np
import pytest
import torch

from oracle import qlora_linear
from parity import assert_close, bf16_to_np, oracle_bwd, oracle_fwd, oracle_quant, oracle_w_hat
from synth import inputs, workloads

pytestmark = pytest.mark.gpu

qlora = pytest.importorskip("bit_nf4_quantized_02_b200")


def make_case(M, N, K, r, seed, zero_w=False, zero_l2=False):
    g = inputs.rng(seed)
    W = torch.from_numpy(inputs.weight_f32(g, N, K))
    if zero_w:
        W.zero_()
    X = inputs.normal_bf16(g, (M, K))
    L1, L2 = inputs.lora_factors(g, K, N, r)
    if zero_l2:
        L2.zero_()
    dY = inputs.normal_bf16(g, (M, N))
    return W, X, L1, L2, dY


def run_and_check(M, N, K, r, s, seed, grad_dtype=torch.bfloat16, recompute_T=False, **kw):
    W, X, L1, L2, dY = make_case(M, N, K, r, seed, **kw)
    q = qlora.quantize_nf4_dq(W.cuda())
    oq = oracle_quant(W)
    w_hat = oracle_w_hat(oq)
    # the stored format the linear reads is bit-identical to the oracle's
    assert np.array_equal(q.codes.cpu().numpy(), oq["packed"])
    Xd, L1d, L2d, dYd = X.cuda(), L1.cuda(), L2.cuda(), dY.cuda()
    Y, T = qlora.linear_fwd(Xd, q, L1d, L2d, s)
    dX, dL1, dL2 = qlora.linear_bwd(dYd, Xd, None if recompute_T else T, q, L1d, L2d, s, grad_dtype=grad_dtype)
    torch.cuda.synchronize()
    assert qlora.last_device_error() == 0
    Y_ref, T_ref = oracle_fwd(X, w_hat, L1, L2, s)
    dX_ref, dL1_ref, dL2_ref = oracle_bwd(dY, X, w_hat, L1, L2, s)
    assert_close(bf16_to_np(Y), Y_ref, "Y")
    assert_close(qlora.t_value(T).cpu().numpy(), T_ref, "T")
    assert_close(bf16_to_np(dX), dX_ref, "dX")
    assert dL1.dtype == grad_dtype and dL2.dtype == grad_dtype
    assert_close(dL1.float().cpu().numpy(), dL1_ref, "dL1")
    assert_close(dL2.float().cpu().numpy(), dL2_ref, "dL2")
    return Y, dX, dL1, dL2


@pytest.mark.parametrize("M,N,K,r", [
    (1, 8, 64, 8),
    (37, 136, 192, 8),
    (128, 1024, 1024, 8),       # the single-linear workload's shape
    (300, 264, 320, 64),        # ragged M and N, several tiles
    (129, 520, 576, 72),        # rank > 64 -> 128-wide rank tiles
    (256, 384, 256, 128),
    (200, 72, 128, 256),        # rank 256, N below one tile
    (513, 2056, 1088, 16),      # N spans 9 tiles of 256 with a tail of 8
])
def test_linear_parity(M, N, K, r):
    run_and_check(M, N, K, r, s=16.0 / r, seed=1000 + M + N + K + r)


def test_config1_exact_workload():
    wl = workloads.SINGLE_1024
    run_and_check(wl.M, 1024, 1024, wl.r, wl.s, wl.seed)


def test_fp32_gradients_and_recomputed_T():
    run_and_check(190, 264, 384, 64, 0.25, 77, grad_dtype=torch.float32, recompute_T=True)


def test_zero_l2_is_plain_gemm_against_torch():
    """With L2 = 0 the output is X W_hat^T: compare with torch's own GEMM on the
    library's dequantized weight (fp32 accumulation on both sides)."""
    M, N, K, r = 320, 512, 768, 16
    W, X, L1, L2, dY = make_case(M, N, K, r, 91, zero_l2=True)
    q = qlora.quantize_nf4_dq(W.cuda())
    Y, _ = qlora.linear_fwd(X.cuda(), q, L1.cuda(), L2.cuda(), 1.0)
    w_hat = qlora.dequant(q)
    ref = (X.cuda().float() @ w_hat.float().T)
    err = (Y.float() - ref).abs().max().item()
    assert err <= 1e-2 * ref.abs().max().item()


def test_zero_weight_is_pure_lora():
    M, N, K, r = 200, 136, 256, 8
    W, X, L1, L2, dY = make_case(M, N, K, r, 92, zero_w=True)
    q = qlora.quantize_nf4_dq(W.cuda())
    assert torch.all(q.codes == 0x77)
    Y, T = qlora.linear_fwd(X.cuda(), q, L1.cuda(), L2.cuda(), 2.0)
    ref = 2.0 * bf16_to_np(X).astype(np.float64) @ bf16_to_np(L1) @ bf16_to_np(L2)
    assert_close(bf16_to_np(Y), ref, "Y(pure LoRA)")


def test_no_tokens():
    N, K, r = 64, 128, 8
    W, X, L1, L2, dY = make_case(4, N, K, r, 93)
    q = qlora.quantize_nf4_dq(W.cuda())
    X0 = torch.empty(0, K, dtype=torch.bfloat16, device="cuda")
    Y, T = qlora.linear_fwd(X0, q, L1.cuda(), L2.cuda(), 1.0)
    assert Y.shape == (0, N)
    dY0 = torch.empty(0, N, dtype=torch.bfloat16, device="cuda")
    dX, dL1, dL2 = qlora.linear_bwd(dY0, X0, T, q, L1.cuda(), L2.cuda(), 1.0)
    assert torch.all(dL1 == 0) and torch.all(dL2 == 0)


def test_skip_dx():
    M, N, K, r = 64, 64, 128, 8
    W, X, L1, L2, dY = make_case(M, N, K, r, 94)
    q = qlora.quantize_nf4_dq(W.cuda())
    Y, T = qlora.linear_fwd(X.cuda(), q, L1.cuda(), L2.cuda(), 1.0)
    dX, dL1, dL2 = qlora.linear_bwd(dY.cuda(), X.cuda(), T, q, L1.cuda(), L2.cuda(), 1.0, need_dX=False)
    assert dX is None
    _, dL1_ref, dL2_ref = oracle_bwd(dY, X, oracle_w_hat(oracle_quant(W)), L1, L2, 1.0)
    assert_close(dL1.float().cpu().numpy(), dL1_ref, "dL1")
    assert_close(dL2.float().cpu().numpy(), dL2_ref, "dL2")


def test_error_statuses():
    from bit_nf4_quantized_02_b200 import _lib
    lib = _lib.load()
    N, K, r = 64, 128, 8
    W, X, L1, L2, dY = make_case(4, N, K, r, 95)
    q = qlora.quantize_nf4_dq(W.cuda())
    Xd, L1d, L2d = X.cuda(), L1.cuda(), L2.cuda()
    Y = torch.empty(4, N, dtype=torch.bfloat16, device="cuda")
    ws = torch.empty(lib.qlora_linear_fwd_workspace_size(4, N, K, r), dtype=torch.uint8, device="cuda")
    st = torch.cuda.current_stream().cuda_stream
    ok = lib.qlora_linear_fwd(Xd.data_ptr(), 4, q.as_struct(), L1d.data_ptr(), L2d.data_ptr(), r, 1.0, Y.data_ptr(),
                              None, ws.data_ptr(), ws.numel(), st)
    assert ok == _lib.QLORA_OK
    small = lib.qlora_linear_fwd(Xd.data_ptr(), 4, q.as_struct(), L1d.data_ptr(), L2d.data_ptr(), r, 1.0,
                                 Y.data_ptr(), None, ws.data_ptr(), ws.numel() - 1, st)
    assert small == _lib.QLORA_ERR_WORKSPACE
    mis = lib.qlora_linear_fwd(Xd.data_ptr() + 2, 4, q.as_struct(), L1d.data_ptr(), L2d.data_ptr(), r, 1.0,
                               Y.data_ptr(), None, ws.data_ptr(), ws.numel(), st)
    assert mis == _lib.QLORA_ERR_MISALIGNED
    torch.cuda.synchronize()
    assert qlora.last_device_error() == 0


@pytest.mark.slow
@pytest.mark.parametrize("lin", [workloads.LLAMA7B_LAYER.linears[0], workloads.LLAMA7B_LAYER.linears[4],
                                 workloads.LLAMA7B_LAYER.linears[6]], ids=lambda l: l.name)
def test_llama7b_linear_full_size_sampled(lin):
    """Full M = 8192 tokens at a LLaMA-7B linear's shape, in the launch
    configuration the benchmark times: Y and dX on 256 sampled token rows
    (rows are independent), T on the same rows, dL1 and dL2 in full."""
    wl = workloads.LLAMA7B_LAYER
    M, N, K, r, s = wl.M, lin.n_out, lin.k_in, wl.r, wl.s
    g = inputs.rng(wl.seed + N + K)
    W = torch.from_numpy(inputs.weight_f32(g, N, K))
    X = inputs.normal_bf16(g, (M, K))
    L1, L2 = inputs.lora_factors(g, K, N, r)
    dY = inputs.normal_bf16(g, (M, N))
    q = qlora.quantize_nf4_dq(W.cuda())
    Xd, L1d, L2d, dYd = X.cuda(), L1.cuda(), L2.cuda(), dY.cuda()
    Y, T = qlora.linear_fwd(Xd, q, L1d, L2d, s)
    dX, dL1, dL2 = qlora.linear_bwd(dYd, Xd, T, q, L1d, L2d, s)
    torch.cuda.synchronize()
    assert qlora.last_device_error() == 0
    w_hat = oracle_w_hat(oracle_quant(W))
    rows = np.sort(np.random.default_rng(0).choice(M, 256, replace=False))
    Xr, dYr = bf16_to_np(X)[rows], bf16_to_np(dY)[rows]
    Y_ref, T_ref = qlora_linear.forward_rows(Xr, w_hat, bf16_to_np(L1), bf16_to_np(L2), s)
    assert_close(bf16_to_np(Y)[rows], Y_ref, "Y[rows]")
    assert_close(qlora.t_value(T).cpu().numpy()[rows], T_ref, "T[rows]")
    dX_ref = qlora_linear.backward_dx_rows(dYr, w_hat, bf16_to_np(L1), bf16_to_np(L2), s)
    assert_close(bf16_to_np(dX)[rows], dX_ref, "dX[rows]")
    dL1_ref, dL2_ref = qlora_linear.adapter_grads(bf16_to_np(dY), bf16_to_np(X), bf16_to_np(L1), bf16_to_np(L2), s)
    assert_close(dL1.float().cpu().numpy(), dL1_ref, "dL1")
    assert_close(dL2.float().cpu().numpy(), dL2_ref, "dL2")
