"""GPU parity of the fused few-token forward (M <= 128 tokens: the weight is
decoded into tensor memory for the tensor core and never written to HBM as
bf16) against the float64 oracle, and its decoded weight against
doubleDequant's exact bf16 weight, bit for bit."""

import numpy as np
import pytest
import torch

from oracle import nf4dq, qlora_linear
from parity import assert_close, bf16_to_np, oracle_bwd, oracle_fwd, oracle_quant, oracle_w_hat
from synth import inputs, workloads

pytestmark = pytest.mark.gpu

qlora = pytest.importorskip("bit_nf4_quantized_02_b200")


def _case(M, N, K, r, seed):
    g = inputs.rng(seed)
    W = torch.from_numpy(inputs.weight_f32(g, N, K))
    X = inputs.normal_bf16(g, (M, K))
    L1, L2 = inputs.lora_factors(g, K, N, r)
    return W, X, L1, L2


@pytest.mark.parametrize("M", [1, 5, 8, 9, 16, 17, 32, 33, 64, 65, 100, 128])
@pytest.mark.parametrize("N,K,r", [(72, 320, 8), (520, 1088, 64), (1032, 2048, 136), (264, 64, 16), (136, 1280, 16)])
def test_few_token_forward_parity(M, N, K, r):
    W, X, L1, L2 = _case(M, N, K, r, 500 + M + N + K + r)
    s = 16.0 / r
    q = qlora.quantize_nf4_dq(W.cuda())
    Y, T = qlora.linear_fwd(X.cuda(), q, L1.cuda(), L2.cuda(), s)
    torch.cuda.synchronize()
    assert qlora.last_device_error() == 0
    w_hat = oracle_w_hat(oracle_quant(W))
    Y_ref, T_ref = oracle_fwd(X, w_hat, L1, L2, s)
    assert_close(bf16_to_np(Y), Y_ref, "Y")
    assert_close(qlora.t_value(T).cpu().numpy(), T_ref, "T")
    # with L2 = 0 the product matches torch's GEMM on qlora_dequant's output up to
    # fp32 accumulation and the decode's bf16 roundings (2^-7 relative per weight)
    Y0, _ = qlora.linear_fwd(X.cuda(), q, L1.cuda(), torch.zeros_like(L2).cuda(), s)
    ref0 = (X.cuda().float() @ qlora.dequant(q).float().T)
    assert (Y0.float() - ref0).abs().max().item() <= 1e-2 * (ref0.abs().max().item() + 1e-6) + 1e-6


def test_few_token_forward_then_backward():
    M, N, K, r = 16, 264, 512, 16
    W, X, L1, L2 = _case(M, N, K, r, 601)
    dY = inputs.normal_bf16(inputs.rng(602), (M, N))
    q = qlora.quantize_nf4_dq(W.cuda())
    Y, T = qlora.linear_fwd(X.cuda(), q, L1.cuda(), L2.cuda(), 1.0)
    dX, dL1, dL2 = qlora.linear_bwd(dY.cuda(), X.cuda(), T, q, L1.cuda(), L2.cuda(), 1.0)
    torch.cuda.synchronize()
    w_hat = oracle_w_hat(oracle_quant(W))
    dX_ref, dL1_ref, dL2_ref = oracle_bwd(dY, X, w_hat, L1, L2, 1.0)
    assert_close(bf16_to_np(dX), dX_ref, "dX")
    assert_close(dL1.float().cpu().numpy(), dL1_ref, "dL1")
    assert_close(dL2.float().cpu().numpy(), dL2_ref, "dL2")


def test_repeated_calls_reuse_workspace():
    """Back-to-back calls on one workspace (the zero region is re-cleared)."""
    M, N, K, r = 16, 520, 1024, 64
    W, X, L1, L2 = _case(M, N, K, r, 603)
    q = qlora.quantize_nf4_dq(W.cuda())
    outs = [qlora.linear_fwd(X.cuda(), q, L1.cuda(), L2.cuda(), 0.25)[0].float() for _ in range(3)]
    torch.cuda.synchronize()
    w_hat = oracle_w_hat(oracle_quant(W))
    Y_ref, _ = oracle_fwd(X, w_hat, L1, L2, 0.25)
    for Y in outs:
        assert_close(Y.cpu().numpy(), Y_ref, "Y(repeat)")


@pytest.mark.slow
@pytest.mark.parametrize("lin", [workloads.LLAMA65B_LAYER.linears[0], workloads.LLAMA65B_LAYER.linears[4],
                                 workloads.LLAMA65B_LAYER.linears[6]], ids=lambda l: l.name)
def test_llama65b_linear_16_tokens_sampled(lin):
    """The decode-sized workload at full LLaMA-65B linear sizes (16 tokens), in
    the launch configuration the benchmark times: Y checked on 128 sampled
    output features (the oracle dequantizes just those weight rows), all tokens."""
    wl = workloads.LLAMA65B_LAYER
    M, N, K, r, s = wl.extra["M_decode"], lin.n_out, lin.k_in, wl.r, wl.s
    Wd = inputs.device_normal((N, K), inputs.WEIGHT_STD, wl.seed + N + K, "cuda")
    g = inputs.rng(wl.seed + 3 * N + K)
    X = inputs.normal_bf16(g, (M, K))
    L1, L2 = inputs.lora_factors(g, K, N, r)
    q = qlora.quantize_nf4_dq(Wd)
    Y, T = qlora.linear_fwd(X.cuda(), q, L1.cuda(), L2.cuda(), s)
    torch.cuda.synchronize()
    assert qlora.last_device_error() == 0
    rows = np.sort(np.random.default_rng(1).choice(N, 128, replace=False))
    w_rows = nf4dq.dequantize_rows(Wd.cpu().numpy(), rows)
    Xf, L1f, L2f = bf16_to_np(X).astype(np.float64), bf16_to_np(L1).astype(np.float64), bf16_to_np(L2).astype(np.float64)
    # output features are independent: Y[:, rows] = X W_hat[rows]^T + T L2[:, rows]
    Y_ref, T_ref = qlora_linear.forward(Xf, w_rows, L1f, L2f[:, rows], s)
    assert_close(bf16_to_np(Y)[:, rows], Y_ref, "Y[:, sampled features]")
    assert_close(qlora.t_value(T).cpu().numpy(), T_ref, "T")


@pytest.mark.parametrize("K", [1088, 1280])
@pytest.mark.parametrize("M", [16, 48, 128])
@pytest.mark.parametrize("table", ["nf4", "fp4"])
def test_decoded_weight_is_double_dequant(M, table, K):
    """One-hot token rows pick single input features, so with L2 = 0 each
    output is one decoded weight (an fp32 sum of one product, exact in bf16):
    the few-token product decodes exactly doubleDequant's bf16 weight, bit for
    bit, zero codes included (K = 1088 ends on a stage of one 64-block, K =
    1280 on a whole stage)."""
    N, r = 264, 8
    g = inputs.rng(700 + M)
    W = torch.from_numpy(inputs.weight_f32(g, N, K))
    W[:, 5] = 0.0                                   # exact zeros inside nonzero blocks
    ks = np.sort(np.random.default_rng(M).choice(K, M, replace=False))
    ks[0] = 5
    X = torch.zeros(M, K, dtype=torch.bfloat16)
    X[np.arange(M), ks] = 1.0
    L1 = torch.zeros(K, r, dtype=torch.bfloat16)
    L2 = torch.zeros(r, N, dtype=torch.bfloat16)
    q = qlora.quantize_nf4_dq(W.cuda(), table=table)
    Y, _ = qlora.linear_fwd(X.cuda(), q, L1.cuda(), L2.cuda(), 1.0)
    exact = qlora.dequant(q)[:, torch.as_tensor(ks, device="cuda")].T     # [M, N] bf16
    torch.cuda.synchronize()
    assert qlora.last_device_error() == 0
    assert not Y[0].float().abs().any()
    assert torch.equal(Y.view(torch.int16), exact.contiguous().view(torch.int16))
