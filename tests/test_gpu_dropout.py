"""GPU parity of the linear with LoRA dropout (QLoRA Appendix B.2) against the
oracle's forward_dropout / backward_dropout, on the same seeded inputs and
keep masks (the mask is an input, drawn by synth.inputs.dropout_mask)."""

import numpy as np
import pytest
import torch

from oracle import qlora_linear
from parity import assert_close, bf16_to_np, oracle_quant, oracle_w_hat, sample_idx
from synth import inputs, workloads

pytestmark = pytest.mark.gpu

qlora = pytest.importorskip("bit_nf4_quantized_02_b200")


def _case(M, N, K, r, seed, p, mask_kind="random"):
    g = inputs.rng(seed)
    W = torch.from_numpy(inputs.weight_f32(g, N, K))
    X = inputs.normal_bf16(g, (M, K))
    L1, L2 = inputs.lora_factors(g, K, N, r)
    dY = inputs.normal_bf16(g, (M, N))
    if mask_kind == "random":
        words = inputs.dropout_mask(g, M, K, p)
    else:
        keep = np.full((M, K), mask_kind == "keep")
        words = inputs.pack_mask(keep)
    return W, X, L1, L2, dY, words


def _run(W, X, L1, L2, dY, words, s, p, grad_dtype=torch.float32):
    q = qlora.quantize_nf4_dq(W.cuda())
    mask = torch.from_numpy(words.view(np.int32)).cuda()
    Xd, L1d, L2d, dYd = X.cuda(), L1.cuda(), L2.cuda(), dY.cuda()
    Xm = torch.empty_like(Xd)
    Y, T = qlora.linear_fwd(Xd, q, L1d, L2d, s, dropout_mask=mask, dropout_p=p, Xm=Xm)
    dX, dL1, dL2 = qlora.linear_bwd(dYd, Xd, T, q, L1d, L2d, s, grad_dtype=grad_dtype, dropout_mask=mask,
                                    dropout_p=p, Xm=Xm)
    # the backward also recomputes T and the masked input when none is saved
    _, dL1b, dL2b = qlora.linear_bwd(dYd, Xd, None, q, L1d, L2d, s, need_dX=False, grad_dtype=grad_dtype,
                                     dropout_mask=mask, dropout_p=p)
    torch.cuda.synchronize()
    assert qlora.last_device_error() == 0
    keep = torch.from_numpy(inputs.unpack_mask(words, X.shape[1])).cuda()
    assert torch.equal(Xm.view(torch.int16), torch.where(keep, Xd, torch.zeros_like(Xd)).view(torch.int16))
    return q, Y, T, dX, dL1, dL2, dL1b, dL2b


@pytest.mark.parametrize("shape", [(200, 192, 256, 16), (300, 264, 320, 64), (16, 128, 128, 8), (129, 512, 192, 32)])
@pytest.mark.parametrize("p", [0.1, 0.05])
def test_dropout_linear_small(shape, p):
    M, N, K, r = shape
    s = 16.0 / r
    W, X, L1, L2, dY, words = _case(M, N, K, r, 700 + M + N + K + int(100 * p), p)
    q, Y, T, dX, dL1, dL2, dL1b, dL2b = _run(W, X, L1, L2, dY, words, s, p)
    w_hat = oracle_w_hat(oracle_quant(W))
    keep = inputs.unpack_mask(words, K)
    Xn, L1n, L2n, dYn = map(bf16_to_np, (X, L1, L2, dY))
    Y_ref, T_ref = qlora_linear.forward_dropout(Xn, w_hat, L1n, L2n, s, keep, p)
    dX_ref, dL1_ref, dL2_ref = qlora_linear.backward_dropout(dYn, Xn, w_hat, L1n, L2n, s, keep, p)
    assert_close(bf16_to_np(Y), Y_ref, "Y")
    assert_close(bf16_to_np(qlora.t_value(T)), T_ref, "T")
    assert_close(bf16_to_np(dX), dX_ref, "dX")
    for name, got, ref in (("dL1", dL1, dL1_ref), ("dL2", dL2, dL2_ref), ("dL1 (T recomputed)", dL1b, dL1_ref),
                           ("dL2 (T recomputed)", dL2b, dL2_ref)):
        assert_close(got.float().cpu().numpy(), ref, name)


def test_dropout_keep_all_p0_matches_plain_linear():
    M, N, K, r, s = 256, 256, 256, 16, 1.0
    W, X, L1, L2, dY, words = _case(M, N, K, r, 811, 0.0, "keep")
    q, Y, T, dX, dL1, dL2, _, _ = _run(W, X, L1, L2, dY, words, s, 0.0)
    Xd, L1d, L2d, dYd = X.cuda(), L1.cuda(), L2.cuda(), dY.cuda()
    Y0, T0 = qlora.linear_fwd(Xd, q, L1d, L2d, s)
    dX0, dL10, dL20 = qlora.linear_bwd(dYd, Xd, T0, q, L1d, L2d, s, grad_dtype=torch.float32)
    torch.cuda.synchronize()
    # same forward kernels on the same operands (X * 1 = X): identical bits
    assert torch.equal(Y, Y0) and torch.equal(T, T0)
    torch.testing.assert_close(dL1, dL10, rtol=0, atol=0)
    torch.testing.assert_close(dL2, dL20, rtol=0, atol=0)
    # dX takes the masked-addend route: same values up to the final rounding order
    assert_close(bf16_to_np(dX), bf16_to_np(dX0).astype(np.float64), "dX vs plain")


def test_dropout_drop_all_leaves_the_base_path():
    M, N, K, r, s = 192, 128, 256, 16, 1.0
    W, X, L1, L2, dY, words = _case(M, N, K, r, 812, 0.1, "drop")
    q, Y, T, dX, dL1, dL2, _, _ = _run(W, X, L1, L2, dY, words, s, 0.1)
    assert torch.count_nonzero(T) == 0
    assert torch.count_nonzero(dL1) == 0 and torch.count_nonzero(dL2) == 0
    w_hat = oracle_w_hat(oracle_quant(W))
    assert_close(bf16_to_np(Y), bf16_to_np(X) @ w_hat.T.astype(np.float64), "Y (base only)")
    assert_close(bf16_to_np(dX), bf16_to_np(dY).astype(np.float64) @ w_hat, "dX (base only)")


def test_dropout_rejects_bad_arguments():
    M, N, K, r = 64, 64, 64, 8
    W, X, L1, L2, dY, words = _case(M, N, K, r, 813, 0.1)
    q = qlora.quantize_nf4_dq(W.cuda())
    mask = torch.from_numpy(words.view(np.int32)).cuda()
    with pytest.raises(RuntimeError):
        qlora.linear_fwd(X.cuda(), q, L1.cuda(), L2.cuda(), 1.0, dropout_mask=mask, dropout_p=1.0)
    with pytest.raises(ValueError):
        qlora.linear_fwd(X.cuda(), q, L1.cuda(), L2.cuda(), 1.0, dropout_mask=mask[:, :1].contiguous(), dropout_p=0.1)


@pytest.mark.slow
def test_dropout_llama7b_q_full_size_sampled():
    """LLaMA-7B q-shaped linear at 8192 tokens, p = 0.1: Y and dX on 256
    sampled rows (rows are independent), T on those rows, dL1 and dL2 in full."""
    wl = workloads.LLAMA7B_LAYER
    lin = wl.linears[0]
    M, N, K, r, s, p = wl.M, lin.n_out, lin.k_in, wl.r, wl.s, 0.1
    W, X, L1, L2, dY, words = _case(M, N, K, r, wl.seed + 77, p)
    q, Y, T, dX, dL1, dL2, _, _ = _run(W, X, L1, L2, dY, words, s, p, grad_dtype=torch.bfloat16)
    w_hat = oracle_w_hat(oracle_quant(W))
    keep = inputs.unpack_mask(words, K)
    Xn, L1n, L2n, dYn = map(bf16_to_np, (X, L1, L2, dY))
    rows = sample_idx(M, 256, 3)
    Y_ref, T_ref = qlora_linear.forward_dropout(Xn[rows], w_hat, L1n, L2n, s, keep[rows], p)
    assert_close(bf16_to_np(Y)[rows], Y_ref, "Y[rows]")
    assert_close(bf16_to_np(qlora.t_value(T))[rows], T_ref, "T[rows]")
    G_rows = s * (dYn[rows].astype(np.float64) @ L2n.T.astype(np.float64))
    dX_ref = dYn[rows].astype(np.float64) @ w_hat + (G_rows @ L1n.T.astype(np.float64)) * keep[rows] / (1 - p)
    assert_close(bf16_to_np(dX)[rows], dX_ref, "dX[rows]")
    Xd = qlora_linear.dropped(Xn, keep, p)
    G = s * (dYn.astype(np.float64) @ L2n.T.astype(np.float64))
    assert_close(dL1.float().cpu().numpy(), Xd.T @ G, "dL1")
    assert_close(dL2.float().cpu().numpy(), (s * (Xd @ L1n.astype(np.float64))).T @ dYn.astype(np.float64), "dL2")
