"""Shared helpers of the GPU parity tests: run the oracle on the same seeded
inputs the CUDA path gets, and compare within the stated tolerances."""

from __future__ import annotations

import numpy as np
import torch

from oracle import nf4dq, qlora_linear

# Tolerance for outputs and gradients (float64 oracle on the dequantized
# weight): per-tensor relative Frobenius error and per-element bound.
REL_FROB = 1e-2
ELEM_ABS = 2e-2


def bf16_to_np(t: torch.Tensor) -> np.ndarray:
    return t.detach().to("cpu", torch.float32).numpy()


def assert_close(got, ref, name: str, rel_frob: float = REL_FROB, elem: float = ELEM_ABS, unit: float = 1.0):
    """Relative Frobenius error <= rel_frob and |err| <= elem * (|ref| + unit) everywhere.

    ``unit`` is 1 for tensors computed from the configs' N(0, 1)-scaled inputs.
    For a layer whose inputs carry another scale (deep in a stack), it is the
    scale of the output in units of those inputs (see ``pow2_unit``): the
    stated bound applied to the same computation with the inputs rescaled by
    a power of two, which every rounding on the path commutes with exactly.
    """
    got = np.asarray(got, np.float64)
    ref = np.asarray(ref, np.float64)
    assert got.shape == ref.shape, (name, got.shape, ref.shape)
    err = got - ref
    nref = np.linalg.norm(ref)
    rf = np.linalg.norm(err) / max(nref, 1e-30)
    assert np.all(np.isfinite(got)), f"{name}: non-finite output"
    assert rf <= rel_frob or np.linalg.norm(err) <= 1e-30, f"{name}: relative Frobenius error {rf:.3e} > {rel_frob}"
    bad = np.abs(err) > elem * (np.abs(ref) + unit)
    assert not bad.any(), (f"{name}: {bad.sum()} elements beyond {elem}*(|ref|+{unit:g}); worst at "
                           f"{np.unravel_index(np.argmax(np.abs(err) - elem * (np.abs(ref) + unit)), err.shape)}")
    return rf


def pow2_unit(x) -> float:
    """max(1, the power of two nearest the RMS of an input tensor): 1 for N(0, 1) data.

    Scaling an input of the linear by 2^-e scales its outputs by exactly 2^-e
    (bf16 and fp32 roundings commute with powers of two away from overflow
    and underflow), so a check in these units is the stated check on inputs
    of unit scale.
    """
    if isinstance(x, torch.Tensor):
        rms = float(x.detach().float().square().mean().sqrt())
    else:
        rms = float(np.sqrt(np.mean(np.asarray(x, np.float64) ** 2)))
    return max(1.0, 2.0 ** round(np.log2(rms))) if rms > 0 else 1.0


def oracle_quant(W_cpu: torch.Tensor) -> dict:
    """Oracle NF4+DQ of a CPU weight (fp32 or bf16 values)."""
    return nf4dq.quantize_nf4_dq(W_cpu.to(torch.float32).numpy())


def gpu_quant_to_np(q) -> dict:
    return {
        "packed": q.codes.cpu().numpy(),
        "c2_fp8": q.c2_fp8.cpu().numpy(),
        "c1": q.c1.cpu().numpy(),
        "mu": np.float32(q.c2_mean.cpu().numpy()[0]),
    }


def oracle_w_hat(oq: dict) -> np.ndarray:
    """The oracle's doubleDequant-ed weight (float32 values of bf16)."""
    return nf4dq.dequantize(oq)


def oracle_fwd(X, W_hat, L1, L2, s):
    return qlora_linear.forward(bf16_to_np(X), W_hat, bf16_to_np(L1), bf16_to_np(L2), s)


def oracle_bwd(dY, X, W_hat, L1, L2, s):
    return qlora_linear.backward(bf16_to_np(dY), bf16_to_np(X), W_hat, bf16_to_np(L1), bf16_to_np(L2), s)


def sample_idx(n: int, k: int, seed: int) -> np.ndarray:
    """Sorted sample of min(k, n) distinct indices of range(n)."""
    return np.sort(np.random.default_rng(seed).choice(n, min(k, n), replace=False))


def check_linear_sampled(W_np, X, dY, L1, L2, s, Y, T, dX, dL1, dL2, tag="", n=256, seed=0):
    """Parity of one linear at full size on sampled outputs.

    Y and dX are checked on a block of sampled token rows x sampled feature
    columns (each element is an independent dot product, so the oracle
    computes exactly those, from the rows or columns of the doubleDequant-ed
    weight that they need); T on the sampled rows; dL1 and dL2 in full.
    Arguments are the GPU's tensors (bf16 on any device) and the fp32 weight
    as a numpy array; None skips Y/T (or dX).
    """
    from oracle import nf4dq
    M, K = X.shape
    N = W_np.shape[0]
    ux, uy = pow2_unit(X), pow2_unit(dY)     # 1 for N(0, 1) inputs
    rows = sample_idx(M, n, seed)
    Xr = bf16_to_np(X[torch.as_tensor(rows, device=X.device)])
    L1n, L2n = bf16_to_np(L1), bf16_to_np(L2)
    if Y is not None:
        ycols = sample_idx(N, n, seed + 1)
        w_r = nf4dq.dequantize_rows(W_np, ycols)
        Y_ref, T_ref = qlora_linear.forward_rows(Xr, w_r, L1n, L2n[:, ycols], s)
        assert_close(bf16_to_np(Y)[rows][:, ycols], Y_ref, f"{tag}Y[rows, cols]", unit=ux)
        r = L1.shape[1]
        Tv = T[:, :r].float() + T[:, r:].float()
        assert_close(Tv.cpu().numpy()[rows], T_ref, f"{tag}T[rows]", unit=ux)
    dYn = bf16_to_np(dY)
    if dX is not None:
        xcols = sample_idx(K, n, seed + 2)
        w_c = nf4dq.dequantize_cols(W_np, xcols)
        dX_ref = qlora_linear.backward_dx_rows(dYn[rows], w_c, L1n[xcols], L2n, s)
        assert_close(bf16_to_np(dX)[rows][:, xcols], dX_ref, f"{tag}dX[rows, cols]", unit=uy)
    dL1_ref, dL2_ref = qlora_linear.adapter_grads(dYn, bf16_to_np(X), L1n, L2n, s)
    assert_close(dL1.float().cpu().numpy(), dL1_ref, f"{tag}dL1", unit=ux * uy)
    assert_close(dL2.float().cpu().numpy(), dL2_ref, f"{tag}dL2", unit=ux * uy)
