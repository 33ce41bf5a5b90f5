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


def assert_close(got, ref, name: str, rel_frob: float = REL_FROB, elem: float = ELEM_ABS):
    got = np.asarray(got, np.float64)
    ref = np.asarray(ref, np.float64)
    assert got.shape == ref.shape, (name, got.shape, ref.shape)
    err = got - ref
    nref = np.linalg.norm(ref)
    rf = np.linalg.norm(err) / max(nref, 1e-30)
    assert np.all(np.isfinite(got)), f"{name}: non-finite output"
    assert rf <= rel_frob or np.linalg.norm(err) <= 1e-30, f"{name}: relative Frobenius error {rf:.3e} > {rel_frob}"
    bad = np.abs(err) > elem * (np.abs(ref) + 1.0)
    assert not bad.any(), (f"{name}: {bad.sum()} elements beyond {elem}*(|ref|+1); worst at "
                           f"{np.unravel_index(np.argmax(np.abs(err) - elem * (np.abs(ref) + 1)), err.shape)}")
    return rf


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
