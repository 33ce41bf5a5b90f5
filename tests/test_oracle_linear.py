"""Pins of the oracle's QLoRA linear forward/backward: torch autograd in float64
(library), special cases, adjoint identities and finite differences.
"""

import numpy as np
import torch

from oracle import qlora_linear
from synth import inputs


def _case(seed, M=6, K=64, N=12, r=4):
    g = inputs.rng(seed)
    X = inputs.normal_f32(g, (M, K))
    W = inputs.normal_f32(g, (N, K), 0.02)
    L1 = inputs.normal_f32(g, (K, r), 1 / np.sqrt(K))
    L2 = inputs.normal_f32(g, (r, N), 0.5)
    dY = inputs.normal_f32(g, (M, N))
    return X, W, L1, L2, dY


def test_forward_backward_match_torch_autograd():
    X, W, L1, L2, dY = _case(31)
    s = 0.7
    Y, T = qlora_linear.forward(X, W, L1, L2, s)
    dX, dL1, dL2 = qlora_linear.backward(dY, X, W, L1, L2, s)
    tX = torch.tensor(X, dtype=torch.float64, requires_grad=True)
    tL1 = torch.tensor(L1, dtype=torch.float64, requires_grad=True)
    tL2 = torch.tensor(L2, dtype=torch.float64, requires_grad=True)
    tW = torch.tensor(W, dtype=torch.float64)                 # frozen: no gradient
    tY = torch.nn.functional.linear(tX, tW) + s * (tX @ tL1) @ tL2
    tY.backward(torch.tensor(dY, dtype=torch.float64))
    assert np.allclose(Y, tY.detach().numpy(), rtol=1e-13, atol=1e-13)
    assert np.allclose(T, s * (X.astype(np.float64) @ L1), rtol=1e-13, atol=1e-13)
    assert np.allclose(dX, tX.grad.numpy(), rtol=1e-12, atol=1e-12)
    assert np.allclose(dL1, tL1.grad.numpy(), rtol=1e-12, atol=1e-12)
    assert np.allclose(dL2, tL2.grad.numpy(), rtol=1e-12, atol=1e-12)


def test_zero_l2_is_a_plain_linear():
    X, W, L1, L2, _ = _case(32)
    Y, _ = qlora_linear.forward(X, W, L1, np.zeros_like(L2), 2.0)
    ref = torch.nn.functional.linear(torch.tensor(X, dtype=torch.float64), torch.tensor(W, dtype=torch.float64))
    assert np.allclose(Y, ref.numpy(), rtol=1e-13, atol=1e-13)


def test_zero_weight_is_pure_lora():
    X, W, L1, L2, dY = _case(33)
    s = 2.0
    Y, _ = qlora_linear.forward(X, np.zeros_like(W), L1, L2, s)
    ref = s * np.linalg.multi_dot([X.astype(np.float64), L1, L2])
    assert np.allclose(Y, ref, rtol=1e-13, atol=1e-13)
    dX, _, _ = qlora_linear.backward(dY, X, np.zeros_like(W), L1, L2, s)
    assert np.allclose(dX, s * np.linalg.multi_dot([dY.astype(np.float64), L2.T, L1.T]), rtol=1e-12, atol=1e-12)


def test_adjoint_identities():
    X, W, L1, L2, dY = _case(34, M=9, K=128, N=20, r=8)
    s = 0.25
    Y, T = qlora_linear.forward(X, W, L1, L2, s)
    dX, dL1, dL2 = qlora_linear.backward(dY, X, W, L1, L2, s)
    lora_out = T @ L2
    ip = lambda a, b: float(np.sum(np.asarray(a, np.float64) * np.asarray(b, np.float64)))
    assert np.isclose(ip(dX, X), ip(dY, Y), rtol=1e-12)
    assert np.isclose(ip(dL1, L1), ip(dY, lora_out), rtol=1e-12)
    assert np.isclose(ip(dL2, L2), ip(dY, lora_out), rtol=1e-12)


def test_finite_differences():
    X, W, L1, L2, dY = _case(35, M=2, K=64, N=4, r=2)
    s = 1.5
    X, W, L1, L2, dY = [a.astype(np.float64) for a in (X, W, L1, L2, dY)]
    E = lambda X_, L1_, L2_: float(np.sum(dY * qlora_linear.forward(X_, W, L1_, L2_, s)[0]))
    dX, dL1, dL2 = qlora_linear.backward(dY, X, W, L1, L2, s)
    h = 1e-6
    for arr, grad, which in ((X, dX, 0), (L1, dL1, 1), (L2, dL2, 2)):
        num = np.zeros_like(arr)
        for idx in np.ndindex(arr.shape):
            args_p = [X.copy(), L1.copy(), L2.copy()]
            args_m = [X.copy(), L1.copy(), L2.copy()]
            args_p[which][idx] += h
            args_m[which][idx] -= h
            num[idx] = (E(*args_p) - E(*args_m)) / (2 * h)
        assert np.allclose(num, grad, rtol=1e-6, atol=1e-8)


def test_adapter_grads_equal_backward():
    X, W, L1, L2, dY = _case(36)
    _, dL1, dL2 = qlora_linear.backward(dY, X, W, L1, L2, 0.3)
    a1, a2 = qlora_linear.adapter_grads(dY, X, L1, L2, 0.3)
    assert np.array_equal(a1, dL1) and np.array_equal(a2, dL2)
