"""Pins of the oracle's LoRA-dropout forward and backward (QLoRA Appendix B.2:
LoRA dropout in training; read as dropout on the adapter input).

Each pin is fixed by something other than the oracle's own formula: the
no-dropout oracle (p = 0 with an all-keep mask, and the dropout-free base path
with an all-drop mask), central finite differences of the forward, and the
mask format's round trip and keep rate."""

import numpy as np
import pytest

from oracle import qlora_linear as ql
from synth import inputs


def _small(seed, M=6, K=64, N=5, r=3):
    g = np.random.default_rng(seed)
    X = g.standard_normal((M, K))
    W = g.standard_normal((N, K)) * 0.1
    L1 = g.standard_normal((K, r)) * 0.2
    L2 = g.standard_normal((r, N)) * 0.2
    dY = g.standard_normal((M, N))
    return X, W, L1, L2, dY


def test_keep_all_with_p0_is_the_plain_linear():
    X, W, L1, L2, dY = _small(1)
    keep = np.ones(X.shape, dtype=bool)
    Y0, T0 = ql.forward(X, W, L1, L2, 0.7)
    Y1, T1 = ql.forward_dropout(X, W, L1, L2, 0.7, keep, 0.0)
    np.testing.assert_array_equal(Y1, Y0)
    np.testing.assert_array_equal(T1, T0)
    g0 = ql.backward(dY, X, W, L1, L2, 0.7)
    g1 = ql.backward_dropout(dY, X, W, L1, L2, 0.7, keep, 0.0)
    for a, b in zip(g1, g0):
        np.testing.assert_allclose(a, b, rtol=1e-14, atol=1e-14)


def test_drop_all_leaves_the_base_product():
    X, W, L1, L2, dY = _small(2)
    drop = np.zeros(X.shape, dtype=bool)
    Y, T = ql.forward_dropout(X, W, L1, L2, 0.7, drop, 0.1)
    np.testing.assert_array_equal(T, 0.0)
    np.testing.assert_allclose(Y, X @ W.T, rtol=1e-14)
    dX, dL1, dL2 = ql.backward_dropout(dY, X, W, L1, L2, 0.7, drop, 0.1)
    np.testing.assert_allclose(dX, dY @ W, rtol=1e-14)
    np.testing.assert_array_equal(dL1, 0.0)
    np.testing.assert_array_equal(dL2, 0.0)


@pytest.mark.parametrize("p", [0.1, 0.5])
def test_backward_matches_finite_differences(p):
    """E = sum(Y * dY) with a fixed mask: dE/dX, dE/dL1, dE/dL2 by central
    differences of the forward against the oracle's backward."""
    X, W, L1, L2, dY = _small(3 + int(10 * p))
    keep = np.random.default_rng(9).random(X.shape) >= p
    s, h = 0.6, 1e-6

    def E(X_, L1_, L2_):
        return float(np.sum(ql.forward_dropout(X_, W, L1_, L2_, s, keep, p)[0] * dY))

    dX, dL1, dL2 = ql.backward_dropout(dY, X, W, L1, L2, s, keep, p)
    for name, A, G in (("X", X, dX), ("L1", L1, dL1), ("L2", L2, dL2)):
        num = np.zeros_like(A)
        for idx in np.ndindex(A.shape):
            Ap, Am = A.copy(), A.copy()
            Ap[idx] += h
            Am[idx] -= h
            args_p = {"X": (Ap, L1, L2), "L1": (X, Ap, L2), "L2": (X, L1, Ap)}[name]
            args_m = {"X": (Am, L1, L2), "L1": (X, Am, L2), "L2": (X, L1, Am)}[name]
            num[idx] = (E(*args_p) - E(*args_m)) / (2 * h)
        np.testing.assert_allclose(G, num, rtol=1e-6, atol=1e-7, err_msg=name)


def test_mask_pack_round_trip_and_keep_rate():
    g = inputs.rng(5)
    words = inputs.dropout_mask(g, 64, 4096, 0.1)
    assert words.shape == (64, 128) and words.dtype == np.uint32
    keep = inputs.unpack_mask(words, 4096)
    np.testing.assert_array_equal(inputs.pack_mask(keep), words)
    # element (i, 32w + b) is bit b of word w
    i, w, b = 3, 17, 29
    assert keep[i, 32 * w + b] == bool((words[i, w] >> b) & 1)
    rate = keep.mean()
    assert abs(rate - 0.9) < 4 * np.sqrt(0.09 / keep.size)
