"""QLoRA linear layer, forward and backward, in float64 (oracle).

TEST INFRASTRUCTURE ONLY (see the package docstring).

Source: "QLoRA: Efficient Finetuning of Quantized LLMs"
(aiingo.vercel.app/paper/paper-2305-14314):
  §2 "Low-rank Adapters", Eq. 3:   Y = X W + s X L1 L2,  L1 in R^{h x r}, L2 in R^{r x o};
  §3 "QLoRA", Eq. 5:               Y = X doubleDequant(c1, c2, W) + X L1 L2;
  §3, paragraph after Eq. 6:       only the adapter gradients dE/dL_i are needed, not
                                   dE/dW; the gradient flows through the weight
                                   dequantized to BFloat16.

Readings: the scale s of Eq. 3 is kept in Eq. 5 (which prints it without s);
the frozen weight is stored as W_hat[N, K] (out features x in features,
row-major), i.e. the paper's W in R^{h x o} transposed, so the base product is
X @ W_hat.T.  The oracle takes the bfloat16 values of X, W_hat, L1, L2 and dY
(widened exactly to float64) and evaluates every product in float64 without
any intermediate rounding; GPU intermediates (a bfloat16 T, a bfloat16 Y) are
absorbed by the tolerance.
"""

from __future__ import annotations

import numpy as np


def _f64(a) -> np.ndarray:
    return np.asarray(a, dtype=np.float64)


def forward(X, W_hat, L1, L2, s: float):
    """Eq. 3 / Eq. 5 with the frozen weight already doubleDequant-ed.

    X [M, K], W_hat [N, K], L1 [K, r], L2 [r, N].  Returns (Y [M, N], T [M, r])
    where T = s X L1 is the adapter's down-projection saved for the backward.
    """
    X, W_hat, L1, L2 = map(_f64, (X, W_hat, L1, L2))
    T = s * (X @ L1)
    Y = X @ W_hat.T + T @ L2
    return Y, T


def backward(dY, X, W_hat, L1, L2, s: float):
    """Gradients of E with dE/dY = dY, for the adapter only (no dW).

    G   = s dY L2^T           [M, r]
    dX  = dY W_hat + G L1^T   [M, K]   (through the dequantized weight)
    dL2 = s (X L1)^T dY       [r, N]
    dL1 = X^T G               [K, r]
    """
    dY, X, W_hat, L1, L2 = map(_f64, (dY, X, W_hat, L1, L2))
    G = s * (dY @ L2.T)
    dX = dY @ W_hat + G @ L1.T
    dL2 = s * ((X @ L1).T @ dY)
    dL1 = X.T @ G
    return dX, dL1, dL2


def forward_rows(X_rows, W_hat, L1, L2, s: float):
    """Forward for a subset of token rows only (rows are independent)."""
    return forward(X_rows, W_hat, L1, L2, s)


def backward_dx_rows(dY_rows, W_hat, L1, L2, s: float):
    """dX for a subset of token rows only (rows are independent)."""
    dY_rows, W_hat, L1, L2 = map(_f64, (dY_rows, W_hat, L1, L2))
    G = s * (dY_rows @ L2.T)
    return dY_rows @ W_hat + G @ L1.T


def adapter_grads(dY, X, L1, L2, s: float):
    """(dL1, dL2) of ``backward`` alone; they do not involve the frozen weight."""
    dY, X, L1, L2 = map(_f64, (dY, X, L1, L2))
    G = s * (dY @ L2.T)
    dL2 = s * ((X @ L1).T @ dY)
    dL1 = X.T @ G
    return dL1, dL2


# --------------------------------------------------------------------------- LoRA dropout
# QLoRA Appendix B.2 trains with LoRA dropout (0.1 up to 13B, 0.05 at 33B and
# 65B).  The pages do not say where it acts; the reading taken is the usual
# LoRA one: on the adapter's input only,
#     Y = X W_hat^T + s (drop(X) L1) L2,   drop(X) = X * m / (1 - p),
# with m a 0/1 keep mask drawn once per step and passed in (it is an input,
# not drawn here).  The base product sees X unchanged.

def dropped(X, mask, p: float) -> np.ndarray:
    """drop(X) = X * m / (1 - p) in float64; mask is a 0/1 (or bool) array shaped like X."""
    return _f64(X) * _f64(mask) / (1.0 - p)


def forward_dropout(X, W_hat, L1, L2, s: float, mask, p: float):
    """Forward with LoRA dropout.  Returns (Y [M, N], T [M, r]) with T = s drop(X) L1."""
    X, W_hat, L1, L2 = map(_f64, (X, W_hat, L1, L2))
    T = s * (dropped(X, mask, p) @ L1)
    Y = X @ W_hat.T + T @ L2
    return Y, T


def backward_dropout(dY, X, W_hat, L1, L2, s: float, mask, p: float):
    """Adapter-only backward of ``forward_dropout`` (no dW).

    G   = s dY L2^T                          [M, r]
    dX  = dY W_hat + (G L1^T) * m / (1 - p)  [M, K]  (the mask gates only the adapter path)
    dL2 = T^T dY, T = s drop(X) L1           [r, N]
    dL1 = drop(X)^T G                        [K, r]
    """
    dY, X, W_hat, L1, L2 = map(_f64, (dY, X, W_hat, L1, L2))
    Xd = dropped(X, mask, p)
    G = s * (dY @ L2.T)
    dX = dY @ W_hat + (G @ L1.T) * _f64(mask) / (1.0 - p)
    dL2 = (s * (Xd @ L1)).T @ dY
    dL1 = Xd.T @ G
    return dX, dL1, dL2
