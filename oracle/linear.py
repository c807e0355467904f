"""Oracle for the QLoRA linear layer, forward and backward, in float64.
TEST INFRASTRUCTURE ONLY (see the package docstring).

Source: "QLoRA: Efficient Finetuning of Quantized LLMs" (intuitivepapers.ai),
§LoRA (Y = XW + s·X·L1·L2 with s = alpha/r) and §The QLoRA layer, end to end
(the forward/backward listing: dx = dy·Wᵀ + s·(dy·L2ᵀ)·L1ᵀ,
dL1 = s·xᵀ·(dy·L2ᵀ), dL2 = s·(x·L1)ᵀ·dy, no gradient for W).

Conventions of this library: the frozen weight is stored [N, K] (out x in),
so the page's W (h x o) is our W_hatᵀ; A = L1 is [K, r]; B = L2 is [r, N].
All inputs are bfloat16 bit patterns; everything is computed in float64 from
the same bits the GPU sees (including the same dequantised W_hat).
"""
from __future__ import annotations

import numpy as np

from .nf4 import bf16_to_f64


def forward(x_bits, w_hat_bits, a_bits, b_bits, s: float, rows=None) -> dict:
    """Y = X·W_hatᵀ + s·(X·A)·B.  ``rows`` selects a subset of token rows
    (for sampled checks on large shapes).  Returns float64 Y and T = X·A."""
    X = bf16_to_f64(x_bits)
    if rows is not None:
        X = X[rows]
    W = bf16_to_f64(w_hat_bits)
    A = bf16_to_f64(a_bits)
    B = bf16_to_f64(b_bits)
    T = X @ A
    Y = X @ W.T + s * (T @ B)
    return {"Y": Y, "T": T}


def backward(x_bits, dy_bits, w_hat_bits, a_bits, b_bits, s: float) -> dict:
    """dX = dY·W_hat + s·(dY·Bᵀ)·Aᵀ;  dA = s·Xᵀ·(dY·Bᵀ);  dB = s·(X·A)ᵀ·dY."""
    X = bf16_to_f64(x_bits)
    dY = bf16_to_f64(dy_bits)
    W = bf16_to_f64(w_hat_bits)
    A = bf16_to_f64(a_bits)
    B = bf16_to_f64(b_bits)
    U = dY @ B.T
    T = X @ A
    dX = dY @ W + s * (U @ A.T)
    dA = s * (X.T @ U)
    dB = s * (T.T @ dY)
    return {"dX": dX, "dA": dA, "dB": dB, "U": U, "T": T}


def adapter_grads(x_bits, dy_bits, a_bits, b_bits, s: float) -> dict:
    """dA = s·Xᵀ·(dY·Bᵀ) and dB = s·(X·A)ᵀ·dY without dX: the adapter gradients
    need no W_hat, so they stay cheap at shapes where dY·W_hat is not."""
    X = bf16_to_f64(x_bits)
    dY = bf16_to_f64(dy_bits)
    A = bf16_to_f64(a_bits)
    B = bf16_to_f64(b_bits)
    return {"dA": s * (X.T @ (dY @ B.T)), "dB": s * ((X @ A).T @ dY)}


def backward_dx_rows(rows, dy_bits, w_hat_bits, a_bits, b_bits, s: float) -> np.ndarray:
    """dX restricted to the given token rows (dX rows depend only on dY rows)."""
    dY = bf16_to_f64(dy_bits)[rows]
    W = bf16_to_f64(w_hat_bits)
    A = bf16_to_f64(a_bits)
    B = bf16_to_f64(b_bits)
    return dY @ W + s * ((dY @ B.T) @ A.T)


def flops(m: int, n: int, k: int, r: int) -> dict:
    """Algorithmic flop counts: forward 2MNK + 2Mr(K+N); backward 2MNK + 4Mr(K+N)
    (dY·Bᵀ, its product with Aᵀ, dA and dB; T is saved by the forward)."""
    return {"fwd": 2.0 * m * n * k + 2.0 * m * r * (k + n),
            "bwd": 2.0 * m * n * k + 4.0 * m * r * (k + n)}
