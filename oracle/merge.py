"""Oracle for merging a trained adapter into the quantised base weight and
requantising the result.  TEST INFRASTRUCTURE ONLY (see the package docstring).

Sources (web pages on QLoRA):
  [P3] "QLoRA: quantising the part you are not training" (addaly.com),
       §What it costs, item 3: the adapter was fitted against the quantised
       base; merging it into that base means requantising, and the
       requantisation adds an error of its own.
  [P2] "QLoRA: Efficient Finetuning of Quantized LLMs" (intuitivepapers.ai),
       §LoRA and §The QLoRA layer, end to end: the layer computes
       X·W_hatᵀ + s·(X·A)·B, so the weight the adapter adds is s·(A·B)ᵀ
       (this library stores W as [N, K], A as [K, r], B as [r, N]).

Readings taken where the pages are silent:
  * merged weight: W_eff[n, k] = W_hat[n, k] + s·sum_j A[k, j]·B[j, n], the
    exact value rounded once to float32 (round to nearest even), then stored
    as bfloat16 (round to nearest even) — bfloat16 being the type the
    quantiser takes its weights in.  Rounding twice differs from rounding the
    exact value straight to bfloat16 only when the float32 result lands on a
    bfloat16 midpoint; ``tests/test_oracle_merge.py`` pins such a case by hand;
  * s is a float32 (the type of the layer's scale);
  * requantisation is the quantiser itself (blockwise NF4 with double
    quantisation, ``oracle.nf4.quantize_nf4``) applied to W_eff.

Parity status: pinned (tests/test_oracle_merge.py): exact rationals on small
inputs and at hand-made rounding ties, the zero adapter (identity, and the
NF4 codes are a fixed point of dequantise-then-quantise), a rank-one adapter
(position and value of the single changed weight), and agreement with the
layer's forward oracle.
"""
from __future__ import annotations

from fractions import Fraction

import numpy as np

from .nf4 import (_round_fraction_to_f32, bf16_to_f64, dequantize_nf4, f32_to_bf16_rne,
                  quantize_nf4)

_F32 = np.float32
_F64 = np.float64
_U = 2.0 ** -53          # unit roundoff of float64


def _exact_f32(w: float, s: float, a_row: np.ndarray, b_col: np.ndarray) -> np.float32:
    """float32 of w + s·sum(a_row·b_col), from the exact value.

    Each term s·a·b is exact in float64: s has 24 significant bits, a and b 8
    each (bfloat16), so the product needs at most 40, and its exponent stays
    far inside float64's range.  The terms are then added exactly as integers
    over their common power-of-two denominator."""
    ratios = [w.as_integer_ratio()] + [(s * x * y).as_integer_ratio()
                                       for x, y in zip(a_row.tolist(), b_col.tolist())]
    den = max(d for _, d in ratios)                 # every denominator is a power of two
    num = sum(n * (den // d) for n, d in ratios)
    return _round_fraction_to_f32(Fraction(num, den))


def merged_weight(w_hat_bits: np.ndarray, a_bits: np.ndarray, b_bits: np.ndarray, s: float) -> np.ndarray:
    """W_eff as bfloat16 bits [N, K] (see the module docstring for the rounding).

    The sum is formed in float64.  Its error is at most
    (r + 4)·2^-53·(|w| + s·sum_j |A||B|) per element; where the float64 value
    lies that close to a float32 rounding boundary (a midpoint between two
    adjacent float32 values), the element is recomputed with exact rationals,
    so every element is the correctly rounded float32 of the exact value."""
    W = bf16_to_f64(w_hat_bits)
    A = bf16_to_f64(a_bits)
    B = bf16_to_f64(b_bits)
    n, k = W.shape
    r = A.shape[1]
    if A.shape[0] != k or B.shape != (r, n):
        raise ValueError("shapes: W [N,K], A [K,r], B [r,N]")
    s32 = _F64(_F32(s))
    delta = (A @ B).T                       # [N, K]: sum_j A[k, j]·B[j, n]
    m64 = W + s32 * delta
    bound = (r + 4) * _U * (np.abs(W) + s32 * (np.abs(A) @ np.abs(B)).T)
    m32 = m64.astype(_F32)
    up = np.nextafter(m32, _F32(np.inf)).astype(_F64)
    dn = np.nextafter(m32, _F32(-np.inf)).astype(_F64)
    c = m32.astype(_F64)
    near = (np.abs(m64 - (c + up) / 2) <= bound) | (np.abs(m64 - (c + dn) / 2) <= bound)
    for i, j in zip(*np.nonzero(near)):
        m32[i, j] = _exact_f32(float(W[i, j]), float(s32), A[j, :], B[:, i])
    return f32_to_bf16_rne(m32)


def merge_requantize(q: dict, a_bits: np.ndarray, b_bits: np.ndarray, s: float) -> dict:
    """Dequantise the stored weight ``q`` (oracle.nf4 format), add the adapter,
    requantise.  Returns the merged bfloat16 weight and the new stored weight."""
    w_hat = dequantize_nf4(q)
    merged = merged_weight(w_hat, a_bits, b_bits, s)
    return {"w_hat": w_hat, "merged": merged, "q": quantize_nf4(merged, q["levels"])}


def requant_error(merged_bits: np.ndarray, q_new: dict) -> dict:
    """Error the requantisation adds: W_eff against its own NF4 round trip."""
    W = bf16_to_f64(merged_bits)
    R = bf16_to_f64(dequantize_nf4(q_new))
    d = W - R
    return {"rel_fro": float(np.linalg.norm(d) / max(np.linalg.norm(W), 1e-300)),
            "max_abs": float(np.max(np.abs(d))) if d.size else 0.0}
