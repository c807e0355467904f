"""Oracle for the storage-format variants of the quantiser: other 4-bit code
books, other block sizes, and other treatments of the block constants.
TEST INFRASTRUCTURE ONLY (see the package docstring).

Sources (web pages on QLoRA):
  [P2] "QLoRA: Efficient Finetuning of Quantized LLMs" (intuitivepapers.ai):
       §Quantize in blocks (absmax quantisation with an int8 grid: the scale is
       127 over the block's absmax, codes are rounded), §NormalFloat (the
       uniform Int4 grid set against NF4), §Double quantization (constants in
       8 bits, groups of 256, mean subtracted), §It matches 16-bit finetuning
       (NF4 with double quantisation against two "4-bit float variants" and
       4-bit integers).
  [P1] "QLoRA Review: 4-Bit Finetuning for 65B Models on One GPU"
       (tildalice.io) §What Would Trip You Up in Practice: smaller blocks give
       better precision and more overhead, larger blocks the reverse.

Readings taken where the pages are silent:
  * Int4: the symmetric absmax integer grid, levels k/7 for k = -7..7 (the
    int8 recipe of §Quantize in blocks with 7 in place of 127; the level
    -8/7 completes the 16-entry table and is never the nearest to a value in
    [-1, 1]);
  * the two 4-bit float variants: the pages name no layout; we take the two
    sign + 3-bit layouts, E2M1 (exponent bias 1, one subnormal step: 0, 0.5,
    1, 1.5, 2, 3, 4, 6) and E3M0 (bias 3, no mantissa: 0, 0.25, ..., 16),
    each divided by its largest value so the block's absmax maps to +-1; their
    two zeros (+0, -0) both become the level +0, and the nearest-level rule
    with ties to the lower index only ever picks the first of the two;
  * every code book is used like NF4: x_hat = float32(w / absmax), nearest
    level of the float32 table, ties to the lower index;
  * block sizes 32, 64, 128 and 256 run along the flattened tensor like the
    64 of the main format; double-quantisation groups stay at 256 blocks;
  * block constants: kept as float32 ("none", 32 bits per block), the main
    format's E4M3 of the mean-centred constants ("e4m3"), or the int8 absmax
    grid of §Quantize in blocks applied to the mean-centred constants per
    group ("int8": S_g = float32(amax_g / 127), e = round-half-even of
    float32(dev / S_g), reconstruction fmaf(e, S_g, mu) as for E4M3).

Parity status: pinned (tests/test_oracle_formats.py): code-book values from
the bit-field definitions of the float layouts and the integer grid; brute
force nearest level; the NF4 / 64 / E4M3 special case equals oracle.nf4 bit for
bit; the storage figures the pages print; the block-size and code-book
orderings the pages state; the int8 reconstruction error bound.
"""
from __future__ import annotations

from fractions import Fraction

import numpy as np

from . import nf4

_F32 = np.float32
_F64 = np.float64

CODEBOOKS = ("nf4", "int4", "fp4_e2m1", "fp4_e3m0")
BLOCKS = (32, 64, 128, 256)
DQ_MODES = ("none", "e4m3", "int8")
GROUP = nf4.GROUP
INT8_MAX = 127.0


def _float4_values(exp_bits: int, man_bits: int, bias: int) -> np.ndarray:
    """All non-negative values of a sign + exponent + mantissa 4-bit float with
    subnormals at exponent field 0 (no infinities, no NaN)."""
    out = []
    for e in range(1 << exp_bits):
        for m in range(1 << man_bits):
            if e == 0:
                out.append(m / (1 << man_bits) * 2.0 ** (1 - bias))
            else:
                out.append((1 + m / (1 << man_bits)) * 2.0 ** (e - bias))
    return np.array(out, _F64)


def codebook(name: str) -> np.ndarray:
    """16 ascending float32 levels in [-1, 1] (see the module docstring)."""
    if name == "nf4":
        return nf4.nf4_levels()
    if name == "int4":
        return (np.arange(-8, 8, dtype=_F64) / 7.0).astype(_F32)
    if name == "fp4_e2m1":
        pos = _float4_values(2, 1, 1)
    elif name == "fp4_e3m0":
        pos = _float4_values(3, 0, 3)
    else:
        raise ValueError(name)
    pos = pos / pos.max()
    nz = pos[pos > 0]
    v = np.concatenate([-nz[::-1], [0.0, 0.0], nz])  # the layout's +0 and -0, both stored as +0
    return v.astype(_F32)


def quantize_codes(w_bits: np.ndarray, levels: np.ndarray, block: int) -> tuple[np.ndarray, np.ndarray]:
    """Per block of ``block`` consecutive weights of the flattened tensor:
    absmax c (float32), x_hat = float32(w / c), code = nearest level (ties to
    the lower index); an all-zero block codes every weight to the first zero
    level.  Returns (codes per element, absmax per block)."""
    w = nf4.bf16_to_f64(w_bits).astype(_F32).reshape(-1, block)
    if not np.all(np.isfinite(w)):
        raise ValueError("non-finite weight")
    c = np.max(np.abs(w), axis=1)
    safe = np.where(c == 0, _F32(1), c).astype(_F32)
    xhat = (w / safe[:, None]).astype(_F32)
    xhat[c == 0] = 0
    return nf4.nearest_level(xhat, levels).reshape(-1), c


def _int8_encode(x: np.ndarray) -> np.ndarray:
    """float32 -> nearest integer, ties to even, clamped to [-127, 127]."""
    return np.clip(np.rint(np.asarray(x, _F32).astype(_F64)), -INT8_MAX, INT8_MAX).astype(np.int8)


def double_quantize(c: np.ndarray, dq: str):
    """Block constants -> stored form.  Returns (consts, group scales, mean):
    'none'  -> (float32 absmax, empty, 0);
    'e4m3'  -> the main format's second quantisation (oracle.nf4);
    'int8'  -> int8 codes of the mean-centred constants, S_g = amax_g / 127."""
    c = np.asarray(c, _F32)
    if dq == "none":
        return c.copy(), np.zeros(0, _F32), _F32(0)
    if dq == "e4m3":
        return nf4.double_quantize(c)
    if dq != "int8":
        raise ValueError(dq)
    nb = c.size
    mu = nf4.fixed_order_mean(c)
    dev = (c - mu).astype(_F32)
    ng = -(-nb // GROUP)
    s = np.empty(ng, _F32)
    e = np.zeros(nb, np.int8)
    for g in range(ng):
        d = dev[g * GROUP:(g + 1) * GROUP]
        sg = _F32(np.max(np.abs(d)) / _F32(INT8_MAX))
        s[g] = sg
        if sg != 0:
            e[g * GROUP:(g + 1) * GROUP] = _int8_encode((d / sg).astype(_F32))
    return e, s, mu


def _fma_f32(a: np.ndarray, b: np.ndarray, c: np.float32) -> np.ndarray:
    """float32(a·b + c) with one rounding, for float32 a, b with a·b exact in
    float64 (|a| has at most 8 significant bits here)."""
    p = np.asarray(a, _F64) * np.asarray(b, _F64)
    m = _F64(c)
    tot = p + m
    bb = tot - p
    err = (p - (tot - bb)) + (m - bb)
    out = tot.astype(_F32)
    for i in np.nonzero(err != 0)[0]:
        out[i] = nf4._round_fraction_to_f32(Fraction(float(p[i])) + Fraction(float(m)))
    return out


def reconstruct(consts, s: np.ndarray, mu: np.float32, dq: str, nb: int) -> np.ndarray:
    """Block constants the dequantiser uses (float32)."""
    if dq == "none":
        return np.asarray(consts, _F32)
    if dq == "e4m3":
        return nf4.reconstruct_c2(consts, s, mu)
    sg = np.repeat(np.asarray(s, _F32), GROUP)[:nb]
    return _fma_f32(np.asarray(consts, np.int8).astype(_F64), sg, mu)


def dequantize(codes: np.ndarray, c_hat: np.ndarray, levels: np.ndarray, block: int, n: int, k: int) -> np.ndarray:
    """w_hat = bf16(float32(level[code] · c_hat_b)), bfloat16 bits [n, k]."""
    q = np.asarray(levels, _F32).astype(_F64)
    prod = (q[codes].reshape(-1, block) * np.asarray(c_hat, _F64)[:, None]).astype(_F32)
    return nf4.f32_to_bf16_rne(prod).reshape(n, k)


def quantize(w_bits: np.ndarray, cb: str, block: int, dq: str) -> dict:
    """W [N, K] bfloat16 bits -> stored weight of the given format."""
    n, k = w_bits.shape
    if (n * k) % block:
        raise ValueError("N*K must be a multiple of the block size")
    lv = codebook(cb)
    codes, c = quantize_codes(w_bits, lv, block)
    consts, s, mu = double_quantize(c, dq)
    return {"N": n, "K": k, "codebook": cb, "block": block, "dq": dq, "levels": lv,
            "codes": nf4.pack_nibbles(codes), "consts": consts, "c1": s, "mean": mu, "absmax": c}


def dequantize_q(q: dict) -> np.ndarray:
    codes = nf4.unpack_nibbles(q["codes"])
    nb = codes.size // q["block"]
    c_hat = reconstruct(q["consts"], q["c1"], q["mean"], q["dq"], nb)
    return dequantize(codes, c_hat, q["levels"], q["block"], q["N"], q["K"])


def storage_bits_per_weight(block: int, dq: str, n: int, k: int) -> float:
    """Stored bits per weight: 4 for the code, plus the block constants
    (32 bits per block, or 8 per block + 32 per group of 256 blocks + the
    32-bit mean)."""
    nb = n * k // block
    if dq == "none":
        bits = 4 * n * k + 32 * nb
    else:
        bits = 4 * n * k + 8 * nb + 32 * (-(-nb // GROUP)) + 32
    return bits / (n * k)


def error_stats(w_bits: np.ndarray, w_hat_bits: np.ndarray) -> dict:
    """Quantisation error of a round trip: relative Frobenius error, largest
    and mean absolute error."""
    w = nf4.bf16_to_f64(w_bits)
    d = w - nf4.bf16_to_f64(w_hat_bits)
    return {"rel_fro": float(np.linalg.norm(d) / max(np.linalg.norm(w), 1e-300)),
            "max_abs": float(np.max(np.abs(d))), "mean_abs": float(np.mean(np.abs(d)))}
