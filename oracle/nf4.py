"""Oracle for the NF4 storage format: code points, blockwise quantisation,
double quantisation and double dequantisation.  TEST INFRASTRUCTURE ONLY
(see the package docstring).

Sources (web pages on QLoRA):
  [P2] "QLoRA: Efficient Finetuning of Quantized LLMs" (intuitivepapers.ai)
       §Quantize in blocks, §NormalFloat, §Double quantization,
       §The QLoRA layer, end to end.
  [P1] "QLoRA Review: 4-Bit Finetuning for 65B Models on One GPU"
       (tildalice.io) §What QLoRA Actually Does.
  [P5] "4-bit QLoRA" glossary (inferensys.com), double quantization entry.

Readings taken where the pages are silent or garbled:
  * code points: the offset recipe of [P2] §NormalFloat (the literal
    ``Q^-1(i/2^k)`` of [P1] is infinite at i = 0); computed in float64,
    normalised by the largest magnitude, then rounded to float32;
  * nearest level with ties going to the lower index;
  * zero block: every code is the exact-zero level (index 7);
  * nibble order: element 2j of the flat tensor in the high nibble of byte j,
    element 2j+1 in the low nibble;
  * the 8-bit float of the second quantisation is OCP FP8 E4M3FN, rounded to
    nearest-even and saturated at +-448 ([P2] "an 8-bit float", [P5] "FP8");
  * the mean subtracted before the second quantisation is one float32 value
    per tensor, summed in a fixed order (a float64 pairwise tree within each
    group of 256 blocks, then a pairwise tree over the group sums);
  * a group is 256 consecutive blocks of the flat block index; the last group
    may be partial.
"""
from __future__ import annotations

from fractions import Fraction

import numpy as np
from scipy.special import ndtri

BLOCK = 64          # weights per absmax block, [P2] §Quantize in blocks
GROUP = 256         # block constants per second-level group, [P2] §Double quantization
E4M3_MAX = 448.0    # largest finite OCP E4M3FN value
OFFSET = 0.9677083  # tail offset of the code-point recipe, [P2] §NormalFloat

_F32 = np.float32
_F64 = np.float64


# ---------------------------------------------------------------------------
# scalar formats
# ---------------------------------------------------------------------------
def bf16_to_f64(bits: np.ndarray) -> np.ndarray:
    """bfloat16 bit patterns -> float64 (exact)."""
    return ((np.asarray(bits, np.uint16).astype(np.uint32) << 16).view(_F32)).astype(_F64)


def f32_to_bf16_rne(x: np.ndarray) -> np.ndarray:
    """float32 -> bfloat16 bits, round to nearest, ties to even (the definition:
    keep the upper 16 bits, add half of the dropped range, ties decided by the
    kept LSB).  NaN maps to the quiet NaN 0x7FC0."""
    x = np.ascontiguousarray(x, dtype=_F32)
    u = x.view(np.uint32).astype(np.uint64)
    lsb = (u >> 16) & 1
    r = ((u + 0x7FFF + lsb) >> 16).astype(np.uint16)
    return np.where(np.isnan(x), np.uint16(0x7FC0), r)


def e4m3_decode(codes: np.ndarray) -> np.ndarray:
    """OCP FP8 E4M3FN code -> float64: bias 7, 3 mantissa bits, subnormals
    when the exponent field is 0, only S.1111.111 is NaN, no infinities."""
    c = np.asarray(codes, np.uint8).astype(np.int64)
    sign = np.where(c >> 7, -1.0, 1.0)
    e = (c >> 3) & 0xF
    m = c & 7
    mag = np.where(e == 0, m / 8.0 * 2.0 ** -6, (1.0 + m / 8.0) * np.exp2(e - 7.0))
    mag = np.where((e == 15) & (m == 7), np.nan, mag)
    return sign * mag


_E4M3_POS = e4m3_decode(np.arange(127, dtype=np.uint8))  # codes 0..126, increasing


def e4m3_encode(x: np.ndarray) -> np.ndarray:
    """float32 -> OCP FP8 E4M3FN code: nearest representable value, ties to the
    even code (even mantissa), magnitudes beyond 448 saturate to 448."""
    x = np.asarray(x, dtype=_F32).astype(_F64)
    a = np.abs(x)
    j = np.searchsorted(_E4M3_POS, a, side="right") - 1       # v_j <= a
    j = np.clip(j, 0, 126)
    jn = np.minimum(j + 1, 126)
    lo = _E4M3_POS[j]
    hi = _E4M3_POS[jn]
    d_lo = a - lo
    d_hi = hi - a
    pick_hi = (d_hi < d_lo) | ((d_hi == d_lo) & (j % 2 == 1))
    code = np.where(pick_hi, jn, j)
    code = np.where(a >= E4M3_MAX, 126, code)
    sign = np.signbit(x).astype(np.int64) << 7
    return (code | sign).astype(np.uint8)


# ---------------------------------------------------------------------------
# NF4 code points ([P2] §NormalFloat)
# ---------------------------------------------------------------------------
def nf4_levels_f64() -> np.ndarray:
    """The 16 NormalFloat-4 levels in float64, before rounding.

    Eight positive levels are normal quantiles at probabilities evenly spaced
    from OFFSET down towards 1/2 (nine points, the last one, 1/2, dropped);
    seven negative levels mirror quantiles at eight points spaced the same way
    (the last dropped); one exact zero.  Sorted, then divided by the largest
    magnitude so the ends are exactly -1 and +1.  Quantiles from
    ``scipy.special.ndtri`` (Cephes)."""
    p_pos = np.linspace(OFFSET, 0.5, 9)[:8]
    p_neg = np.linspace(OFFSET, 0.5, 8)[:7]
    pos = ndtri(p_pos)
    neg = -ndtri(p_neg)
    v = np.sort(np.concatenate([neg, np.zeros(1), pos]))
    return v / np.max(np.abs(v))


def nf4_levels() -> np.ndarray:
    """float32 NF4 table, index 0 = -1, index 7 = 0, index 15 = +1."""
    return nf4_levels_f64().astype(_F32)


def nf4_midpoints(levels: np.ndarray) -> np.ndarray:
    """Exact float64 midpoints between adjacent float32 levels."""
    q = np.asarray(levels, _F32).astype(_F64)
    return (q[:-1] + q[1:]) / 2.0


def nf4_thresholds(levels: np.ndarray) -> np.ndarray:
    """float32 decision thresholds t_i = the smallest float32 strictly above
    midpoint i, so that ``code = #{i : x >= t_i}`` is the nearest level with
    ties to the lower index.  (Needed only to check the library's table.)"""
    m = nf4_midpoints(levels)
    t = m.astype(_F32)
    up = np.nextafter(t, _F32(np.inf))
    return np.where(t.astype(_F64) <= m, up, t).astype(_F32)


def nearest_level(xhat: np.ndarray, levels: np.ndarray) -> np.ndarray:
    """Index of the nearest level (|x - q_i| in float64), ties to the lower
    index ([P1] §What QLoRA Actually Does: "assigns each weight to the nearest
    quantile"; tie rule is a reading).  Processes in chunks to bound memory."""
    q = np.asarray(levels, _F32).astype(_F64)
    x = np.asarray(xhat, _F32).astype(_F64).reshape(-1)
    out = np.empty(x.size, np.uint8)
    step = 1 << 20
    for s in range(0, x.size, step):
        d = np.abs(x[s:s + step, None] - q[None, :])
        out[s:s + step] = np.argmin(d, axis=1)   # first minimum = lowest index
    return out.reshape(np.shape(xhat))


# ---------------------------------------------------------------------------
# blockwise quantisation ([P2] §Quantize in blocks, §NormalFloat)
# ---------------------------------------------------------------------------
def block_absmax(w_bits: np.ndarray) -> np.ndarray:
    """c2_b = max |w| over the 64 consecutive elements of flat block b (float32)."""
    w = bf16_to_f64(w_bits).astype(_F32).reshape(-1, BLOCK)
    return np.max(np.abs(w), axis=1)


def quantize_codes(w_bits: np.ndarray, levels: np.ndarray) -> tuple[np.ndarray, np.ndarray]:
    """Return (codes uint8 per element, absmax float32 per block).

    Each weight is divided by its block's absmax in float32 (IEEE division,
    round to nearest) and mapped to the nearest level.  A block whose absmax
    is 0 maps every element to the zero level (index 7)."""
    w = bf16_to_f64(w_bits).astype(_F32).reshape(-1, BLOCK)
    if not np.all(np.isfinite(w)):
        raise ValueError("non-finite weight")
    c2 = np.max(np.abs(w), axis=1)
    safe = np.where(c2 == 0, _F32(1), c2).astype(_F32)
    xhat = (w / safe[:, None]).astype(_F32)
    xhat[c2 == 0] = 0
    codes = nearest_level(xhat, levels).reshape(-1)
    return codes, c2


def pack_nibbles(codes: np.ndarray) -> np.ndarray:
    """Two 4-bit codes per byte: even element -> high nibble, odd -> low."""
    c = np.asarray(codes, np.uint8).reshape(-1, 2)
    return ((c[:, 0] << 4) | c[:, 1]).astype(np.uint8)


def unpack_nibbles(packed: np.ndarray) -> np.ndarray:
    p = np.asarray(packed, np.uint8).reshape(-1)
    out = np.empty(p.size * 2, np.uint8)
    out[0::2] = p >> 4
    out[1::2] = p & 0xF
    return out


# ---------------------------------------------------------------------------
# double quantisation ([P2] §Double quantization; [P5])
# ---------------------------------------------------------------------------
def _pairwise_tree(a: np.ndarray) -> np.ndarray:
    """Pairwise tree along the last axis (length a power of two): for
    h = n/2, n/4, ..., 1 every a[i] (i < h) becomes a[i] + a[i+h]."""
    a = a.copy()
    h = a.shape[-1] // 2
    while h >= 1:
        a[..., :h] = a[..., :h] + a[..., h:2 * h]
        h //= 2
    return a[..., 0]


def fixed_order_mean(c2: np.ndarray) -> np.float32:
    """Mean of the block constants in one fixed float64 summation order: a
    pairwise tree over each group of 256 blocks (the last group zero-padded),
    then the same kind of tree over the group sums (zero-padded to a power of
    two), then one float64 division by the block count rounded to float32.
    (The pages only say the mean is subtracted first; the order is this
    library's reading, chosen so the sum is deterministic and parallel.)"""
    c = np.asarray(c2, _F32).astype(_F64)
    nb = c.size
    ng = -(-nb // GROUP)
    padded = np.zeros(ng * GROUP, _F64)
    padded[:nb] = c
    group_sums = _pairwise_tree(padded.reshape(ng, GROUP))
    size = 1
    while size < ng:
        size *= 2
    a = np.zeros(size, _F64)
    a[:ng] = group_sums
    return _F32(_pairwise_tree(a) / nb)


def double_quantize(c2: np.ndarray) -> tuple[np.ndarray, np.ndarray, np.float32]:
    """Block constants -> (E4M3 codes per block, float32 scale per group, mean).

    The mean is subtracted first so a symmetric quantiser can be used; each
    group of 256 centred constants gets scale S_g = amax_g / 448 and each
    constant becomes E4M3(dev / S_g).  A group with amax 0 has S_g = 0 and all
    codes 0."""
    c = np.asarray(c2, _F32)
    nb = c.size
    mu = fixed_order_mean(c)
    dev = (c - mu).astype(_F32)
    ng = -(-nb // GROUP)
    s = np.empty(ng, _F32)
    e = np.empty(nb, np.uint8)
    for g in range(ng):
        d = dev[g * GROUP:(g + 1) * GROUP]
        amax = np.max(np.abs(d))
        sg = _F32(amax / _F32(E4M3_MAX))
        s[g] = sg
        if sg == 0:
            e[g * GROUP:(g + 1) * GROUP] = 0
        else:
            e[g * GROUP:(g + 1) * GROUP] = e4m3_encode((d / sg).astype(_F32))
    return e, s, mu


def _round_fraction_to_f32(v: Fraction) -> np.float32:
    """Correctly rounded (nearest-even) float32 of an exact rational."""
    r = _F32(float(v))
    for _ in range(2):
        up = np.nextafter(r, _F32(np.inf))
        dn = np.nextafter(r, _F32(-np.inf))
        mid_up = (Fraction(float(r)) + Fraction(float(up))) / 2
        mid_dn = (Fraction(float(r)) + Fraction(float(dn))) / 2
        if v > mid_up or (v == mid_up and (int(up.view(np.uint32)) & 1) == 0):
            r = up
        elif v < mid_dn or (v == mid_dn and (int(dn.view(np.uint32)) & 1) == 0):
            r = dn
        else:
            break
    return r


def reconstruct_c2(e: np.ndarray, s: np.ndarray, mu: np.float32, groups: np.ndarray | None = None) -> np.ndarray:
    """Inner dequant of [P2] §The QLoRA layer: c2_hat_b = e_b * S_g + mu,
    rounded once to float32 (the exact value, as a fused multiply-add gives).
    ``groups`` gives each entry of ``e`` its group (default: entry b is block b,
    in group b // 256)."""
    e64 = e4m3_decode(e)
    nb = e64.size
    if groups is None:
        sg = np.repeat(np.asarray(s, _F32).astype(_F64), GROUP)[:nb]
    else:
        sg = np.asarray(s, _F32).astype(_F64)[np.asarray(groups, np.int64)]
    p = e64 * sg                                # exact: <= 4 x 24 significant bits
    m = _F64(mu)
    tot = p + m
    bb = tot - p                                # TwoSum: tot + err == p + m exactly
    err = (p - (tot - bb)) + (m - bb)
    out = tot.astype(_F32)
    for i in np.nonzero(err != 0)[0]:
        out[i] = _round_fraction_to_f32(Fraction(float(p[i])) + Fraction(float(m)))
    return out


def dequantize(packed: np.ndarray, e: np.ndarray, s: np.ndarray, mu: np.float32,
               levels: np.ndarray, n: int, k: int) -> np.ndarray:
    """doubleDequant ([P2] §The QLoRA layer): recover each block constant
    from (e, S_g, mu), then w_hat = bf16(float32(q[code] * c2_hat)).
    Returns bfloat16 bits [n, k]."""
    codes = unpack_nibbles(packed)
    c2h = reconstruct_c2(e, s, mu).astype(_F64)
    q = np.asarray(levels, _F32).astype(_F64)
    prod = (q[codes].reshape(-1, BLOCK) * c2h[:, None]).astype(_F32)   # exact product, one rounding
    return f32_to_bf16_rne(prod).reshape(n, k)


# ---------------------------------------------------------------------------
# whole format
# ---------------------------------------------------------------------------
def quantize_nf4(w_bits: np.ndarray, levels: np.ndarray | None = None) -> dict:
    """W [N,K] bfloat16 bits -> packed NF4 + double-quantised constants."""
    n, k = w_bits.shape
    if (n * k) % BLOCK:
        raise ValueError("N*K must be a multiple of 64")
    lv = nf4_levels() if levels is None else levels
    codes, c2 = quantize_codes(w_bits, lv)
    e, s, mu = double_quantize(c2)
    return {"N": n, "K": k, "codes": pack_nibbles(codes), "c2q": e, "c1": s,
            "mean": mu, "absmax": c2, "levels": lv}


def dequantize_nf4(q: dict) -> np.ndarray:
    return dequantize(q["codes"], q["c2q"], q["c1"], q["mean"], q["levels"], q["N"], q["K"])


def quantize_nf4_blocks(w_bits: np.ndarray, blocks, levels: np.ndarray | None = None) -> dict:
    """quantize_nf4 evaluated only for the flat blocks listed in ``blocks``, for
    tensors too large to quantise whole on the host in a test.  The steps are
    those of quantize_nf4: the absmax of every block (the mean and the group
    scales depend on all of them), the fixed-order mean, each group's scale
    S_g = amax_g|c2 - mu| / 448; then, for the listed blocks only, the codes
    (nearest level of w / c2) and the E4M3 constant of (c2 - mu) / S_g.
    Returns the listed blocks' packed codes [len, 32], E4M3 constants and
    absmax, every group scale, and the mean."""
    n, k = w_bits.shape
    if (n * k) % BLOCK:
        raise ValueError("N*K must be a multiple of 64")
    lv = nf4_levels() if levels is None else levels
    blocks = np.asarray(blocks, np.int64).reshape(-1)
    c2 = block_absmax(w_bits)
    mu = fixed_order_mean(c2)
    dev = (c2 - mu).astype(_F32)
    nb = c2.size
    ng = -(-nb // GROUP)
    amax = np.zeros(ng * GROUP, _F32)
    amax[:nb] = np.abs(dev)
    s = (amax.reshape(ng, GROUP).max(axis=1) / _F32(E4M3_MAX)).astype(_F32)
    sg = s[blocks // GROUP]
    safe = np.where(sg == 0, _F32(1), sg).astype(_F32)
    e = np.where(sg == 0, np.uint8(0), e4m3_encode((dev[blocks] / safe).astype(_F32))).astype(np.uint8)
    codes, c2_sel = quantize_codes(np.asarray(w_bits).reshape(-1, BLOCK)[blocks], lv)
    return {"N": n, "K": k, "blocks": blocks, "codes": pack_nibbles(codes).reshape(-1, BLOCK // 2),
            "c2q": e, "c1": s, "mean": mu, "absmax": c2_sel, "levels": lv}


def dequantize_nf4_blocks(qb: dict) -> np.ndarray:
    """doubleDequant of the blocks held by a quantize_nf4_blocks result:
    bfloat16 bits [len(blocks), 64]."""
    codes = unpack_nibbles(qb["codes"]).reshape(-1, BLOCK)
    c2h = reconstruct_c2(qb["c2q"], qb["c1"], qb["mean"], groups=qb["blocks"] // GROUP).astype(_F64)
    q = np.asarray(qb["levels"], _F32).astype(_F64)
    prod = (q[codes] * c2h[:, None]).astype(_F32)
    return f32_to_bf16_rne(prod).reshape(-1, BLOCK)


def storage_bytes(n: int, k: int, double_quant: bool = True) -> int:
    """Bytes of the stored weight: 4-bit codes, plus either one float32 per
    block, or one E4M3 per block + one float32 per 256-block group + the
    float32 mean."""
    nb = n * k // BLOCK
    if not double_quant:
        return n * k // 2 + 4 * nb
    return n * k // 2 + nb + 4 * (-(-nb // GROUP)) + 4
