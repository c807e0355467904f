"""Pins for the oracle's blockwise quantiser, double quantisation, scalar
formats and storage accounting.

Pages: "QLoRA: Efficient Finetuning of Quantized LLMs" (intuitivepapers.ai)
§Quantize in blocks, §NormalFloat, §Double quantization, §The QLoRA layer,
end to end; "QLoRA and NF4" (addaly.com); "QLoRA Review" (tildalice.io).
"""
import math
import os
from fractions import Fraction

import numpy as np
import pytest
import torch

from bit_nf4_quantised_codebook_b200.inputs import to_bf16_bits, weight_bf16
from oracle import nf4

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")
LV = nf4.nf4_levels()


# ---------------------------------------------------------------- scalar formats
def test_bf16_rne_matches_torch():
    rng = np.random.default_rng(1)
    x = np.concatenate([
        rng.standard_normal(200000).astype(np.float32) * 10.0 ** rng.integers(-30, 30, 200000),
        np.array([0.0, -0.0, 1.0, 1.00390625, 1.0078125, 1.01171875, 3.4e38, -3.4e38, 1e-40], np.float32),
    ]).astype(np.float32)
    ref = torch.from_numpy(x).to(torch.bfloat16).view(torch.int16).numpy().view(np.uint16)
    assert np.array_equal(nf4.f32_to_bf16_rne(x), ref)


def test_bf16_ties_to_even():
    # 1 + 2^-8 sits halfway between bf16 1.0 and 1.0078125: goes to the even mantissa (1.0)
    assert nf4.f32_to_bf16_rne(np.array([1.00390625], np.float32))[0] == 0x3F80
    # 1 + 3*2^-8 sits halfway between 1.0078125 (odd) and 1.015625 (even)
    assert nf4.f32_to_bf16_rne(np.array([1.01171875], np.float32))[0] == 0x3F82


def test_e4m3_decode_known_values():
    d = nf4.e4m3_decode(np.array([0x00, 0x01, 0x07, 0x08, 0x38, 0x39, 0x7E, 0x80, 0xB8, 0xFE], np.uint8))
    want = [0.0, 2.0 ** -9, 7 * 2.0 ** -9, 2.0 ** -6, 1.0, 1.125, 448.0, -0.0, -1.0, -448.0]
    assert list(d) == want
    assert np.isnan(nf4.e4m3_decode(np.array([0x7F, 0xFF], np.uint8))).all()


def test_e4m3_roundtrip_all_codes():
    codes = np.array([c for c in range(256) if c not in (0x7F, 0xFF)], np.uint8)
    vals = nf4.e4m3_decode(codes).astype(np.float32)
    assert np.array_equal(nf4.e4m3_encode(vals), codes)


def test_e4m3_ties_and_saturation():
    enc = lambda v: int(nf4.e4m3_encode(np.array([v], np.float32))[0])
    assert enc(1.0625) == 0x38      # halfway 1.0 (even) / 1.125 (odd)
    assert enc(1.1875) == 0x3A      # halfway 1.125 (odd) / 1.25 (even)
    assert enc(1.0625 + 1e-6) == 0x39
    assert enc(460.0) == 0x7E and enc(1e9) == 0x7E and enc(-1e9) == 0xFE
    assert enc(2.0 ** -10) == 0x00  # halfway 0 / 2^-9 -> even (0)
    assert enc(3 * 2.0 ** -10) == 0x02


def test_e4m3_encode_matches_torch_in_range():
    rng = np.random.default_rng(2)
    x = (rng.standard_normal(100000) * 10.0 ** rng.uniform(-3, 2.5, 100000)).astype(np.float32)
    x = x[np.abs(x) <= 448]
    ref = torch.from_numpy(x).to(torch.float8_e4m3fn).view(torch.uint8).numpy()
    assert np.array_equal(nf4.e4m3_encode(x), ref)


# ---------------------------------------------------------------- quantiser
def test_quantiser_brute_force():
    w = weight_bf16(8, 256, 0.02, 7, outlier_frac=0.01)
    codes, c2 = nf4.quantize_codes(w, LV)
    wf = nf4.bf16_to_f64(w).reshape(-1, 64)
    assert np.array_equal(c2.astype(np.float64), np.abs(wf).max(axis=1))
    cf = codes.reshape(-1, 64)
    for b in range(wf.shape[0]):
        for j in range(64):
            # x_hat is the correctly rounded float32 of w / c2
            exact = Fraction(wf[b, j]) / Fraction(float(c2[b]))
            xh = np.float32(float(exact))
            assert abs(Fraction(float(xh)) - exact) <= abs(Fraction(float(np.nextafter(xh, np.float32(2)))) - exact)
            q = [abs(Fraction(float(xh)) - Fraction(float(v))) for v in LV]
            best = min(q)
            assert cf[b, j] == q.index(best)


def test_zero_block_and_block_max():
    w = np.zeros((2, 128), np.float32)
    w[1, 64:] = np.linspace(-0.5, 0.25, 64)
    bits = to_bf16_bits(w)
    codes, c2 = nf4.quantize_codes(bits, LV)
    assert c2[0] == 0 and c2[1] == 0 and np.all(codes[:128] == 7)
    blk = codes.reshape(-1, 64)[3]
    assert blk[0] == 0                   # -0.5 is the block max in magnitude -> level -1
    assert blk[-1] != 15                 # 0.25 is not the block's absmax
    q = nf4.quantize_nf4(bits)
    deq = nf4.bf16_to_f64(nf4.dequantize_nf4(q))
    assert np.all(deq[0] == 0) and np.all(deq[1, :64] == 0)     # exact zero, [P2] §NormalFloat


def test_positive_block_max_maps_to_top_level():
    w = np.full((1, 64), 0.01, np.float32)
    w[0, 5] = 0.3
    codes, _ = nf4.quantize_codes(to_bf16_bits(w), LV)
    assert codes[5] == 15


def test_roundtrip_of_level_multiples():
    c = 0.0625                           # power of two: q_i * c is exact in float32
    rng = np.random.default_rng(3)
    idx = rng.integers(0, 16, size=(4, 64)).astype(np.uint8)
    idx[:, 0] = 15                       # make c the absmax of every block
    w = LV[idx] * np.float32(c)
    bits = to_bf16_bits(w)
    codes, c2 = nf4.quantize_codes(bits, LV)
    assert np.all(c2 == np.float32(c))
    assert np.array_equal(codes, idx.reshape(-1))


def test_nibble_packing_order():
    codes = np.array([1, 2, 15, 0, 7, 8], np.uint8)
    p = nf4.pack_nibbles(codes)
    assert list(p) == [0x12, 0xF0, 0x78]
    assert np.array_equal(nf4.unpack_nibbles(p), codes)


# ---------------------------------------------------------------- double quantisation
def test_fixed_order_mean_vs_exact_sum():
    rng = np.random.default_rng(4)
    for nb in (1, 255, 256, 257, 1000, 70000):
        c = np.abs(rng.standard_normal(nb)).astype(np.float32) * np.float32(0.05)
        mu = nf4.fixed_order_mean(c)
        exact = math.fsum(float(v) for v in c) / nb
        assert abs(float(mu) - exact) <= float(np.spacing(np.float32(exact)))


def test_fixed_order_mean_is_order_defined():
    """The summation order is part of the definition.  Four blocks (one group,
    zero-padded to 256): the pairwise tree adds (c0 + c2) + (c1 + c3) and keeps
    both 2^-53 terms; a left-to-right sum loses each of them to round-to-even.
    The float64 sums then fall on either side of a float32 midpoint of the mean:
    tree -> 0.25 + 2^-25, left-to-right -> 0.25."""
    c = np.array([1.0, 2.0 ** -53, 2.0 ** -24, 2.0 ** -53], np.float32)
    seq = 0.0
    for v in c:
        seq += float(v)
    assert np.float32(seq / 4) == np.float32(0.25)
    assert nf4.fixed_order_mean(c) == np.float32(0.25 + 2.0 ** -25)


def test_double_quant_error_bound_and_format():
    w = weight_bf16(64, 4096, 0.02, 11, outlier_frac=0.001)
    q = nf4.quantize_nf4(w)
    c2 = q["absmax"]
    nb = c2.size
    assert q["c2q"].dtype == np.uint8 and q["c2q"].size == nb
    assert q["c1"].size == -(-nb // 256)
    c2h = nf4.reconstruct_c2(q["c2q"], q["c1"], q["mean"]).astype(np.float64)
    dev = np.abs(c2.astype(np.float64) - float(q["mean"]))
    sg = np.repeat(q["c1"].astype(np.float64), 256)[:nb]
    # E4M3 keeps 3 mantissa bits (relative half-gap 2^-4) and an absolute step of 2^-9 at the bottom
    bound = dev * 2.0 ** -4 + sg * 2.0 ** -10 + 2 * np.spacing(c2.astype(np.float32)).astype(np.float64)
    assert np.all(np.abs(c2h - c2) <= bound)
    # every group's largest deviation is encoded as +-448 (the scale is amax/448)
    e = nf4.e4m3_decode(q["c2q"])
    for g in range(q["c1"].size):
        assert np.max(np.abs(e[g * 256:(g + 1) * 256])) in (448.0, 416.0)


def test_reconstruct_is_single_rounding():
    rng = np.random.default_rng(6)
    e = rng.integers(0, 256, 3000).astype(np.uint8)
    e[(e & 0x7F) == 0x7F] = 0
    s = (np.abs(rng.standard_normal(12)) * 1e-4).astype(np.float32)
    for mu in (np.float32(0.05), np.float32(3.0e-3), np.float32(1e-9)):
        got = nf4.reconstruct_c2(e, s, mu)
        ev = nf4.e4m3_decode(e)
        sg = np.repeat(s, 256)[:e.size]
        for i in range(0, e.size, 7):
            exact = Fraction(float(ev[i])) * Fraction(float(sg[i])) + Fraction(float(mu))
            g = Fraction(float(got[i]))
            up = Fraction(float(np.nextafter(got[i], np.float32(np.inf))))
            dn = Fraction(float(np.nextafter(got[i], np.float32(-np.inf))))
            assert abs(g - exact) <= abs(up - exact) and abs(g - exact) <= abs(dn - exact)


def test_dequant_error_bound():
    w = weight_bf16(32, 1024, 0.02, 12, outlier_frac=0.002)
    q = nf4.quantize_nf4(w)
    wh = nf4.bf16_to_f64(nf4.dequantize_nf4(q))
    wf = nf4.bf16_to_f64(w)
    c2 = np.repeat(q["absmax"].astype(np.float64), 64).reshape(wf.shape)
    c2h = np.repeat(nf4.reconstruct_c2(q["c2q"], q["c1"], q["mean"]).astype(np.float64), 64).reshape(wf.shape)
    half_gap = np.max(np.diff(LV.astype(np.float64))) / 2      # largest half gap between levels
    assert abs(half_gap - (1 - 0.6961928906) / 2) < 1e-6
    bound = c2 * half_gap + np.abs(c2 - c2h) + np.abs(wh) * 2.0 ** -8 + 1e-30
    assert np.all(np.abs(wf - wh) <= bound)


def test_dequant_formula_elementwise():
    w = weight_bf16(4, 512, 0.02, 13)
    q = nf4.quantize_nf4(w)
    wh = nf4.dequantize_nf4(q).reshape(-1)
    codes = nf4.unpack_nibbles(q["codes"])
    c2h = nf4.reconstruct_c2(q["c2q"], q["c1"], q["mean"])
    for i in range(0, codes.size, 13):
        prod = np.float32(Fraction(float(LV[codes[i]])) * Fraction(float(c2h[i // 64])))  # exact -> f32 (one rounding)
        ref = torch.tensor([float(prod)], dtype=torch.float32).to(torch.bfloat16).view(torch.int16).item() & 0xFFFF
        assert wh[i] == ref


# ---------------------------------------------------------------- storage accounting
def _golden_figures():
    out = {}
    with open(os.path.join(GOLDEN, "storage_figures.txt")) as f:
        for ln in f:
            if ln.strip() and not ln.startswith("#"):
                name, val, tol, _src = ln.split()
                out[name] = (float(val), float(tol))
    return out


def test_storage_figures():
    g = _golden_figures()
    chk = lambda name, v: abs(v - g[name][0]) <= g[name][1] + 1e-12
    n = k = 4096
    per_param = lambda nn, kk, dq: nf4.storage_bytes(nn, kk, dq) * 8 / (nn * kk)
    assert chk("overhead_bits_no_dq", per_param(n, k, False) - 4)
    assert chk("bits_per_weight_no_dq", per_param(n, k, False))
    # the pages' overhead figure 8/64 + 32/(64*256); the stored mean adds 32 bits per tensor
    assert chk("overhead_bits_dq", per_param(n, k, True) - 4)
    assert chk("bits_per_weight_dq", per_param(n, k, True))
    assert chk("saving_bits", per_param(n, k, False) - per_param(n, k, True))
    assert chk("saving_65b_gb", (per_param(n, k, False) - per_param(n, k, True)) * 65e9 / 8 / 1e9)
    assert chk("layer4096_bf16_mb", n * k * 2 / 1e6)
    assert chk("layer4096_nf4dq_mb", nf4.storage_bytes(n, k) / 1e6)
    assert chk("layer4096_block_scales", n * k // 64)
    assert chk("layer4096_adapter_r64_thousands", (k * 64 + 64 * n) / 1e3)
    assert chk("layer4096_adapter_r64_mb", (k * 64 + 64 * n) * 2 / 1e6)
    bits = per_param(8192, 8192, True)
    assert chk("model8b_nf4_gb", 8e9 * bits / 8 / 1e9)
    assert chk("model70b_nf4_gb", 70e9 * bits / 8 / 1e9)
    assert chk("model70b_bf16_gb", 70e9 * 2 / 1e9)
    assert chk("model8b_bf16_gb", 8e9 * 2 / 1e9)


def test_quantize_output_sizes():
    w = weight_bf16(256, 11008, 0.02, 14)    # K = 172 blocks per row: groups straddle rows
    q = nf4.quantize_nf4(w)
    nb = 256 * 11008 // 64
    assert q["codes"].size == 256 * 11008 // 2
    assert q["c2q"].size == nb and q["c1"].size == -(-nb // 256)
    w2 = weight_bf16(3, 64 * 100, 0.02, 15)  # 300 blocks: last group partial
    q2 = nf4.quantize_nf4(w2)
    assert q2["c1"].size == 2
    d = nf4.dequantize_nf4(q2)
    assert d.shape == (3, 6400)


@pytest.mark.parametrize("n,k,frac,seed", [(40, 1536, 0.002, 31), (3, 11008, 0.001, 32), (1, 64, 0.0, 33)])
def test_block_subset_equals_whole_tensor(n, k, frac, seed):
    """The block-subset form gives, block for block, what the whole-tensor
    quantiser and dequantiser give (rows straddling groups, a partial last
    group, outliers, a single block)."""
    w = weight_bf16(n, k, 0.02, seed, frac)
    full = nf4.quantize_nf4(w)
    wh = nf4.dequantize_nf4(full).reshape(-1, 64)
    nb = n * k // 64
    rng = np.random.default_rng(seed)
    blocks = np.unique(np.concatenate([[0, nb - 1], rng.integers(0, nb, size=min(nb, 50))]))
    sub = nf4.quantize_nf4_blocks(w, blocks)
    assert np.array_equal(sub["codes"], full["codes"].reshape(-1, 32)[blocks])
    assert np.array_equal(sub["c2q"], full["c2q"][blocks])
    assert np.array_equal(sub["absmax"], full["absmax"][blocks])
    assert np.array_equal(sub["c1"], full["c1"]) and sub["mean"] == full["mean"]
    assert np.array_equal(nf4.dequantize_nf4_blocks(sub), wh[blocks])
