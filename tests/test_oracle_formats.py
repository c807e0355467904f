"""Pins for the oracle of the storage-format variants (other code books, block
sizes and treatments of the block constants).

Pages: "QLoRA: Efficient Finetuning of Quantized LLMs" (intuitivepapers.ai)
§Quantize in blocks, §NormalFloat, §Double quantization, §It matches 16-bit
finetuning; "QLoRA Review" (tildalice.io) §What Would Trip You Up in Practice.
"""
import os

import numpy as np
import pytest

from bit_nf4_quantised_codebook_b200.inputs import to_bf16_bits, weight_bf16
from oracle import formats as F
from oracle import nf4

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")


def _golden(name):
    for ln in open(os.path.join(GOLDEN, "storage_figures.txt")):
        if ln.strip() and not ln.startswith("#") and ln.split()[0] == name:
            return float(ln.split()[1]), float(ln.split()[2])
    raise KeyError(name)


def test_float4_code_books_are_the_layouts_values():
    # E2M1: 0, 0.5 (subnormal), 1, 1.5, 2, 3, 4, 6 (largest) -- the OCP 4-bit float
    e2m1 = np.array([0, 0.5, 1, 1.5, 2, 3, 4, 6]) / 6
    # E3M0 with bias 3: 0 and the powers of two 2^-2 .. 2^4
    e3m0 = np.array([0, 0.25, 0.5, 1, 2, 4, 8, 16]) / 16
    for name, pos in (("fp4_e2m1", e2m1), ("fp4_e3m0", e3m0)):
        lv = F.codebook(name)
        want = np.sort(np.concatenate([-pos, pos])).astype(np.float32)
        assert np.array_equal(lv, want), name
        assert lv[0] == -1 and lv[-1] == 1 and np.count_nonzero(lv == 0) == 2
        assert not np.signbit(lv[lv == 0]).any()


def test_int4_grid():
    lv = F.codebook("int4")
    assert np.array_equal(lv[1:], np.array([k / 7 for k in range(-7, 8)], np.float32))
    assert lv[0] < -1
    # absmax blocks put every x_hat in [-1, 1]: the extra level is never used, the rest are
    w = weight_bf16(64, 1024, 0.02, 3)
    codes, _ = F.quantize_codes(w, lv, 64)
    assert codes.min() == 1 and codes.max() == 15


@pytest.mark.parametrize("cb", F.CODEBOOKS)
def test_nearest_level_by_midpoints(cb):
    """code = #{i : x > m_i} with the exact midpoints (ties to the lower level):
    compared by level value, since the float code books hold 0 twice."""
    lv = F.codebook(cb)
    m = (lv[:-1].astype(np.float64) + lv[1:].astype(np.float64)) / 2
    rng = np.random.default_rng(7)
    x = np.concatenate([rng.uniform(-1, 1, 20000),
                        m[np.abs(m) <= 1],                                   # exact ties where representable
                        np.nextafter(m.astype(np.float32), np.float32(2)).astype(np.float64),
                        [0.0, -1.0, 1.0]]).astype(np.float32)
    x = x[np.abs(x) <= 1]
    w = np.zeros((x.size + (-x.size) % 64,), np.float32)
    w[:x.size] = x
    w[::64] = 1.0                                                          # absmax 1: x_hat == w
    codes, c = F.quantize_codes(to_bf16_bits(w)[None, :], lv, 64)
    xh = nf4.bf16_to_f64(to_bf16_bits(w))
    want = np.array([lv[np.count_nonzero(v > m)] for v in xh])
    assert np.array_equal(lv[codes], want.astype(np.float32))
    # of two equal levels only the first is ever used (ties go to the lower index)
    for i in range(15):
        if lv[i] == lv[i + 1]:
            assert not np.any(codes == i + 1)


def test_main_format_is_the_special_case():
    w = weight_bf16(40, 1600, 0.02, 11, 0.002)
    q = F.quantize(w, "nf4", 64, "e4m3")
    ref = nf4.quantize_nf4(w)
    assert np.array_equal(q["codes"], ref["codes"])
    assert np.array_equal(q["consts"], ref["c2q"])
    assert np.array_equal(q["c1"].view(np.uint32), ref["c1"].view(np.uint32))
    assert np.float32(q["mean"]) == np.float32(ref["mean"])
    assert np.array_equal(F.dequantize_q(q), nf4.dequantize_nf4(ref))


def test_storage_figures_the_pages_print():
    v, tol = _golden("bits_per_weight_dq")
    assert abs(F.storage_bits_per_weight(64, "e4m3", 4096, 4096) - v) <= tol
    assert abs(F.storage_bits_per_weight(64, "int8", 4096, 4096) - v) <= tol
    v, tol = _golden("bits_per_weight_no_dq")
    assert abs(F.storage_bits_per_weight(64, "none", 4096, 4096) - v) <= tol
    # 32 bits of constant per block: 1.0 / 0.5 / 0.25 / 0.125 extra bits per weight
    assert [F.storage_bits_per_weight(b, "none", 64, 4096) for b in F.BLOCKS] == [5.0, 4.5, 4.25, 4.125]


def test_smaller_blocks_are_more_precise_and_cost_more():
    w = weight_bf16(128, 4096, 0.02, 12, 0.001)
    for cb in ("nf4", "int4", "fp4_e2m1"):
        errs = [F.error_stats(w, F.dequantize_q(F.quantize(w, cb, b, "e4m3")))["rel_fro"] for b in F.BLOCKS]
        assert all(a < b for a, b in zip(errs, errs[1:])), (cb, errs)
    bits = [F.storage_bits_per_weight(b, "e4m3", 128, 4096) for b in F.BLOCKS]
    assert all(a > b for a, b in zip(bits, bits[1:]))


def test_nf4_rounds_normal_weights_best():
    w = weight_bf16(128, 4096, 0.02, 13)
    err = {cb: F.error_stats(w, F.dequantize_q(F.quantize(w, cb, 64, "none")))["rel_fro"] for cb in F.CODEBOOKS}
    assert err["nf4"] < min(err["int4"], err["fp4_e2m1"], err["fp4_e3m0"]), err


def test_int8_constants_error_bound():
    w = weight_bf16(64, 8192, 0.02, 14, 0.002)
    q = F.quantize(w, "nf4", 64, "int8")
    c = q["absmax"].astype(np.float64)
    nb = c.size
    ch = F.reconstruct(q["consts"], q["c1"], q["mean"], "int8", nb).astype(np.float64)
    sg = np.repeat(q["c1"].astype(np.float64), 256)[:nb]
    bound = sg * (0.5 + 127 * 2.0 ** -23) + 2.0 ** -23 * (np.abs(c) + abs(float(q["mean"])))
    assert np.all(np.abs(c - ch) <= bound)
    assert np.all(np.abs(q["consts"].astype(np.int64)) <= 127)
    # every group uses its full int8 range (the constant farthest from the mean maps to +-127)
    e = np.abs(q["consts"].astype(np.int64))
    assert all(e[g * 256:(g + 1) * 256].max() == 127 for g in range(-(-nb // 256)))


def test_int8_reconstruction_is_one_rounding():
    from fractions import Fraction
    w = weight_bf16(8, 8192, 0.02, 15)
    q = F.quantize(w, "nf4", 64, "int8")
    nb = q["consts"].size
    ch = F.reconstruct(q["consts"], q["c1"], q["mean"], "int8", nb)
    for b in range(0, nb, 7):
        exact = Fraction(int(q["consts"][b])) * Fraction(float(q["c1"][b // 256])) + Fraction(float(q["mean"]))
        got = Fraction(float(ch[b]))
        up = Fraction(float(np.nextafter(ch[b], np.float32(np.inf))))
        dn = Fraction(float(np.nextafter(ch[b], np.float32(-np.inf))))
        assert abs(got - exact) <= abs(up - exact) and abs(got - exact) <= abs(dn - exact)


def test_error_stats_hand_computed():
    """Values worked out by hand: a dropped square root, a missing division by
    the weight's norm or a maximum taken along one axis only fails one of them."""
    w = to_bf16_bits(np.array([[3.0, 4.0, 0.0, 0.0], [0.0, 0.0, 0.0, 0.0]]))
    zero = to_bf16_bits(np.zeros((2, 4)))
    # W_hat = 0: the error is W itself, |W| = 5
    assert F.error_stats(w, zero) == {"rel_fro": 1.0, "max_abs": 4.0, "mean_abs": 7.0 / 8.0}
    # W_hat = W / 2 (exact in bfloat16): error W / 2
    half = to_bf16_bits(np.array([[1.5, 2.0, 0.0, 0.0], [0.0, 0.0, 0.0, 0.0]]))
    assert F.error_stats(w, half) == {"rel_fro": 0.5, "max_abs": 2.0, "mean_abs": 7.0 / 16.0}
    # error [[0.5, 0], [0, -4]] on W = [[1, 0], [0, -6]]: |d|^2 = 16.25, |W|^2 = 37;
    # the largest error is in the second row and the second column
    w2 = to_bf16_bits(np.array([[1.0, 0.0], [0.0, -6.0]]))
    h2 = to_bf16_bits(np.array([[0.5, 0.0], [0.0, -2.0]]))
    st = F.error_stats(w2, h2)
    assert abs(st["rel_fro"] - (65.0 / 148.0) ** 0.5) < 1e-15
    assert st["max_abs"] == 4.0 and st["mean_abs"] == 4.5 / 4.0
