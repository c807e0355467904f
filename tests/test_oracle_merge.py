"""Pins for the oracle of the adapter merge and requantisation.

Pages: "QLoRA: quantising the part you are not training" (addaly.com) §What it
costs (merging into the quantised base means requantising); "QLoRA: Efficient
Finetuning of Quantized LLMs" (intuitivepapers.ai) §LoRA, §The QLoRA layer, end
to end (the layer the merged weight must reproduce).
"""
from fractions import Fraction

import numpy as np
import torch

from bit_nf4_quantised_codebook_b200.inputs import dyadic_bf16, normal_bf16, to_bf16_bits, weight_bf16
from oracle import linear, merge, nf4


def _bits(x):
    return to_bf16_bits(np.asarray(x, np.float64))


def _torch_bf16(x64: float) -> int:
    """float64 -> float32 -> bfloat16 bits, by torch's conversions."""
    t = torch.tensor([x64], dtype=torch.float64).to(torch.float32).to(torch.bfloat16)
    return t.view(torch.int16).item() & 0xFFFF


def test_elements_against_exact_rationals():
    n, k, r, s = 8, 64, 16, 0.3
    W = weight_bf16(n, k, 0.02, 11)
    A = normal_bf16((k, r), 0.05, 12)
    B = normal_bf16((r, n), 0.05, 13)
    got = merge.merged_weight(W, A, B, s)
    Wf, Af, Bf = (nf4.bf16_to_f64(x) for x in (W, A, B))
    s32 = Fraction(float(np.float32(s)))
    checked = 0
    for i in range(n):
        for j in range(k):
            v = Fraction(float(Wf[i, j])) + s32 * sum(Fraction(float(Af[j, t])) * Fraction(float(Bf[t, i]))
                                                     for t in range(r))
            f64 = float(v)                       # correctly rounded to float64
            f32 = np.float32(f64)
            # skip the (never expected) case of a float64 exactly on a float32 midpoint,
            # where float64 -> float32 would round twice
            nb = np.nextafter(f32, np.float32(np.inf)) if f64 > float(f32) else np.nextafter(f32, np.float32(-np.inf))
            if f64 == (float(f32) + float(nb)) / 2 and Fraction(f64) != v:
                continue
            assert got[i, j] == _torch_bf16(f64), (i, j)
            checked += 1
    assert checked == n * k


def test_rounds_to_float32_then_bfloat16():
    # exact value 1 + 2^-8 + 2^-30: float32 gives 1 + 2^-8, the bfloat16 midpoint
    # between 1.0 and 1.0078125, which goes to the even one (1.0).  Rounding the
    # exact value straight to bfloat16 would give 1.0078125.
    W = _bits([[1.0]] * 1)
    W = np.repeat(W, 64, axis=1)
    A = _bits(np.tile([2.0 ** -4, 2.0 ** -15], (64, 1)))
    B = _bits([[2.0 ** -4], [2.0 ** -15]])
    assert merge.merged_weight(W, A, B, 1.0)[0, 0] == 0x3F80
    # exact value 1 + 2^-8 + 2^-23 is a float32 above the midpoint: 1.0078125
    A = _bits(np.tile([2.0 ** -4, 2.0 ** -11], (64, 1)))
    B = _bits([[2.0 ** -4], [2.0 ** -12]])
    assert merge.merged_weight(W, A, B, 1.0)[0, 0] == 0x3F81


def test_float64_near_a_float32_midpoint_is_recomputed_exactly():
    # exact value 1 + 2^-8 + 2^-24 + 2^-80: float64 drops 2^-80 and lands on the
    # float32 midpoint between 1 + 2^-8 (even) and 1 + 2^-8 + 2^-23; the exact
    # value is above it, so float32 is 1 + 2^-8 + 2^-23 and bfloat16 1.0078125
    W = np.repeat(_bits([[1.0]]), 64, axis=1)
    A = _bits(np.tile([2.0 ** -4, 2.0 ** -12, 2.0 ** -40], (64, 1)))
    B = _bits([[2.0 ** -4], [2.0 ** -12], [2.0 ** -40]])
    assert merge.merged_weight(W, A, B, 1.0)[0, 0] == 0x3F81
    # and with the last term negative the exact value is below the midpoint
    B = _bits([[2.0 ** -4], [2.0 ** -12], [-(2.0 ** -40)]])
    assert merge.merged_weight(W, A, B, 1.0)[0, 0] == 0x3F80


def test_zero_adapter_is_identity_and_codes_are_a_fixed_point():
    W = weight_bf16(96, 1024, 0.02, 21, outlier_frac=0.002)
    q = nf4.quantize_nf4(W)
    assert np.all(nf4.reconstruct_c2(q["c2q"], q["c1"], q["mean"]) > 0)
    A = normal_bf16((1024, 16), 0.05, 22)
    B = np.zeros((16, 96), np.uint16)
    out = merge.merge_requantize(q, A, B, 0.25)
    assert np.array_equal(out["merged"], out["w_hat"])
    # every block holds a weight at +-c2_hat (its absmax mapped to level 0 or 15),
    # so dequantise-then-quantise returns the same codes
    assert np.array_equal(out["q"]["codes"], q["codes"])


def test_rank_one_adapter_position_and_value():
    n, k, r = 48, 192, 4
    q = nf4.quantize_nf4(np.zeros((n, k), np.uint16))
    A = np.zeros((k, r), np.float64)
    B = np.zeros((r, n), np.float64)
    A[5, 3] = 2.0
    B[3, 17] = 3.0
    out = merge.merge_requantize(q, _bits(A), _bits(B), 0.25)
    m = nf4.bf16_to_f64(out["merged"])
    assert m[17, 5] == 1.5
    m[17, 5] = 0.0
    assert not m.any()
    codes = nf4.unpack_nibbles(out["q"]["codes"]).reshape(n, k)
    assert codes[17, 5] == 15
    codes[17, 5] = 7
    assert np.all(codes == 7)
    blk = (17 * k + 5) // 64
    assert out["q"]["absmax"][blk] == 1.5
    assert np.count_nonzero(out["q"]["absmax"]) == 1


def test_merged_layer_reproduces_the_adapted_layer():
    n, k, r, m_tok, s = 64, 256, 16, 12, 0.25
    W = weight_bf16(n, k, 0.02, 31)
    q = nf4.quantize_nf4(W)
    w_hat = nf4.dequantize_nf4(q)
    A = normal_bf16((k, r), 0.2, 32)
    B = normal_bf16((r, n), 0.2, 33)
    X = normal_bf16((m_tok, k), 1.0, 34)
    Wm = nf4.bf16_to_f64(merge.merged_weight(w_hat, A, B, s))
    y_layer = linear.forward(X, w_hat, A, B, s)["Y"]
    Xf = nf4.bf16_to_f64(X)
    y_merged = Xf @ Wm.T
    # W_eff is the exact sum rounded twice (float32, then bfloat16): within
    # 2^-8 of itself relative, element by element
    bound = np.abs(Xf) @ (np.abs(Wm) * 2.0 ** -8).T + 1e-12
    assert np.all(np.abs(y_merged - y_layer) <= bound)
    # and the adapter's contribution is far above that bound (the test can see a lost s or B)
    y_base = Xf @ nf4.bf16_to_f64(w_hat).T
    assert np.median(np.abs(y_layer - y_base)) > 10 * np.median(bound)


def test_requantisation_error_bound():
    W = weight_bf16(32, 1024, 0.02, 41, outlier_frac=0.002)
    q = nf4.quantize_nf4(W)
    A = dyadic_bf16((1024, 64), 8, 7, 42)
    B = dyadic_bf16((64, 32), 8, 7, 43)
    out = merge.merge_requantize(q, A, B, 0.25)
    q2 = out["q"]
    wm = nf4.bf16_to_f64(out["merged"])
    wr = nf4.bf16_to_f64(nf4.dequantize_nf4(q2))
    c2 = np.repeat(q2["absmax"].astype(np.float64), 64).reshape(wm.shape)
    c2h = np.repeat(nf4.reconstruct_c2(q2["c2q"], q2["c1"], q2["mean"]).astype(np.float64), 64).reshape(wm.shape)
    half_gap = (1 - 0.6961928906) / 2
    assert np.all(np.abs(wm - wr) <= c2 * half_gap + np.abs(c2 - c2h) + np.abs(wr) * 2.0 ** -8 + 1e-30)
    err = merge.requant_error(out["merged"], q2)
    assert 0.0 < err["rel_fro"] < 0.2
    # the merge moved the weights: codes changed in some blocks
    assert not np.array_equal(q2["codes"], q["codes"])


def test_requant_error_hand_computed():
    """Two blocks whose round trip is worked out by hand.  Both blocks have
    absmax 1, so the mean of the constants is 1, every deviation is 0, the
    group scale is 0 and the reconstructed constant is exactly 1.  Row 0,
    [1, 0, ...], is exact.  In row 1, [0.5, -1, 0, ...], -1 is level 0
    exactly and 0.5 goes to the nearest level 0.4407098 (the next one up is
    0.5626170), stored as bfloat16 0.44140625: error 0.05859375 at (1, 0).
    |W| = sqrt(1 + 0.25 + 1) = 1.5."""
    row0 = np.zeros(64)
    row0[0] = 1.0
    row1 = np.zeros(64)
    row1[0], row1[1] = 0.5, -1.0
    w = _bits(np.stack([row0, row1]))
    q = nf4.quantize_nf4(w)
    err = merge.requant_error(w, q)
    assert err["max_abs"] == 0.05859375
    assert abs(err["rel_fro"] - 0.05859375 / 1.5) < 1e-15
    # weights already on the bfloat16 images of the levels (block absmax 1) round-trip exactly
    lv = nf4.bf16_to_f64(_bits(nf4.nf4_levels().astype(np.float64)))
    exact = _bits(np.tile(lv, 4).reshape(1, 64))
    assert merge.requant_error(exact, nf4.quantize_nf4(exact)) == {"rel_fro": 0.0, "max_abs": 0.0}
