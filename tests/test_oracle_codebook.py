"""Pins for the oracle's NF4 code points and decision thresholds.

Pages: "QLoRA: Efficient Finetuning of Quantized LLMs" (intuitivepapers.ai)
§NormalFloat; "QLoRA Review" (tildalice.io) §What QLoRA Actually Does.
"""
import math
import os
import statistics
from fractions import Fraction

import numpy as np
import pytest

from oracle import nf4

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")


def _levels_with_stdlib_quantiles():
    """The same recipe evaluated with Python's own inverse normal CDF
    (statistics.NormalDist, a different algorithm from scipy's Cephes ndtri)."""
    nd = statistics.NormalDist()
    off = nf4.OFFSET
    p_pos = [off + i * ((0.5 - off) / 8) for i in range(8)]
    p_neg = [off + i * ((0.5 - off) / 7) for i in range(7)]
    vals = [nd.inv_cdf(p) for p in p_pos] + [-nd.inv_cdf(p) for p in p_neg] + [0.0]
    vals.sort()
    mx = max(abs(v) for v in vals)
    return np.array([v / mx for v in vals], dtype=np.float64)


def test_printed_levels():
    lv = nf4.nf4_levels()
    with open(os.path.join(GOLDEN, "nf4_printed_levels.txt")) as f:
        rows = [ln.split() for ln in f if ln.strip() and not ln.startswith("#")]
    for idx, val, dec in rows:
        assert round(float(lv[int(idx)]), int(dec)) == float(val), (idx, lv[int(idx)])
    assert lv[7] == 0.0 and lv[0] == -1.0 and lv[15] == 1.0


def test_level_invariants():
    lv = nf4.nf4_levels()
    assert lv.dtype == np.float32 and lv.size == 16
    assert np.all(np.diff(lv) > 0)                 # distinct, strictly monotone
    assert np.sum(lv < 0) == 7 and np.sum(lv > 0) == 8 and np.sum(lv == 0) == 1


def test_levels_match_independent_quantile_function():
    ref = _levels_with_stdlib_quantiles()
    ours = nf4.nf4_levels_f64()
    assert np.max(np.abs(ref - ours)) < 1e-14
    # the float32 table is decided by the float64 values; they must agree bit-for-bit
    assert np.array_equal(ref.astype(np.float32).view(np.uint32), nf4.nf4_levels().view(np.uint32))


def test_quantile_function_against_erfc():
    """Phi(ndtri(p)) == p, with Phi written from math.erfc (a closed form)."""
    from scipy.special import ndtri
    ps = list(np.linspace(nf4.OFFSET, 0.5, 9)[:8]) + list(np.linspace(nf4.OFFSET, 0.5, 8)[:7])
    for p in ps:
        x = float(ndtri(p))
        phi = 0.5 * math.erfc(-x / math.sqrt(2.0))
        assert abs(phi - p) < 2e-16 * 8, (p, phi)


def test_thresholds_are_exact_midpoint_cuts():
    lv = nf4.nf4_levels()
    t = nf4.nf4_thresholds(lv)
    m = nf4.nf4_midpoints(lv)
    assert np.all(t.astype(np.float64) > m)
    below = np.nextafter(t, np.float32(-np.inf)).astype(np.float64)
    assert np.all(below <= m)                      # t is the smallest float32 above m
    # several midpoints are exactly representable in float32: those are ties
    exact = m.astype(np.float32).astype(np.float64) == m
    assert exact.sum() >= 1


def _brute_nearest(x: float, lv) -> int:
    """Exact rational argmin, ties to the lower index."""
    xf = Fraction(float(x))
    best, bi = None, -1
    for i, q in enumerate(lv):
        d = abs(xf - Fraction(float(q)))
        if best is None or d < best:
            best, bi = d, i
    return bi


def test_nearest_level_brute_force_on_ties_and_neighbours():
    lv = nf4.nf4_levels()
    m = nf4.nf4_midpoints(lv)
    pts = []
    for mi in m:
        c = np.float32(mi)
        for k in range(-3, 4):
            v = c
            for _ in range(abs(k)):
                v = np.nextafter(v, np.float32(np.inf if k > 0 else -np.inf))
            pts.append(v)
    pts += list(lv) + [np.float32(0), np.float32(-0.0), np.float32(1e-30), np.float32(-1e-30)]
    rng = np.random.default_rng(5)
    pts += list(rng.uniform(-1, 1, 2000).astype(np.float32))
    pts = np.array(pts, np.float32)
    got = nf4.nearest_level(pts, lv)
    want = np.array([_brute_nearest(p, lv) for p in pts])
    assert np.array_equal(got, want)
    # the threshold form used by the library gives the same code
    t = nf4.nf4_thresholds(lv)
    thr = (pts[:, None] >= t[None, :]).sum(axis=1)
    assert np.array_equal(thr, want)


def test_ties_go_to_lower_index():
    lv = nf4.nf4_levels()
    m = nf4.nf4_midpoints(lv)
    for i, mi in enumerate(m):
        if np.float32(mi).astype(np.float64) == mi:
            assert nf4.nearest_level(np.array([mi], np.float32), lv)[0] == i


def _phi(x):
    return 0.5 * math.erfc(-x / math.sqrt(2.0))


def test_equal_mass_quantile_bins():
    """Cuts at Phi^-1(i/16): a N(0,1) sample lands 1/16 in each bin (5 sigma)."""
    from scipy.special import ndtri
    rng = np.random.default_rng(0)
    x = rng.standard_normal(1 << 24)
    cuts = ndtri(np.arange(1, 16) / 16.0)
    freq = np.bincount(np.searchsorted(cuts, x), minlength=16) / x.size
    sigma = math.sqrt((1 / 16) * (15 / 16) / x.size)
    assert np.all(np.abs(freq - 1 / 16) < 5 * sigma), freq


def test_nf4_bins_near_equal_frequency():
    """NF4 nearest-level bins on N(0,1) data scaled by the recipe's own
    normaliser: frequencies equal the closed-form normal masses (5 sigma), and
    each is 1/16 within the stated tolerance 0.010."""
    from scipy.special import ndtri
    lv = nf4.nf4_levels()
    scale = float(ndtri(nf4.OFFSET))            # the recipe divides by this
    cuts = nf4.nf4_midpoints(lv) * scale        # bin edges in N(0,1) units
    edges = [-math.inf] + list(cuts) + [math.inf]
    mass = np.array([_phi(edges[i + 1]) - _phi(edges[i]) for i in range(16)])
    assert abs(mass.sum() - 1) < 1e-12
    assert np.all(np.abs(mass - 1 / 16) <= 0.010), mass
    rng = np.random.default_rng(0)
    x = rng.standard_normal(1 << 22)
    codes = nf4.nearest_level((x / scale).astype(np.float32), lv)
    freq = np.bincount(codes, minlength=16) / x.size
    sig = np.sqrt(mass * (1 - mass) / x.size)
    assert np.all(np.abs(freq - mass) < 5 * sig)


def test_block64_bin_occupancy_range():
    """§NormalFloat: with per-block (64) absmax scaling the bins hold between
    about 2% and 9% of the weights, not 1/16 each."""
    rng = np.random.default_rng(0)
    from bit_nf4_quantised_codebook_b200.inputs import to_bf16_bits
    w = to_bf16_bits(rng.standard_normal((1 << 14, 1024)))
    codes, _ = nf4.quantize_codes(w, nf4.nf4_levels())
    freq = np.bincount(codes, minlength=16) / codes.size
    assert freq.min() >= 0.015 and freq.max() <= 0.095, freq
    assert freq.min() < 0.03 and freq.max() > 0.08      # clearly not equiprobable
