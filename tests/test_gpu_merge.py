"""GPU parity of the adapter merge and requantisation (qlora_merge_requantize)
against the CPU oracle (oracle/merge.py).

Exact cases: adapters on a dyadic grid (integers in [-8, 8] times 2^-7).  Every
product is a multiple of 2^-14 below 2^-8 and every partial sum of at most 256
of them stays below 1, so all of them are exact in float32 and the tensor
cores' summation order cannot change the result.  Then the merged weight and
the whole new stored weight (codes, E4M3 constants, group scales, mean) must be
bit-identical to the oracle's.

General cases (Gaussian adapters): the tensor cores' float32 sum differs from
the exact one by at most r·2^-23·sum_j |A[k,j]·B[j,n]|, so the merged bfloat16
weight may differ from the oracle's by one bfloat16 step, and only where the
exact value lies within that much (plus a float32 rounding) of the midpoint
between the two.  Blocks whose merged values all agree must get identical
codes.  The fused requantisation must also equal the library's own quantiser
run on the merged weight it returned, bit for bit.
"""
import numpy as np
import pytest
import torch

from bit_nf4_quantised_codebook_b200 import inputs
from oracle import merge, nf4
from tests.gpu_util import api, assert_close, bits, check_dev_err, to_dev

pytestmark = pytest.mark.gpu


def _stored(q):
    return {"codes": q.codes.cpu().numpy(), "c2q": q.c2q.cpu().numpy(), "c1": q.c1.cpu().numpy(),
            "mean": np.float32(q.mean.cpu().numpy()[0])}


def _assert_same_format(got, ref, what=""):
    assert np.array_equal(got["codes"], ref["codes"]), f"{what}packed codes differ"
    assert np.array_equal(got["c2q"], ref["c2q"]), f"{what}E4M3 block constants differ"
    assert np.array_equal(got["c1"].view(np.uint32), np.asarray(ref["c1"], np.float32).view(np.uint32)), \
        f"{what}group scales differ"
    assert got["mean"].view(np.uint32) == np.float32(ref["mean"]).view(np.uint32), f"{what}mean differs"


def _gpu_merge(q_ref, A, B, s, in_place=False):
    """Load the oracle's stored weight onto the GPU, merge there; returns
    (new stored weight as numpy, merged bf16 bits, device weight)."""
    a = api()
    n, k = q_ref["N"], q_ref["K"]
    w = a.alloc_weight(n, k)
    w.codes.copy_(torch.from_numpy(q_ref["codes"]))
    w.c2q.copy_(torch.from_numpy(q_ref["c2q"]))
    w.c1.copy_(torch.from_numpy(np.asarray(q_ref["c1"], np.float32)))
    w.mean[0] = float(q_ref["mean"])
    err = a.new_error_word()
    wm = torch.empty((n, k), dtype=torch.bfloat16, device="cuda")
    out = a.qlora_merge_requantize(w, to_dev(A), to_dev(B), s, out=w if in_place else None, W_merged=wm,
                                   dev_err=err)
    check_dev_err(err)
    return _stored(out), bits(wm), out


def _case(n, k, r, seed, w_std=0.02, outliers=0.001):
    W = inputs.weight_bf16(n, k, w_std, seed, outliers)
    A = inputs.dyadic_bf16((k, r), 8, 7, seed + 1)
    B = inputs.dyadic_bf16((r, n), 8, 7, seed + 2)
    return nf4.quantize_nf4(W), A, B


EXACT = [
    ("tiny_256x256_r8", 256, 256, 8, 2.0),
    ("ragged_200x320_r16", 200, 320, 16, 0.25),
    ("rows_straddle_64x11008_r64", 64, 11008, 64, 0.25),
    ("two_slices_136x1024_r128", 136, 1024, 128, 0.125),
    ("four_slices_96x512_r256", 96, 512, 256, 0.0625),
    ("single_block_8x64_r8", 8, 64, 8, 1.0),
    ("r24_40x448", 40, 448, 24, 0.5),
]


@pytest.mark.parametrize("name,n,k,r,s", EXACT, ids=[c[0] for c in EXACT])
def test_merge_bit_exact_on_dyadic_adapters(name, n, k, r, s):
    q, A, B = _case(n, k, r, 100 + n)
    ref = merge.merge_requantize(q, A, B, s)
    got, wm, _ = _gpu_merge(q, A, B, s)
    assert np.array_equal(wm, ref["merged"]), "merged weight differs"
    _assert_same_format(got, ref["q"])
    # the merge changed the weight (not a vacuous pass)
    assert not np.array_equal(got["codes"], q["codes"])


def test_merge_in_place_equals_out_of_place():
    q, A, B = _case(200, 640, 64, 7)
    got, wm, _ = _gpu_merge(q, A, B, 0.25)
    got_ip, wm_ip, _ = _gpu_merge(q, A, B, 0.25, in_place=True)
    assert np.array_equal(wm, wm_ip)
    _assert_same_format(got_ip, got, "in place: ")


def test_zero_adapter_keeps_the_codes():
    q, A, _ = _case(128, 2048, 64, 9)
    B = np.zeros((64, 128), np.uint16)
    got, wm, _ = _gpu_merge(q, A, B, 0.25)
    assert np.array_equal(wm, nf4.dequantize_nf4(q))
    assert np.array_equal(got["codes"], q["codes"])
    _assert_same_format(got, merge.merge_requantize(q, A, B, 0.25)["q"])


def test_rank_one_adapter_on_a_zero_weight():
    n, k, r = 48, 192, 8
    q = nf4.quantize_nf4(np.zeros((n, k), np.uint16))
    A = np.zeros((k, r))
    B = np.zeros((r, n))
    A[5, 3], B[3, 17] = 2.0, 3.0
    A, B = inputs.to_bf16_bits(A), inputs.to_bf16_bits(B)
    got, wm, _ = _gpu_merge(q, A, B, 0.25)
    ref = merge.merge_requantize(q, A, B, 0.25)
    assert np.array_equal(wm, ref["merged"])
    assert nf4.bf16_to_f64(wm)[17, 5] == 1.5
    _assert_same_format(got, ref["q"])


def test_full_size_projection_bit_exact():
    """4096 x 4096, r = 64 (the 7B projection), dyadic adapter: every output bit."""
    q, A, B = _case(4096, 4096, 64, 3)
    ref = merge.merge_requantize(q, A, B, 0.25)
    got, wm, _ = _gpu_merge(q, A, B, 0.25)
    assert np.array_equal(wm, ref["merged"])
    _assert_same_format(got, ref["q"])


@pytest.mark.parametrize("n,k,r", [(256, 1024, 64), (72, 4096, 16)])
def test_merge_gaussian_adapter(n, k, r):
    W = inputs.weight_bf16(n, k, 0.02, 51, 0.001)
    A = inputs.normal_bf16((k, r), 0.03, 52)
    B = inputs.normal_bf16((r, n), 0.03, 53)
    s = 0.25
    q = nf4.quantize_nf4(W)
    ref = merge.merge_requantize(q, A, B, s)
    got, wm, dev_w = _gpu_merge(q, A, B, s)

    # merged weight: equal, or one bfloat16 step apart at a rounding boundary
    g = nf4.bf16_to_f64(wm)
    o = nf4.bf16_to_f64(ref["merged"])
    Af, Bf = nf4.bf16_to_f64(A), nf4.bf16_to_f64(B)
    exact = nf4.bf16_to_f64(ref["w_hat"]) + s * (Af @ Bf).T
    slack = s * r * 2.0 ** -23 * (np.abs(Af) @ np.abs(Bf)).T + 2.0 ** -23 * np.abs(exact) + 1e-30
    diff = np.nonzero(wm != ref["merged"])
    assert diff[0].size <= 0.01 * wm.size
    for i, j in zip(*diff):
        step = 2.0 ** (np.floor(np.log2(max(abs(g[i, j]), abs(o[i, j])))) - 7)
        assert abs(g[i, j] - o[i, j]) <= step, (i, j, g[i, j], o[i, j])
        assert abs(exact[i, j] - (g[i, j] + o[i, j]) / 2) <= slack[i, j], (i, j)

    # blocks whose merged values agree are coded identically
    same = np.all((wm == ref["merged"]).reshape(-1, 64), axis=1)
    gc = nf4.unpack_nibbles(got["codes"]).reshape(-1, 64)
    oc = nf4.unpack_nibbles(ref["q"]["codes"]).reshape(-1, 64)
    assert same.mean() > 0.5
    assert np.array_equal(gc[same], oc[same])
    assert abs(float(got["mean"]) - float(ref["q"]["mean"])) <= 2.0 ** -20 * abs(float(ref["q"]["mean"]))

    # the requantised weights agree as values, and so does the requantisation error
    a = api()
    deq = bits(a.qlora_dequantize(dev_w))
    assert_close(nf4.bf16_to_f64(deq), nf4.bf16_to_f64(nf4.dequantize_nf4(ref["q"])), "requantised weight")
    e_gpu = np.linalg.norm(g - nf4.bf16_to_f64(deq)) / np.linalg.norm(g)
    e_ref = merge.requant_error(ref["merged"], ref["q"])["rel_fro"]
    assert abs(e_gpu - e_ref) <= 0.02 * e_ref

    # fused requantisation == the library's quantiser on the merged weight it returned
    err = a.new_error_word()
    q2 = a.qlora_quantize(to_dev(wm), dev_err=err)
    check_dev_err(err)
    _assert_same_format(got, _stored(q2), "fused vs quantiser: ")


def test_non_finite_merged_weight_is_reported():
    q, A, B = _case(128, 256, 16, 61)
    A = A.copy()
    A[10, 3] = 0x7F80                                    # +Inf
    a = api()
    w = a.alloc_weight(128, 256)
    w.codes.copy_(torch.from_numpy(q["codes"]))
    w.c2q.copy_(torch.from_numpy(q["c2q"]))
    w.c1.copy_(torch.from_numpy(np.asarray(q["c1"], np.float32)))
    w.mean[0] = float(q["mean"])
    err = a.new_error_word()
    a.qlora_merge_requantize(w, to_dev(A), to_dev(B), 0.25, dev_err=err)
    torch.cuda.synchronize()
    assert int(err[0].item()) & a.QLORA_DEVERR_NONFINITE
