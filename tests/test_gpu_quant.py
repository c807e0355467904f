"""GPU parity of the quantiser and the standalone dequantiser: bit-exact
against the CPU oracle for packed codes, E4M3 constants, group scales, the
mean and the dequantised bfloat16 weight."""
import numpy as np
import pytest
import torch

from bit_nf4_quantised_codebook_b200 import inputs
from oracle import nf4
from tests.gpu_util import api, bits, check_dev_err, to_dev

pytestmark = pytest.mark.gpu


def _quant_gpu(wbits):
    a = api()
    err = a.new_error_word()
    q = a.qlora_quantize(to_dev(wbits), dev_err=err)
    check_dev_err(err)
    return q


def _assert_same_format(q, ref):
    assert np.array_equal(q.codes.cpu().numpy(), ref["codes"]), "packed codes differ"
    assert np.array_equal(q.c2q.cpu().numpy(), ref["c2q"]), "E4M3 block constants differ"
    assert np.array_equal(q.c1.cpu().numpy().view(np.uint32), ref["c1"].view(np.uint32)), "group scales differ"
    assert q.mean.cpu().numpy()[0].view(np.uint32) == np.float32(ref["mean"]).view(np.uint32), "mean differs"


CASES = [
    ("tiny_256x256", lambda: inputs.tiny().W()),
    ("rows_straddle_64x11008", lambda: inputs.weight_bf16(64, 11008, 0.02, 21, 0.001)),
    ("partial_group_3x6400", lambda: inputs.weight_bf16(3, 6400, 0.02, 22)),
    ("outliers_128x8192", lambda: inputs.weight_bf16(128, 8192, 0.02, 23, 0.01)),
    ("single_block_1x64", lambda: inputs.weight_bf16(1, 64, 0.02, 24)),
]


@pytest.mark.parametrize("name,make", CASES, ids=[c[0] for c in CASES])
def test_quantize_bit_exact(name, make):
    w = make()
    ref = nf4.quantize_nf4(w)
    q = _quant_gpu(w)
    _assert_same_format(q, ref)
    deq = api().qlora_dequantize(q)
    assert np.array_equal(bits(deq), nf4.dequantize_nf4(ref)), "dequantised weight differs"


def test_zero_blocks_and_ties():
    lv = nf4.nf4_levels()
    w = np.zeros((4, 256), np.float32)
    w[1, :64] = 1.0                     # block max 1 -> x_hat == w exactly
    m = nf4.nf4_midpoints(lv)
    ties = [np.float32(x) for x in m if np.float32(x).astype(np.float64) == x]
    w[1, 1:1 + len(ties)] = ties        # exact ties between levels (go to the lower index)
    w[2, 64:128] = -np.linspace(0, 0.3, 64)
    wb = inputs.to_bf16_bits(w)
    ref = nf4.quantize_nf4(wb)
    q = _quant_gpu(wb)
    _assert_same_format(q, ref)
    deq = bits(api().qlora_dequantize(q))
    assert np.array_equal(deq, nf4.dequantize_nf4(ref))
    # zero blocks come back as exact zeros (the sign of zero follows c2_hat's sign)
    vals = nf4.bf16_to_f64(deq)
    assert np.all(vals[0] == 0) and np.all(vals[3] == 0)


def test_quantize_7b_projection_full():
    case = inputs.proj_7b()
    w = case.W()
    ref = nf4.quantize_nf4(w)
    q = _quant_gpu(w)
    _assert_same_format(q, ref)
    deq = api().qlora_dequantize(q)
    assert np.array_equal(bits(deq), nf4.dequantize_nf4(ref))


def test_quantize_large_sampled():
    """8192 x 28672 with 0.1% Student-t outliers: the mean and every group
    scale are checked in full; codes and E4M3 constants on sampled rows."""
    N, K = 28672, 8192
    w = inputs.weight_bf16(N, K, 0.02, 0, 0.001)
    q = _quant_gpu(w)
    c2 = nf4.block_absmax(w)
    e_ref, s_ref, mu_ref = nf4.double_quantize(c2)
    assert q.mean.cpu().numpy()[0].view(np.uint32) == np.float32(mu_ref).view(np.uint32)
    assert np.array_equal(q.c1.cpu().numpy().view(np.uint32), s_ref.view(np.uint32))
    assert np.array_equal(q.c2q.cpu().numpy(), e_ref)
    rng = np.random.default_rng(0)
    rows = np.sort(rng.choice(N, 24, replace=False))
    codes_gpu = q.codes.cpu().numpy().reshape(N, K // 2)
    lv = nf4.nf4_levels()
    for r in rows:
        codes, _ = nf4.quantize_codes(w[r:r + 1], lv)
        assert np.array_equal(codes_gpu[r], nf4.pack_nibbles(codes)), r


def test_quantize_deterministic():
    w = inputs.weight_bf16(512, 4096, 0.02, 31, 0.001)
    a = _quant_gpu(w)
    b = _quant_gpu(w)
    for x, y in [(a.codes, b.codes), (a.c2q, b.c2q), (a.c1, b.c1), (a.mean, b.mean)]:
        assert torch.equal(x, y)


def test_nonfinite_weight_is_reported():
    w = inputs.weight_bf16(8, 256, 0.02, 32)
    w[3, 17] = 0x7F80   # +inf
    a = api()
    err = a.new_error_word()
    a.qlora_quantize(to_dev(w), dev_err=err)
    torch.cuda.synchronize()
    assert int(err[0].item()) & a.QLORA_DEVERR_NONFINITE
