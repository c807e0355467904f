"""GPU parity of the storage-format variants (qlora_quantize_format,
qlora_dequantize_format, qlora_quant_error) against the CPU oracle
(oracle/formats.py): codes, block constants, group scales, mean and the
dequantised weight bit for bit; the error statistics to float64 rounding."""
import itertools

import numpy as np
import pytest
import torch

from bit_nf4_quantised_codebook_b200 import inputs
from oracle import formats as F
from oracle import nf4
from tests.gpu_util import api, bits, check_dev_err, to_dev

pytestmark = pytest.mark.gpu


def _stored(w):
    out = {"codes": w.codes.cpu().numpy(), "consts": w.consts.cpu().numpy()}
    if w.dq != "none":
        out["c1"] = w.c1.cpu().numpy()[: -(-w.consts.numel() // 256)]
        out["mean"] = np.float32(w.mean.cpu().numpy()[0])
    return out


def _check_against_oracle(wbits, cb, block, dq):
    a = api()
    err = a.new_error_word()
    W = to_dev(wbits)
    w = a.qlora_quantize_format(W, cb, block, dq, dev_err=err)
    check_dev_err(err)
    ref = F.quantize(wbits, cb, block, dq)
    got = _stored(w)
    tag = f"{cb}/{block}/{dq}: "
    assert np.array_equal(got["codes"], ref["codes"]), tag + "codes differ"
    if dq == "none":
        assert np.array_equal(got["consts"].view(np.uint32), ref["consts"].view(np.uint32)), tag + "absmax differs"
    else:
        assert np.array_equal(got["consts"].view(np.uint8), np.asarray(ref["consts"]).view(np.uint8)), \
            tag + "8-bit constants differ"
        assert np.array_equal(got["c1"].view(np.uint32), ref["c1"].view(np.uint32)), tag + "group scales differ"
        assert got["mean"].view(np.uint32) == np.float32(ref["mean"]).view(np.uint32), tag + "mean differs"
    deq = a.qlora_dequantize_format(w)
    ref_deq = F.dequantize_q(ref)
    assert np.array_equal(bits(deq), ref_deq), tag + "dequantised weight differs"
    st = a.qlora_quant_error(W, deq).cpu().numpy()
    w64 = nf4.bf16_to_f64(wbits)
    d = w64 - nf4.bf16_to_f64(ref_deq)
    assert abs(st[0] - np.sum(d * d)) <= 1e-12 * np.sum(d * d) + 1e-300, tag
    assert abs(st[1] - np.sum(w64 * w64)) <= 1e-12 * np.sum(w64 * w64), tag
    assert st[2] == np.max(np.abs(d)), tag


@pytest.mark.parametrize("cb,block,dq", list(itertools.product(F.CODEBOOKS, F.BLOCKS, F.DQ_MODES)),
                         ids=lambda v: str(v))
def test_format_bit_exact(cb, block, dq):
    # 40 x 1536 with outliers: groups straddle rows, the last group is partial for every block size
    _check_against_oracle(inputs.weight_bf16(40, 1536, 0.02, 71, 0.002), cb, block, dq)


@pytest.mark.parametrize("cb", F.CODEBOOKS)
def test_zero_blocks_ties_and_tiny_blocks(cb):
    lv = F.codebook(cb)
    w = np.zeros((4, 512), np.float32)
    w[1, :256] = 1.0                                      # absmax 1 in every block: x_hat == w
    m = (lv[:-1].astype(np.float64) + lv[1:].astype(np.float64)) / 2
    ties = [np.float32(x) for x in m if abs(x) <= 1 and np.float32(x).astype(np.float64) == x]
    w[1, 1:1 + len(ties)] = ties                          # exact ties between levels (lower index wins)
    w[1, 40:48] = [1e-30, -1e-30, 1e-38, 0.0, -0.0, 2e-3, -2e-3, 0.5]
    w[2, 64:128] = np.linspace(-1e-33, 1e-33, 64)         # a block too small for the reciprocal path
    w[3, :] = np.linspace(-0.3, 0.2, 512)
    wb = inputs.to_bf16_bits(w)
    for block in F.BLOCKS:
        for dq in F.DQ_MODES:
            _check_against_oracle(wb, cb, block, dq)


def test_main_format_through_the_variant_path():
    """NF4 / 64 / E4M3 through the variant kernels equals the main quantiser."""
    a = api()
    wbits = inputs.weight_bf16(1024, 4096, 0.02, 72, 0.001)
    W = to_dev(wbits)
    w = a.qlora_quantize_format(W, "nf4", 64, "e4m3")
    q = a.qlora_quantize(W)
    assert torch.equal(w.codes, q.codes) and torch.equal(w.consts, q.c2q)
    assert torch.equal(w.c1[: q.c1.numel()], q.c1) and torch.equal(w.mean[:1], q.mean[:1])
    assert torch.equal(a.qlora_dequantize_format(w), a.qlora_dequantize(q))


def test_non_finite_weight_is_reported():
    w = inputs.weight_bf16(8, 256, 0.02, 73)
    w[3, 17] = 0x7FC0                                     # NaN
    a = api()
    err = a.new_error_word()
    a.qlora_quantize_format(to_dev(w), "int4", 32, "none", dev_err=err)
    torch.cuda.synchronize()
    assert int(err[0].item()) & a.QLORA_DEVERR_NONFINITE
