"""GPU parity of the QLoRA linear forward and backward against the float64
CPU oracle on the identical dequantised weight.  Tolerances (relative
Frobenius <= 1e-2, max error <= 5e-2 x max|ref|) are in tests/gpu_util.py."""
import numpy as np
import pytest
import torch

from bit_nf4_quantised_codebook_b200 import inputs
from oracle import linear, nf4
from tests.gpu_util import api, assert_close, bf16_f64, bits, check_dev_err, f32_f64, to_dev

pytestmark = pytest.mark.gpu


def _setup(case, w_bits=None):
    a = api()
    wb = case.W() if w_bits is None else w_bits
    ref_q = nf4.quantize_nf4(wb)
    what = nf4.dequantize_nf4(ref_q)
    err = a.new_error_word()
    q = a.qlora_quantize(to_dev(wb), dev_err=err)
    check_dev_err(err)
    assert np.array_equal(bits(a.qlora_dequantize(q)), what)
    return a, q, what


def _run(case, w_bits=None, check_lora_alone=True):
    a, q, what = _setup(case, w_bits)
    X, A, B, dY = case.X(), case.A(), case.B(), case.dY()
    Xd, Ad, Bd, dYd = to_dev(X), to_dev(A), to_dev(B), to_dev(dY)
    err = a.new_error_word()
    Y, sT = a.qlora_linear_forward(q, Xd, Ad, Bd, case.s, dev_err=err)
    dX, dA, dB = a.qlora_linear_backward(q, Xd, dYd, Ad, Bd, case.s, T_saved=sT, dev_err=err)
    check_dev_err(err)
    ref_f = linear.forward(X, what, A, B, case.s)
    ref_b = linear.backward(X, dY, what, A, B, case.s)
    assert_close(bf16_f64(Y), ref_f["Y"], "Y")
    assert_close(bf16_f64(sT), case.s * ref_f["T"], "sT")
    assert_close(bf16_f64(dX), ref_b["dX"], "dX")
    assert_close(f32_f64(dA), ref_b["dA"], "dA")
    assert_close(f32_f64(dB), ref_b["dB"], "dB")
    if check_lora_alone:
        # the adapter term is ~1% of Y: check Y - Y(B=0) on its own
        Y0, _ = a.qlora_linear_forward(q, Xd, Ad, torch.zeros_like(Bd), case.s)
        zb = inputs.to_bf16_bits(np.zeros((case.r, case.N)))
        ref0 = linear.forward(X, what, A, zb, case.s)["Y"]
        assert_close(bf16_f64(Y0), ref0, "Y(B=0)")
        # Y - Y(B=0) is the adapter term s·(X·A)·B.  Element-wise bound on the
        # difference of the two bf16 outputs: bf16 rounding of each output
        # (half an ulp <= 2^-8 relative), bf16 rounding of s·T before the B
        # product (<= 2^-8 relative per term), float32 accumulation.
        Yg, Y0g = bf16_f64(Y), bf16_f64(Y0)
        d_gpu = Yg - Y0g
        d_ref = ref_f["Y"] - ref0
        Xf, Wf, Bf = nf4.bf16_to_f64(X), nf4.bf16_to_f64(what), nf4.bf16_to_f64(B)
        abs_lora = np.abs(case.s * ref_f["T"]) @ np.abs(Bf)
        abs_base = np.abs(Xf) @ np.abs(Wf).T
        bound = 2.0 ** -8 * (np.abs(Yg) + np.abs(Y0g) + abs_lora) + 1e-5 * (abs_base + abs_lora) + 1e-30
        assert np.all(np.abs(d_gpu - d_ref) <= bound)
    return a, q, what


def test_tiny_forward_backward():
    _run(inputs.tiny())


def test_ragged_shapes():
    """M, N, K not multiples of the 128 / 256 / 64x4 tiles; r = 24."""
    case = inputs.LinearCase("ragged", M=200, N=264, K=320, r=24, alpha=16.0, w_std=0.02, a_std=0.05,
                             b_std=0.05, seed=3)
    _run(case)


def test_zero_weight_isolates_adapter():
    """An all-zero W quantises to the exact-zero level, so Y = s·X·A·B alone."""
    case = inputs.LinearCase("zeroW", M=160, N=512, K=512, r=64, alpha=16.0, w_std=0.02, a_std=0.05,
                             b_std=0.05, seed=4)
    zero = inputs.to_bf16_bits(np.zeros((case.N, case.K)))
    _run(case, w_bits=zero, check_lora_alone=False)


def test_recompute_t_when_not_saved():
    case = inputs.LinearCase("recompute", M=256, N=256, K=512, r=16, alpha=32.0, w_std=0.02, a_std=0.05,
                             b_std=0.05, seed=5)
    a, q, what = _setup(case)
    Xd, Ad, Bd, dYd = (to_dev(t) for t in (case.X(), case.A(), case.B(), case.dY()))
    _, sT = a.qlora_linear_forward(q, Xd, Ad, Bd, case.s)
    r1 = a.qlora_linear_backward(q, Xd, dYd, Ad, Bd, case.s, T_saved=sT)
    r2 = a.qlora_linear_backward(q, Xd, dYd, Ad, Bd, case.s, T_saved=None)
    for x, y in zip(r1, r2):
        assert torch.equal(x, y)


@pytest.mark.parametrize("m", [1, 8, 16, 64])
def test_small_m_forward(m):
    """Decode-sized batches on an 8192 x 8192 weight (split-K path)."""
    case = inputs.small_m(8192, m)
    a, q, what = _setup(case)
    X, A, B = case.X(), case.A(), case.B()
    err = a.new_error_word()
    Y, sT = a.qlora_linear_forward(q, to_dev(X), to_dev(A), to_dev(B), case.s, dev_err=err)
    check_dev_err(err)
    ref = linear.forward(X, what, A, B, case.s)
    assert_close(bf16_f64(Y), ref["Y"], f"Y[m={m}]")
    assert_close(bf16_f64(sT), case.s * ref["T"], f"sT[m={m}]")


@pytest.mark.parametrize("m,n,k,r", [
    (1, 264, 320, 24),     # ragged W-row tile, 5 K steps, one partial adapter chunk
    (17, 1000, 4096, 136), # 32-token tile, 3 adapter chunks (64 + 64 + 8)
    (33, 512, 32768, 64),  # 48-token tile, the longest K of this path (8 splits x 64 steps)
    (64, 256, 64, 8),      # one K step, no split
    (48, 8, 128, 16),      # fewer W rows than one tile
    (8, 40000, 64, 32),    # one K block per tile: CTAs own several whole tiles
    (40, 12800, 256, 64),  # 48-token tile (one accumulator): ranges mix split and whole tiles
])
def test_small_m_path_edges(m, n, k, r):
    """Forward at M <= 64 (W rows on the MMA M side, tokens on N, K split over
    the CTAs of a cluster): ragged tiles, tiles split over many CTAs or owned
    whole, adapter ranks; backward on the same data."""
    case = inputs.LinearCase(f"smallm_edge_{m}x{n}x{k}_r{r}", M=m, N=n, K=k, r=r, alpha=16.0, w_std=0.02,
                             a_std=0.05, b_std=0.05, seed=11 + m)
    _run(case)


def test_proj7b_full_size_sampled():
    """The 4096^3 projection in the benchmark's launch configuration: sampled
    token rows of Y and dX, full dA and dB."""
    case = inputs.proj_7b()
    a, q, what = _setup(case)
    X, A, B, dY = case.X(), case.A(), case.B(), case.dY()
    Xd, Ad, Bd, dYd = to_dev(X), to_dev(A), to_dev(B), to_dev(dY)
    err = a.new_error_word()
    Y, sT = a.qlora_linear_forward(q, Xd, Ad, Bd, case.s, dev_err=err)
    dX, dA, dB = a.qlora_linear_backward(q, Xd, dYd, Ad, Bd, case.s, T_saved=sT, dev_err=err)
    check_dev_err(err)
    rows = np.array([0, 1, 127, 128, 1000, 2047, 2048, 3333, 4094, 4095])
    ref_y = linear.forward(X, what, A, B, case.s, rows=rows)["Y"]
    assert_close(bf16_f64(Y)[rows], ref_y, "Y rows")
    ref_dx = linear.backward_dx_rows(rows, dY, what, A, B, case.s)
    assert_close(bf16_f64(dX)[rows], ref_dx, "dX rows")
    ref_g = linear.adapter_grads(X, dY, A, B, case.s)
    assert_close(f32_f64(dA), ref_g["dA"], "dA")
    assert_close(f32_f64(dB), ref_g["dB"], "dB")


def test_llama_down_projection_shape():
    """K = 11008 (172 blocks per row, groups straddle rows), N = 4096, M = 512."""
    case = inputs.LinearCase("down", M=512, N=4096, K=11008, r=64, alpha=16.0, w_std=0.02, a_std=0.01,
                             b_std=0.01, seed=6)
    _run(case, check_lora_alone=False)


@pytest.mark.parametrize("n,k", [(1024, 22016), (22016, 1024)])
def test_65b_shape_slices(n, k):
    """Slices of the 65B shapes (W 22016 x 8192 and 8192 x 22016, 0.1% outliers)
    cut to 2048 tokens and to 1024 W rows or 1024 columns, so that the oracle
    stays within seconds: the long-K path (344 blocks per row) and the wide
    grid (86 column tiles of the pair kernel)."""
    case = inputs.LinearCase(f"65b_slice_{n}x{k}", M=2048, N=n, K=k, r=64, alpha=16.0, w_std=0.015,
                             a_std=0.01, b_std=0.01, outlier_frac=0.001, seed=21)
    _run(case, check_lora_alone=False)
