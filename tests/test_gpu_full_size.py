"""GPU parity at the full sizes of the LLaMA-7B decoder layer (M = 4096) and of
the 65B-class shapes (M = 8192), in the launch configuration the benchmark
times, against the float64 CPU oracle.

The oracle cannot quantise or multiply these tensors whole within a test, so
it evaluates sampled parts that it can compute one by one:
- the stored weight (codes, E4M3 constants) and the dequantised weight on
  sampled 64-blocks, the mean and every group scale in full, bit-exact;
- Y on sampled token rows x sampled W rows (output columns): the first and last
  rows of several 512-token tiles and the edges of 128/256-row tiles;
- dX on the same token rows x the columns of three whole 64-blocks of K;
- dA and dB in full (they need no W_hat).

Within each set the configurations give every linear of one shape the same
seeds, so q, k, v, o are one case, and so are gate and up.
Page: "QLoRA: Efficient Finetuning of Quantized LLMs" (intuitivepapers.ai),
§Guanaco (the 65B model finetuned on one GPU) and §LoRA (adapters on every
linear layer of the block)."""
import numpy as np
import pytest
import torch

from bit_nf4_quantised_codebook_b200 import inputs
from oracle import linear, nf4
from tests.gpu_util import api, assert_close, bits, check_dev_err, f32_f64, to_dev

pytestmark = pytest.mark.gpu


def _rows(m: int) -> np.ndarray:
    return np.array(sorted({0, 1, 511, 512, 1023, m // 2 - 1, m // 2, m - 513, m - 512, m - 2, m - 1}))


def _full_size(case):
    a = api()
    M, N, K, r = case.M, case.N, case.K, case.r
    kb = K // 64
    W = case.W()
    err = a.new_error_word()
    Wd = to_dev(W)
    q = a.qlora_quantize(Wd, dev_err=err)
    del Wd
    X, A, B, dY = case.X(), case.A(), case.B(), case.dY()
    Xd, Ad, Bd, dYd = to_dev(X), to_dev(A), to_dev(B), to_dev(dY)
    Y, sT = a.qlora_linear_forward(q, Xd, Ad, Bd, case.s, dev_err=err)
    dX, dA, dB = a.qlora_linear_backward(q, Xd, dYd, Ad, Bd, case.s, T_saved=sT, dev_err=err)
    check_dev_err(err)
    del Xd, dYd

    rng = np.random.default_rng(M + N + K)
    rows = _rows(M)
    cols = np.array(sorted(set([0, 1, 127, 128, 255, 256, N // 2, N - 129, N - 128, N - 1])
                           | set(rng.integers(0, N, 22).tolist())))
    kblocks = np.array([0, kb // 2, kb - 1])
    kcols = (64 * kblocks[:, None] + np.arange(64)).reshape(-1)
    blocks_y = (cols[:, None] * kb + np.arange(kb)).reshape(-1)      # whole W rows `cols`
    blocks_x = (np.arange(N)[:, None] * kb + kblocks).reshape(-1)    # K-blocks `kblocks` of every row
    blocks = np.unique(np.concatenate([blocks_y, blocks_x]))

    # stored weight and W_hat, bit-exact on the sampled blocks
    ref = nf4.quantize_nf4_blocks(W, blocks)
    bt = torch.from_numpy(blocks).to(q.codes.device)
    assert np.array_equal(q.codes.view(-1, 32)[bt].cpu().numpy(), ref["codes"])
    assert np.array_equal(q.c2q[bt].cpu().numpy(), ref["c2q"])
    assert np.array_equal(q.c1.cpu().numpy(), ref["c1"])
    assert q.mean.cpu().numpy()[0] == ref["mean"]
    wh_ref = nf4.dequantize_nf4_blocks(ref)
    wh_gpu = a.qlora_dequantize(q).view(-1, 64)[bt]
    assert np.array_equal(bits(wh_gpu), wh_ref)
    del wh_gpu

    # Y on sampled token rows x W rows, sT on the same token rows
    w_cols = wh_ref[np.searchsorted(blocks, blocks_y)].reshape(len(cols), K)
    ref_f = linear.forward(X, w_cols, A, B[:, cols], case.s, rows=rows)
    rt = torch.from_numpy(rows).to(Y.device)
    ct = torch.from_numpy(cols).to(Y.device)
    assert_close(Y[rt][:, ct].float().cpu().numpy(), ref_f["Y"], f"{case.name} Y")
    assert_close(sT[rt].float().cpu().numpy(), case.s * ref_f["T"], f"{case.name} sT")

    # dX on the same token rows x three whole K-blocks
    w_k = wh_ref[np.searchsorted(blocks, blocks_x)].reshape(N, len(kcols))
    ref_dx = linear.backward_dx_rows(rows, dY, w_k, A[kcols], B, case.s)
    kt = torch.from_numpy(kcols).to(dX.device)
    assert_close(dX[rt][:, kt].float().cpu().numpy(), ref_dx, f"{case.name} dX")

    # the adapter gradients in full
    ref_g = linear.adapter_grads(X, dY, A, B, case.s)
    assert_close(f32_f64(dA), ref_g["dA"], f"{case.name} dA")
    assert_close(f32_f64(dB), ref_g["dB"], f"{case.name} dB")


def _pick(cases, name):
    return next(c for c in cases if c.name.split("_")[1] == name)


@pytest.mark.parametrize("name", ["gate", "down"])
def test_llama7b_layer_full_size(name):
    """gate/up 11008 x 4096 and down 4096 x 11008 (K = 11008: groups straddle
    rows) at 4096 tokens; q/k/v/o (4096^2) is the 7B-projection case."""
    _full_size(_pick(inputs.llama7b_layer(), name))


@pytest.mark.parametrize("name", ["q", "gate", "down"])
def test_65b_shapes_full_size(name):
    """q/k/v/o 8192^2, gate/up 22016 x 8192, down 8192 x 22016, 8192 tokens,
    weights N(0, 0.015) with 0.1% Student-t(3) outliers."""
    _full_size(_pick(inputs.shapes_65b(), name))
