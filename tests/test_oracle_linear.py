"""Pins for the oracle's QLoRA linear forward and backward.

Page: "QLoRA: Efficient Finetuning of Quantized LLMs" (intuitivepapers.ai),
§LoRA and §The QLoRA layer, end to end.  The gradient formulas are checked by
central finite differences of L = <dY, Y(X, A, B)>; L is linear in each of X,
A and B separately, so central differences are exact up to roundoff.
"""
import numpy as np
import pytest

from bit_nf4_quantised_codebook_b200.inputs import normal_bf16, to_bf16_bits, weight_bf16
from oracle import linear, nf4


def _case(m=5, n=128, k=64, r=8, seed=0):
    W = weight_bf16(n, k, 0.02, seed)
    q = nf4.quantize_nf4(W)
    wh = nf4.dequantize_nf4(q)
    X = normal_bf16((m, k), 1.0, seed + 1)
    A = normal_bf16((k, r), 0.1, seed + 2)
    B = normal_bf16((r, n), 0.1, seed + 3)
    dY = normal_bf16((m, n), 1.0, seed + 4)
    return X, wh, A, B, dY


def _loss(X, W, A, B, dY, s):
    Y = X @ W.T + s * (X @ A) @ B
    return float(np.sum(dY * Y))


@pytest.mark.parametrize("which", ["X", "A", "B"])
def test_gradients_by_finite_differences(which):
    s = 2.0
    X, wh, A, B, dY = _case()
    g = linear.backward(X, dY, wh, A, B, s)
    ga = linear.adapter_grads(X, dY, A, B, s)
    Xf, Wf, Af, Bf, dYf = (nf4.bf16_to_f64(t) for t in (X, wh, A, B, dY))
    base = {"X": Xf, "A": Af, "B": Bf}
    grad = {"X": g["dX"], "A": g["dA"], "B": g["dB"]}[which]
    # the adapter-only form (no dX) is held to the same finite differences
    grad2 = {"X": g["dX"], "A": ga["dA"], "B": ga["dB"]}[which]
    rng = np.random.default_rng(9)
    h = 0.5
    for _ in range(25):
        idx = tuple(rng.integers(0, d) for d in base[which].shape)
        args = dict(X=Xf.copy(), A=Af.copy(), B=Bf.copy())
        args[which][idx] += h
        lp = _loss(args["X"], Wf, args["A"], args["B"], dYf, s)
        args[which][idx] -= 2 * h
        lm = _loss(args["X"], Wf, args["A"], args["B"], dYf, s)
        fd = (lp - lm) / (2 * h)
        assert abs(fd - grad[idx]) <= 1e-9 * (1 + abs(fd)), (which, idx, fd, grad[idx])
        assert abs(fd - grad2[idx]) <= 1e-9 * (1 + abs(fd)), (which, idx, fd, grad2[idx])


def test_forward_matches_definition_and_lora_term():
    s = 2.0
    X, wh, A, B, dY = _case(m=7)
    out = linear.forward(X, wh, A, B, s)
    Xf, Wf, Af, Bf = (nf4.bf16_to_f64(t) for t in (X, wh, A, B))
    # element-by-element sums, no matmul: a different evaluation of the same definition
    for i in range(7):
        for j in range(0, 128, 17):
            base = sum(Xf[i, kk] * Wf[j, kk] for kk in range(64))
            lora = sum(Xf[i, kk] * Af[kk, t] * Bf[t, j] for kk in range(64) for t in range(8))
            assert abs(out["Y"][i, j] - (base + s * lora)) < 1e-10
    zero_b = to_bf16_bits(np.zeros_like(Bf))
    d = out["Y"] - linear.forward(X, wh, A, zero_b, s)["Y"]
    assert np.allclose(d, s * Xf @ Af @ Bf, rtol=0, atol=1e-12)


def test_no_gradient_into_frozen_weight():
    """The backward returns dX, dA, dB only (§The QLoRA layer: dW is never formed)."""
    X, wh, A, B, dY = _case()
    g = linear.backward(X, dY, wh, A, B, 2.0)
    assert "dW" not in g and set(["dX", "dA", "dB"]) <= set(g)


def test_backward_rows_helper():
    X, wh, A, B, dY = _case(m=9)
    full = linear.backward(X, dY, wh, A, B, 0.5)["dX"]
    rows = np.array([0, 4, 8])
    assert np.allclose(linear.backward_dx_rows(rows, dY, wh, A, B, 0.5), full[rows], atol=1e-12)


def test_flop_counts():
    f = linear.flops(4096, 4096, 4096, 64)
    assert abs(f["fwd"] + f["bwd"] - 2.878e11) / 2.878e11 < 1e-3
