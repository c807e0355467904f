"""GPU parity of the fused AdamW step against the float64 oracle: three steps
on tensors of the 7B adapter shapes plus ragged sizes (one launch for all),
moments and float32 parameters within float32 rounding of the oracle, the
bfloat16 copy exactly the rounding of the float32 parameter and within one
bfloat16 step of the oracle's."""
import numpy as np
import pytest
import torch

from oracle import adamw
from oracle.nf4 import f32_to_bf16_rne, bf16_to_f64
from tests.gpu_util import api

pytestmark = pytest.mark.gpu

LR, B1, B2, EPS, WD = 2e-4, 0.9, 0.999, 1e-8, 0.01


def test_adamw_matches_oracle():
    a = api()
    rng = np.random.default_rng(5)
    shapes = [(4096, 64), (64, 4096), (1003,), (3, 5)]
    p0 = [rng.normal(0.0, 0.01, size=s).astype(np.float32) for s in shapes]
    dev = torch.device("cuda")
    P = [torch.tensor(x, device=dev) for x in p0]
    Pb = [torch.empty(x.shape, dtype=torch.bfloat16, device=dev) for x in p0]
    Mm = [torch.zeros(x.shape, dtype=torch.float32, device=dev) for x in p0]
    Vv = [torch.zeros(x.shape, dtype=torch.float32, device=dev) for x in p0]
    ref = [(x.astype(np.float64), np.zeros(x.shape), np.zeros(x.shape)) for x in p0]
    gmax = np.zeros(len(shapes))  # largest |gradient| seen per tensor
    for t in range(1, 4):
        grads = [(rng.normal(size=s) * 10.0 ** rng.integers(-3, 1)).astype(np.float32) for s in shapes]
        gmax = np.maximum(gmax, [np.abs(g).max() for g in grads])
        G = [torch.tensor(g, device=dev) for g in grads]
        a.qlora_adamw_step(list(zip(P, Pb, G, Mm, Vv)), LR, B1, B2, EPS, WD, t)
        ref = [adamw.adamw_step(p, g.astype(np.float64), m, v, t, LR, B1, B2, EPS, WD)
               for (p, m, v), g in zip(ref, grads)]
    torch.cuda.synchronize()
    for k in range(len(shapes)):
        p_ref, m_ref, v_ref = ref[k]
        p_g = P[k].cpu().numpy().astype(np.float64)
        m_g = Mm[k].cpu().numpy().astype(np.float64)
        v_g = Vv[k].cpu().numpy().astype(np.float64)
        # float32 moments: each step rounds m + (1-b1)(g-m) and b2 v + (1-b2) g^2, an error of a
        # few float32 ulps of the gradient scale; m can cancel to near zero, so the bound is absolute
        np.testing.assert_allclose(m_g, m_ref, rtol=1e-5, atol=3 * 2.0 ** -23 * gmax[k])
        np.testing.assert_allclose(v_g, v_ref, rtol=1e-5, atol=3 * 2.0 ** -23 * gmax[k] ** 2)
        # float32 parameters: two roundings of p per step (decay, update) over three steps, a
        # few float32 ulps of the largest |p|, plus the float32 error of the steps themselves
        tol = 8 * 2.0 ** -24 * np.abs(p_ref).max() + 3 * LR * 1e-5
        assert np.max(np.abs(p_g - p_ref)) <= tol
        pb = Pb[k].cpu().view(torch.int16).numpy().view(np.uint16)
        assert np.array_equal(pb, f32_to_bf16_rne(P[k].cpu().numpy()))   # the copy is RN(param)
        ulp = np.abs(bf16_to_f64(f32_to_bf16_rne(p_ref.astype(np.float32))) - bf16_to_f64(pb))
        assert np.all(ulp <= np.abs(p_ref) * 2.0 ** -7 + 1e-30)
