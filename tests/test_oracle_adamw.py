"""Pins of the AdamW oracle against closed forms and an independent library
implementation (torch.optim.AdamW, float64, on the CPU)."""
import numpy as np
import torch

from oracle import adamw

LR, B1, B2, EPS = 2e-4, 0.9, 0.999, 1e-8


def test_first_step_is_a_signed_step_of_lr():
    # t = 1, no decay: m_hat = g and v_hat = g^2, so the step is lr * g / (|g| + eps)
    rng = np.random.default_rng(0)
    p0, g = rng.normal(size=1000), rng.normal(size=1000)
    p, m, v = adamw.adamw_step(p0, g, np.zeros(1000), np.zeros(1000), 1, LR, B1, B2, EPS, 0.0)
    np.testing.assert_allclose(p, p0 - LR * g / (np.abs(g) + EPS), rtol=0, atol=1e-15)
    np.testing.assert_allclose(m, (1 - B1) * g, rtol=1e-15)
    np.testing.assert_allclose(v, (1 - B2) * g * g, rtol=1e-15)


def test_constant_gradient_takes_equal_steps():
    # a constant gradient makes both bias-corrected moments exact: every step is the same
    g = np.array([0.5, -2.0, 1e-3])
    p, m, v = np.zeros(3), np.zeros(3), np.zeros(3)
    for t in range(1, 6):
        p, m, v = adamw.adamw_step(p, g, m, v, t, LR, B1, B2, EPS, 0.0)
        np.testing.assert_allclose(p, -t * LR * g / (np.abs(g) + EPS), rtol=1e-12)


def test_zero_gradient_decays_geometrically():
    p0 = np.array([1.0, -3.0, 0.25])
    p, m, v = p0, np.zeros(3), np.zeros(3)
    for t in range(1, 8):
        p, m, v = adamw.adamw_step(p, np.zeros(3), m, v, t, LR, B1, B2, EPS, 0.01)
    np.testing.assert_allclose(p, p0 * (1 - LR * 0.01) ** 7, rtol=1e-14)


def test_matches_torch_adamw():
    rng = np.random.default_rng(1)
    p0 = rng.normal(size=(64, 32))
    w = torch.nn.Parameter(torch.tensor(p0, dtype=torch.float64))
    opt = torch.optim.AdamW([w], lr=LR, betas=(B1, B2), eps=EPS, weight_decay=0.01, foreach=False)
    p, m, v = p0, np.zeros_like(p0), np.zeros_like(p0)
    for t in range(1, 6):
        g = rng.normal(size=p0.shape) * 10.0 ** rng.integers(-3, 2)
        w.grad = torch.tensor(g)
        opt.step()
        p, m, v = adamw.adamw_step(p, g, m, v, t, LR, B1, B2, EPS, 0.01)
        np.testing.assert_allclose(w.detach().numpy(), p, rtol=1e-13, atol=1e-16)
        st = opt.state[w]
        np.testing.assert_allclose(st["exp_avg"].numpy(), m, rtol=1e-13, atol=1e-300)
        np.testing.assert_allclose(st["exp_avg_sq"].numpy(), v, rtol=1e-13, atol=1e-300)
