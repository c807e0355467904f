"""Shared helpers for the GPU parity tests (CUDA path vs the CPU oracle)."""
import numpy as np
import torch

# Tolerances for floating-point outputs and gradients, against the float64
# oracle evaluated on the identical dequantised weight.
REL_FRO = 1e-2
MAX_REL = 5e-2


def api():
    from bit_nf4_quantised_codebook_b200 import build
    build.build()
    from bit_nf4_quantised_codebook_b200 import api as a
    return a


def to_dev(bits):
    from bit_nf4_quantised_codebook_b200.api import bits_to_tensor
    return bits_to_tensor(bits)


def bits(t):
    from bit_nf4_quantised_codebook_b200.api import tensor_to_bits
    return tensor_to_bits(t)


def bf16_f64(t: torch.Tensor) -> np.ndarray:
    return t.detach().float().cpu().numpy().astype(np.float64)


def f32_f64(t: torch.Tensor) -> np.ndarray:
    return t.detach().cpu().numpy().astype(np.float64)


def assert_close(got: np.ndarray, ref: np.ndarray, name: str) -> dict:
    got = np.asarray(got, np.float64)
    ref = np.asarray(ref, np.float64)
    assert got.shape == ref.shape, (name, got.shape, ref.shape)
    assert np.all(np.isfinite(got)), f"{name}: non-finite output"
    err = got - ref
    nref = np.linalg.norm(ref)
    rel = np.linalg.norm(err) / max(nref, 1e-300)
    mx = np.max(np.abs(err)) / max(np.max(np.abs(ref)), 1e-300)
    assert rel <= REL_FRO, f"{name}: relative Frobenius error {rel:.3e} > {REL_FRO}"
    assert mx <= MAX_REL, f"{name}: max error {mx:.3e} x max|ref| > {MAX_REL}"
    return {"rel_fro": rel, "max_rel": mx}


def check_dev_err(err: torch.Tensor, allowed: int = 0):
    torch.cuda.synchronize()
    v = int(err[0].item())
    assert v & ~allowed == 0, f"device error word {v}"
