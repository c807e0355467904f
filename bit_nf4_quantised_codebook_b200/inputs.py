"""Seeded synthetic inputs for the QLoRA NF4 linear layer.

This module holds none of the method's arithmetic: it only draws random
tensors and rounds them to bfloat16 (round-to-nearest-even, done by torch's
own conversion).  Both the CUDA path and the CPU oracle receive the same
bits from here.

Recipe (the same for every workload):

* one ``numpy.random.default_rng`` per tensor; with base seed ``seed`` the
  sub-seeds are W = seed+0, X = seed+1, A = seed+2, B = seed+3, dY = seed+4;
* values are drawn in float64 as ``N(0, std)`` (second parameter read as a
  standard deviation) and rounded to bfloat16;
* weight outliers: exactly ``floor(frac * N * K)`` positions chosen uniformly
  without replacement (from the W generator, after the Gaussian draw) and
  replaced by ``0.2 * t(3)`` samples.

bfloat16 tensors are returned as ``numpy.uint16`` bit patterns.
"""
from __future__ import annotations

import math
from dataclasses import dataclass, field

import numpy as np
import torch


def to_bf16_bits(x: np.ndarray) -> np.ndarray:
    """Round a float array to float32 and then to bfloat16 (both round to
    nearest-even, torch's conversions, run on all host threads); return uint16 bits."""
    t = torch.from_numpy(np.ascontiguousarray(x))
    if t.dtype != torch.float32:
        t = t.to(torch.float32)
    return t.to(torch.bfloat16).view(torch.int16).numpy().view(np.uint16).copy()


def bf16_bits_to_f32(b: np.ndarray) -> np.ndarray:
    """Exact widening of bfloat16 bit patterns to float32."""
    return (np.asarray(b, dtype=np.uint16).astype(np.uint32) << 16).view(np.float32)


def normal_bf16(shape, std: float, seed: int) -> np.ndarray:
    rng = np.random.default_rng(seed)
    return to_bf16_bits(rng.standard_normal(size=shape) * std)


def dyadic_bf16(shape, k_max: int, exp2: int, seed: int) -> np.ndarray:
    """Integers drawn uniformly from [-k_max, k_max], times 2^-exp2.  Exact in
    bfloat16 for k_max <= 256.  With small k_max every product of two such
    values, and every sum of a few hundred of them, is exact in float32, so a
    contraction over them has one correct result whatever its summation order."""
    rng = np.random.default_rng(seed)
    v = rng.integers(-k_max, k_max + 1, size=shape).astype(np.float64) * 2.0 ** -exp2
    return to_bf16_bits(v)


def weight_bf16(n: int, k: int, std: float, seed: int, outlier_frac: float = 0.0) -> np.ndarray:
    rng = np.random.default_rng(seed)
    w = rng.standard_normal(size=(n, k)) * std
    n_out = int(math.floor(outlier_frac * n * k))
    if n_out:
        flat = w.reshape(-1)
        pos = rng.choice(flat.size, size=n_out, replace=False)
        flat[pos] = 0.2 * rng.standard_t(3, size=n_out)
    return to_bf16_bits(w)


@dataclass
class LinearCase:
    """One QLoRA linear layer: W [N,K], X [M,K], A [K,r], B [r,N], dY [M,N]."""
    name: str
    M: int
    N: int
    K: int
    r: int
    alpha: float
    w_std: float
    a_std: float
    b_std: float
    outlier_frac: float = 0.0
    seed: int = 0
    _cache: dict = field(default_factory=dict, repr=False)

    @property
    def s(self) -> float:
        return self.alpha / self.r

    def W(self) -> np.ndarray:
        if "W" not in self._cache:
            self._cache["W"] = weight_bf16(self.N, self.K, self.w_std, self.seed + 0, self.outlier_frac)
        return self._cache["W"]

    def X(self) -> np.ndarray:
        if "X" not in self._cache:
            self._cache["X"] = normal_bf16((self.M, self.K), 1.0, self.seed + 1)
        return self._cache["X"]

    def A(self) -> np.ndarray:
        if "A" not in self._cache:
            self._cache["A"] = normal_bf16((self.K, self.r), self.a_std, self.seed + 2)
        return self._cache["A"]

    def B(self) -> np.ndarray:
        if "B" not in self._cache:
            self._cache["B"] = normal_bf16((self.r, self.N), self.b_std, self.seed + 3)
        return self._cache["B"]

    def dY(self) -> np.ndarray:
        if "dY" not in self._cache:
            self._cache["dY"] = normal_bf16((self.M, self.N), 1.0, self.seed + 4)
        return self._cache["dY"]

    def with_m(self, m: int) -> "LinearCase":
        return LinearCase(self.name, m, self.N, self.K, self.r, self.alpha, self.w_std,
                          self.a_std, self.b_std, self.outlier_frac, self.seed)

    def flops_fwd(self) -> float:
        return 2.0 * self.M * self.N * self.K + 2.0 * self.M * self.r * (self.K + self.N)

    def flops_bwd(self) -> float:
        return 2.0 * self.M * self.N * self.K + 4.0 * self.M * self.r * (self.K + self.N)


# Workloads.  Shapes follow LLaMA-style projections; W is [out, in] = [N, K].
def tiny() -> LinearCase:
    return LinearCase("tiny_256x256_m32_r8", M=32, N=256, K=256, r=8, alpha=16.0,
                      w_std=0.02, a_std=1.0 / 256.0, b_std=0.01)


def proj_7b() -> LinearCase:
    return LinearCase("proj7b_4096x4096_m4096_r64", M=4096, N=4096, K=4096, r=64, alpha=16.0,
                      w_std=0.02, a_std=0.01, b_std=0.01)


def small_m(n: int, m: int) -> LinearCase:
    return LinearCase(f"smallm_{n}x8192_m{m}_r64", M=m, N=n, K=8192, r=64, alpha=16.0,
                      w_std=0.02, a_std=0.01, b_std=0.01, outlier_frac=0.001)


def llama7b_layer() -> list[LinearCase]:
    shapes = [("q", 4096, 4096), ("k", 4096, 4096), ("v", 4096, 4096), ("o", 4096, 4096),
              ("gate", 11008, 4096), ("up", 11008, 4096), ("down", 4096, 11008)]
    return [LinearCase(f"llama7b_{nm}_{n}x{k}_m4096_r64", M=4096, N=n, K=k, r=64, alpha=16.0,
                       w_std=0.02, a_std=0.01, b_std=0.01) for nm, n, k in shapes]


def shapes_65b() -> list[LinearCase]:
    shapes = [("q", 8192, 8192), ("k", 8192, 8192), ("v", 8192, 8192), ("o", 8192, 8192),
              ("gate", 22016, 8192), ("up", 22016, 8192), ("down", 8192, 22016)]
    return [LinearCase(f"65b_{nm}_{n}x{k}_m8192_r64", M=8192, N=n, K=k, r=64, alpha=16.0,
                       w_std=0.015, a_std=0.01, b_std=0.01, outlier_frac=0.001)
            for nm, n, k in shapes]
