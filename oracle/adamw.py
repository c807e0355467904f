"""Oracle for the adapter optimiser step (AdamW), in float64.
TEST INFRASTRUCTURE ONLY (see the package docstring).

Sources: "QLoRA: Efficient Finetuning of Quantized LLMs" (intuitivepapers.ai),
§Where finetuning memory goes (Adam keeps, for every trained weight, a running
mean and a running variance of its recent gradients, each in 32-bit floats) and
§The QLoRA layer, end to end (the optimiser steps the adapter matrices L1, L2;
the frozen weight has no gradient and no optimiser state); the glossary page
"4-bit QLoRA" (inferensys.com), §Paged optimizers, names AdamW.

The pages give no update formula, so this is AdamW as published by Loshchilov
and Hutter ("Decoupled Weight Decay Regularization", 2019), in the
arrangement PyTorch's AdamW uses: decay the parameter, update the two moments,
then step by the bias-corrected ratio.  Per element, at step t (from 1):
    p  <- p · (1 - lr·wd)
    m  <- m + (1 - b1)·(g - m)
    v  <- b2·v + (1 - b2)·g²
    p  <- p - (lr / (1 - b1^t)) · m / (sqrt(v) / sqrt(1 - b2^t) + eps)
"""
from __future__ import annotations

import numpy as np


def adamw_step(p, g, m, v, t: int, lr: float, b1: float, b2: float, eps: float, wd: float):
    """One step on float64 copies; returns (p, m, v) as new arrays."""
    p = np.asarray(p, np.float64) * (1.0 - lr * wd)
    g = np.asarray(g, np.float64)
    m = np.asarray(m, np.float64) + (1.0 - b1) * (g - np.asarray(m, np.float64))
    v = b2 * np.asarray(v, np.float64) + (1.0 - b2) * g * g
    step_size = lr / (1.0 - b1 ** t)
    denom = np.sqrt(v) / np.sqrt(1.0 - b2 ** t) + eps
    p = p - step_size * m / denom
    return p, m, v
