"""Plain fp64 CPU oracle for the AdamW step of the non-matrix parameters.

TEST INFRASTRUCTURE ONLY.  Nothing on the product path imports this module: only the
tests, the smoke check and the CPU-baseline leg of the benchmark call it.  It shares
no code with the CUDA library.

Scope -- "14 -- modded-nanogpt: the Speedrun Community", section 3 "Muon -- the optimizer
that started the modern speedrun era": Muon applies to the 2-D matmul weights only; the
1-D parameters (biases, norm gains) and the embeddings take AdamW ("the canonical Muon
setup is hybrid").  The pages give no AdamW formula, so this is the textbook algorithm
with decoupled weight decay (Loshchilov and Hutter, "Decoupled Weight Decay
Regularization") in the form PyTorch's AdamW uses:

    m  <- beta1 m + (1 - beta1) g
    v  <- beta2 v + (1 - beta2) g^2
    m_hat = m / (1 - beta1^t),   v_hat = v / (1 - beta2^t)
    p  <- p (1 - lr wd) - lr m_hat / (sqrt(v_hat) + eps)

with t the 1-based step count, the decay taken from the old p and eps added after the
square root.  Everything is float64.

Pinned (tests/test_adamw_oracle_pins.py) by: hand-worked moment recurrences with exactly
representable betas, the constant-gradient property (with bias correction the update is
-lr g / (|g| + eps) at every step), decay-only steps, scale invariance at eps = 0, and the
eps placement on a tiny gradient.
"""
from __future__ import annotations

from typing import Tuple

import numpy as np


def adamw_moments(m: np.ndarray, v: np.ndarray, g: np.ndarray, beta1: float,
                  beta2: float) -> Tuple[np.ndarray, np.ndarray]:
    """First and second moment recurrences."""
    g = np.asarray(g, np.float64)
    m_new = beta1 * np.asarray(m, np.float64) + (1.0 - beta1) * g
    v_new = beta2 * np.asarray(v, np.float64) + (1.0 - beta2) * g * g
    return m_new, v_new


def adamw_direction(m: np.ndarray, v: np.ndarray, beta1: float, beta2: float, eps: float,
                    step: int) -> np.ndarray:
    """Bias-corrected m_hat / (sqrt(v_hat) + eps) after `step` updates (step >= 1)."""
    m_hat = m / (1.0 - beta1 ** step)
    v_hat = v / (1.0 - beta2 ** step)
    return m_hat / (np.sqrt(v_hat) + eps)


def adamw_step(p: np.ndarray, g: np.ndarray, m: np.ndarray, v: np.ndarray, *, lr: float,
               beta1: float, beta2: float, eps: float, weight_decay: float,
               step: int) -> Tuple[np.ndarray, np.ndarray, np.ndarray]:
    """One AdamW step; returns (p_new, m_new, v_new), all float64."""
    if step < 1:
        raise ValueError("step counts from 1")
    m_new, v_new = adamw_moments(m, v, g, beta1, beta2)
    d = adamw_direction(m_new, v_new, beta1, beta2, eps, step)
    p_new = np.asarray(p, np.float64) * (1.0 - lr * weight_decay) - lr * d
    return p_new, m_new, v_new
