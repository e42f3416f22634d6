"""fp64 oracle for the tangent-normalised sCM loss term.

TEST INFRASTRUCTURE ONLY, like the rest of ``oracle/``: only ``tests/``,
``__graft_entry__.smoke()`` and ``bench.py``'s CPU legs may use it.

What it computes.  The sCM term of rCM uses tangent normalisation
(papernotes.org notes on "Large Scale Diffusion Distillation via
Score-Regularized Continuous-Time Consistency", 损失函数 / 训练策略; ai.info AI
summary, Methodology in Plain English: c = 0.1).  Per sample b, over all its
elements i:

    n_b     = sum_i g_bi^2                          (the squared L2 norm of g_b)
    r_bi    = F_bi - F-_bi - g_bi / (n_b + c)
    loss_b  = sum_i r_bi^2                          (the squared L2 norm of r_b)
    grad_bi = 2 r_bi                                (d loss_b / d F_bi)

F is the student output, F- the EMA target's output (no gradient), g the
tangent direction.  The expectation over samples is left to the caller.
Inputs are bf16 bit patterns (widened exactly) or float64 arrays of shape
[B, N]; every sum is a plain numpy fp64 sum.
"""
from __future__ import annotations

import numpy as np


def _widen(x: np.ndarray) -> np.ndarray:
    x = np.asarray(x)
    if x.dtype == np.uint16:
        return (x.astype(np.uint32) << np.uint32(16)).view(np.float32).astype(np.float64)
    if x.dtype == np.float64:
        return x
    raise TypeError(f"oracle inputs must be uint16 (bf16 bits) or float64, got {x.dtype}")


def scm_tangent_loss(f, f_ema, g, c: float = 0.1):
    """Returns (loss [B], grad [B, N]) in float64."""
    f, fe, g = (_widen(a) for a in (f, f_ema, g))
    if not (f.shape == fe.shape == g.shape) or f.ndim != 2:
        raise ValueError("f, f_ema and g must share one [B, N] shape")
    n = np.sum(g * g, axis=1)
    r = f - fe - g / (n + c)[:, None]
    loss = np.sum(r * r, axis=1)
    return loss, 2.0 * r
