"""fp64 oracle for the QKV projection + RMSNorm prologue and its JVP.

TEST INFRASTRUCTURE ONLY, like the rest of ``oracle/``: only ``tests/``,
``__graft_entry__.smoke()`` and ``bench.py``'s CPU legs may use it.

What it computes.  rCM makes JVP work with FSDP by refactoring each layer to
expose a forward and a tangent function ("Large Scale Diffusion Distillation
via Score-Regularized Continuous-Time Consistency", ai.info AI summary, Key
Contributions 1).  The layer in front of attention projects tokens to Q, K, V
and normalises Q and K; its tangent function carries X' through the same
steps, with the weights fixed.  Per token t (t = b L + l) and head h:

    y_q = x W_q[h]^T,  y_k = x W_k[h]^T,  y_v = x W_v[h]^T        (each length d)
    r   = (mean_c y_c^2 + eps)^(-1/2)
    q   = gamma_q * y_q * r_q,   k = gamma_k * y_k * r_k,   v = y_v
    y'  = x' W[h]^T
    q'  = gamma_q * (y_q' r_q - y_q r_q^3 mean_c(y_q y_q'))   (and k' alike)
    v'  = y_v'

Readings where the pages say nothing: the RMSNorm runs over each head's d
channels (QK-norm), with a learned gain gamma of length d shared by all
heads; V is not normalised; the weights carry no tangent.  The fused weight
is W = [W_q; W_k; W_v] of shape [3 H d, D] (one row per output channel, as a
linear layer stores it).  Outputs use the attention layout [B, H, L, d].
Inputs are bf16 bit patterns (widened exactly) or float64.
"""
from __future__ import annotations

import numpy as np


def _widen(x: np.ndarray) -> np.ndarray:
    x = np.asarray(x)
    if x.dtype == np.uint16:
        return (x.astype(np.uint32) << np.uint32(16)).view(np.float32).astype(np.float64)
    if x.dtype in (np.float64, np.float32):
        return x.astype(np.float64)
    raise TypeError(f"unsupported input dtype {x.dtype}")


def _rmsnorm_jvp(y, yd, gamma, eps):
    """Per row of the last axis: (gamma y r, gamma (y' r - y r^3 mean(y y')))."""
    r = 1.0 / np.sqrt(np.mean(y * y, axis=-1, keepdims=True) + eps)
    m = np.mean(y * yd, axis=-1, keepdims=True)
    return gamma * y * r, gamma * (yd * r - y * r ** 3 * m)


def qkv_rmsnorm_jvp(x, x_dot, w_qkv, gamma_q, gamma_k, B, L, H, d, eps=1e-6):
    """x, x_dot: [B*L, D]; w_qkv: [3*H*d, D]; gamma_q, gamma_k: [d].
    Returns (q, k, v, q_dot, k_dot, v_dot), each float64 [B, H, L, d]."""
    x, xd, w = _widen(x), _widen(x_dot), _widen(w_qkv)
    gq, gk = _widen(gamma_q), _widen(gamma_k)
    T, D = x.shape
    if T != B * L or w.shape != (3 * H * d, D) or xd.shape != x.shape:
        raise ValueError("shape mismatch")
    y = x @ w.T          # [T, 3 H d]
    yd = xd @ w.T

    def heads(a, part):  # part 0 q, 1 k, 2 v -> [B, H, L, d]
        return a[:, part * H * d:(part + 1) * H * d].reshape(B, L, H, d).transpose(0, 2, 1, 3)

    q, qd = _rmsnorm_jvp(heads(y, 0), heads(yd, 0), gq, eps)
    k, kd = _rmsnorm_jvp(heads(y, 1), heads(yd, 1), gk, eps)
    v, vd = heads(y, 2), heads(yd, 2)
    return tuple(np.ascontiguousarray(a) for a in (q, k, v, qd, kd, vd))
