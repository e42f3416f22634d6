"""Seeded synthetic inputs for the attention forward + JVP.

This module is shared by the CUDA path's tests and benchmark and by the oracle
side.  It holds input preparation only (random draws, per-row RMS
normalisation of the raw samples, rounding to bf16 storage) and none of the
method's arithmetic.

The workloads are DiT-shaped stand-ins for the image and video models that rCM
distils ("Large Scale Diffusion Distillation via Score-Regularized
Continuous-Time Consistency", ai.info AI summary, Main Findings: T2I at
1360x768 with Cosmos-Predict2, T2V at 480p 832x480x81 with Wan2.1).  No
dataset or trained weight is used; every tensor is drawn from a seeded
generator.

All tensors are returned as ``uint16`` arrays of bf16 bit patterns (round to
nearest even from fp32), laid out ``[B, H, L, d]``.
"""
from __future__ import annotations

import math
from dataclasses import dataclass, field

import numpy as np

STRESS_LENGTHS = (1000, 1024, 2048, 4099, 8192, 16384)
STRESS_DIMS = (64, 128)


def bf16_round_bits(x: np.ndarray) -> np.ndarray:
    """Round float32 values to bf16, nearest-even; returns the uint16 bits."""
    x = np.ascontiguousarray(x, dtype=np.float32)
    u = x.view(np.uint32)
    bias = np.uint32(0x7FFF) + ((u >> np.uint32(16)) & np.uint32(1))
    out = ((u + bias) >> np.uint32(16)).astype(np.uint16)
    nan = np.isnan(x)
    if nan.any():
        out[nan] = np.uint16(0x7FC0)
    return out


def bf16_bits_to_f32(bits: np.ndarray) -> np.ndarray:
    """Widen bf16 bit patterns to float32 (exact)."""
    return (np.asarray(bits, dtype=np.uint16).astype(np.uint32) << np.uint32(16)).view(np.float32)


@dataclass
class Workload:
    name: str
    B: int
    H: int
    Lq: int
    Lk: int
    d: int
    scale: float
    q: np.ndarray
    k: np.ndarray
    v: np.ndarray
    q_dot: np.ndarray
    k_dot: np.ndarray
    v_dot: np.ndarray
    kv_len: np.ndarray | None = None
    meta: dict = field(default_factory=dict)

    def inputs(self):
        return self.q, self.k, self.v, self.q_dot, self.k_dot, self.v_dot

    @property
    def zero_kv_dot(self) -> bool:
        """K' = V' = 0 for every batch (the zero-tangent kernel applies)."""
        return bool(self.meta.get("zero_kv_dot", False))

    def flops_nominal(self) -> float:
        """12 * Lq * Lk * d per (b, h)."""
        return 12.0 * self.Lq * self.Lk * self.d * self.B * self.H

    def flops_valid(self) -> float:
        """Same count over the valid keys only (sum over batches of n_b)."""
        if self.kv_len is None:
            return self.flops_nominal()
        n = np.clip(self.kv_len.astype(np.int64), 0, self.Lk)
        return float(12.0 * self.Lq * self.d * self.H * n.sum())

    def flops_performed(self) -> float:
        """FLOPs the kernel runs on the valid keys: 12 units, or 8 when
        K' = V' = 0 lets it skip Q K'^T and P V'."""
        return self.flops_valid() * (8.0 / 12.0 if self.zero_kv_dot else 1.0)


def _normal(rng: np.random.Generator, shape, chunk: int = 1 << 24) -> np.ndarray:
    """float32 standard normals, drawn in chunks to bound memory."""
    out = np.empty(int(np.prod(shape)), np.float32)
    for s in range(0, out.size, chunk):
        rng.standard_normal(out=out[s:s + chunk], dtype=np.float32)
    return out.reshape(shape)


def _unit_rms_rows(x: np.ndarray) -> np.ndarray:
    """Scale every length-d row to unit root-mean-square (in place, float32)."""
    flat = x.reshape(-1, x.shape[-1])
    for s in range(0, flat.shape[0], 1 << 18):
        blk = flat[s:s + (1 << 18)]
        rms = np.sqrt(np.mean(blk.astype(np.float64) ** 2, axis=1, keepdims=True))
        blk /= np.maximum(rms, 1e-30).astype(np.float32)
    return x


def _to_bits(x: np.ndarray) -> np.ndarray:
    return bf16_round_bits(x)


def make_custom(B: int, H: int, Lq: int, Lk: int, d: int, seed: int = 0, *,
                name: str = "custom", scale: float | None = None,
                q_gain: float = 1.0, tangent_gain=1.0, kv_len=None,
                zero_kv_dot_from: int | None = None, unit_rms_qk: bool = False,
                head_gain_sd: float = 0.0, tangent_log10_range=None) -> Workload:
    """General i.i.d. N(0, 1) workload with the knobs the named configs use.

    - ``q_gain`` multiplies Q (sharp softmax).
    - ``unit_rms_qk`` normalises every Q and K row to unit RMS first;
      ``head_gain_sd`` then multiplies each head of Q and of K by its own draw
      from N(1, head_gain_sd), shared across the batch.
    - ``tangent_log10_range=(lo, hi)`` multiplies Q', K', V' of each head by
      10**u with one u ~ U[lo, hi] per head; ``tangent_gain`` is a plain factor.
    - ``zero_kv_dot_from=b0`` sets K' = V' = 0 for batches b >= b0.
    - ``kv_len`` is an int array [B] (or None).
    """
    rng = np.random.default_rng(seed)
    scale = 1.0 / math.sqrt(d) if scale is None else float(scale)
    qs = (B, H, Lq, d)
    ks = (B, H, Lk, d)
    q = _normal(rng, qs)
    k = _normal(rng, ks)
    v = _normal(rng, ks)
    qd = _normal(rng, qs)
    kd = _normal(rng, ks)
    vd = _normal(rng, ks)
    meta = {}
    if unit_rms_qk:
        _unit_rms_rows(q)
        _unit_rms_rows(k)
    if head_gain_sd:
        gq = (1.0 + head_gain_sd * rng.standard_normal(H)).astype(np.float32)
        gk = (1.0 + head_gain_sd * rng.standard_normal(H)).astype(np.float32)
        q *= gq[None, :, None, None]
        k *= gk[None, :, None, None]
        meta["head_gain_q"] = gq.tolist()
        meta["head_gain_k"] = gk.tolist()
    if q_gain != 1.0:
        q *= np.float32(q_gain)
    tg = np.full(H, float(tangent_gain), np.float64)
    if tangent_log10_range is not None:
        lo, hi = tangent_log10_range
        u = rng.uniform(lo, hi, size=H)
        tg = tg * 10.0 ** u
        meta["tangent_log10"] = u.tolist()
    if not np.all(tg == 1.0):
        t = tg.astype(np.float32)[None, :, None, None]
        qd *= t
        kd *= t
        vd *= t
    if zero_kv_dot_from is not None:
        kd[zero_kv_dot_from:] = 0.0
        vd[zero_kv_dot_from:] = 0.0
        # every batch frozen: callers may pass K' = V' = None
        meta["zero_kv_dot"] = zero_kv_dot_from == 0
    if kv_len is not None:
        kv_len = np.asarray(kv_len, dtype=np.int32).reshape(B)
    return Workload(name, B, H, Lq, Lk, d, scale, _to_bits(q), _to_bits(k), _to_bits(v),
                    _to_bits(qd), _to_bits(kd), _to_bits(vd), kv_len, meta)


# ---------------------------------------------------------------------------
# Named workloads
# ---------------------------------------------------------------------------

def _stress_names():
    out = []
    for d in STRESS_DIMS:
        for L in STRESS_LENGTHS:
            out.append(f"stress_d{d}_L{L}")
    return out


def _stress_sharp_names():
    return [n.replace("stress_", "stress_sharp_") for n in _stress_names()]


NAMED = {
    # tiny self-attention, parity only
    "tiny": dict(B=1, H=2, Lq=128, Lk=128, d=64),
    # T2I self-attention, 64x64 latent tokens (2B-DiT-like)
    "t2i_self": dict(B=2, H=16, Lq=4096, Lk=4096, d=128),
    # T2I/T2V cross-attention to 512 text tokens with per-batch valid length
    "cross": dict(B=4, H=16, Lq=4096, Lk=512, d=128),
    # the same with every batch's keys and values frozen (K' = V' = 0)
    "cross_frozen": dict(B=4, H=16, Lq=4096, Lk=512, d=128),
    # T2V self-attention, 21 latent frames x 30 x 52 patches (14B-DiT-like)
    "t2v_self": dict(B=1, H=40, Lq=32760, Lk=32760, d=128),
    # the same heads at a quarter of the length: small enough for profiler
    # captures, with the same per-head layout and recipe
    "t2v_self_L8192": dict(B=1, H=40, Lq=8192, Lk=8192, d=128),
}
for _n in _stress_names() + _stress_sharp_names():
    _d = int(_n.split("_d")[1].split("_")[0])
    _L = int(_n.split("_L")[1])
    NAMED[_n] = dict(B=1, H=24, Lq=_L, Lk=_L, d=_d)


def names():
    return list(NAMED)


def shape_of(name: str) -> dict:
    return dict(NAMED[name])


def make(name: str, seed: int = 0) -> Workload:
    """Build a named workload.  The recipe per name:

    - ``tiny``: every tensor i.i.d. N(0, 1).
    - ``t2i_self``: Q, K rows at unit RMS times a per-head gain ~ N(1, 0.1)
      (one draw per head and tensor, shared across the batch); V and the
      tangents i.i.d. N(0, 1).
    - ``cross``: all N(0, 1); kv_len[b] ~ U{64..512}; K' = V' = 0 for the
      second half of the batch (frozen text tokens).
    - ``cross_frozen``: as ``cross`` with K' = V' = 0 for every batch.
    - ``t2v_self``: Q, K rows at unit RMS; V and tangents N(0, 1);
      ``t2v_self_L8192`` is the same recipe at L = 8192.
    - ``stress_d{d}_L{L}``: Q x 4; tangents x 10**u, u ~ U[-3, 1] per head.
    - ``stress_sharp_d{d}_L{L}``: as stress but Q x 10, which puts the logit
      standard deviation near 10 and the extremes near +-60.
    """
    s = NAMED[name]
    B, H, Lq, Lk, d = s["B"], s["H"], s["Lq"], s["Lk"], s["d"]
    if name == "tiny":
        return make_custom(B, H, Lq, Lk, d, seed, name=name)
    if name == "t2i_self":
        return make_custom(B, H, Lq, Lk, d, seed, name=name, unit_rms_qk=True,
                           head_gain_sd=0.1)
    if name in ("cross", "cross_frozen"):
        rng = np.random.default_rng([seed, 7])
        kv = rng.integers(64, 513, size=B).astype(np.int32)
        return make_custom(B, H, Lq, Lk, d, seed, name=name, kv_len=kv,
                           zero_kv_dot_from=B // 2 if name == "cross" else 0)
    if name in ("t2v_self", "t2v_self_L8192"):
        return make_custom(B, H, Lq, Lk, d, seed, name=name, unit_rms_qk=True)
    if name.startswith("stress_sharp_"):
        return make_custom(B, H, Lq, Lk, d, seed, name=name, q_gain=10.0,
                           tangent_log10_range=(-3.0, 1.0))
    if name.startswith("stress_"):
        return make_custom(B, H, Lq, Lk, d, seed, name=name, q_gain=4.0,
                           tangent_log10_range=(-3.0, 1.0))
    raise KeyError(name)


def sample_rows(w: Workload, per_head: int = 64, seed: int = 1) -> np.ndarray:
    """Flat query rows for subset parity: per (b, h) the first and last rows,
    every row of the last (possibly partial) 128-row tile's edges, and
    ``per_head`` random rows.  Rows are independent, so parity on them is
    exact parity for those rows."""
    rng = np.random.default_rng([seed, w.B, w.H, w.Lq])
    rows = []
    last_tile = (w.Lq - 1) // 128 * 128
    fixed = {0, 1, 127 % w.Lq, min(128, w.Lq - 1), last_tile, w.Lq - 1, max(w.Lq - 2, 0)}
    for bh in range(w.B * w.H):
        r = set(fixed)
        r.update(rng.integers(0, w.Lq, size=per_head).tolist())
        rows.extend(bh * w.Lq + i for i in sorted(r) if 0 <= i < w.Lq)
    return np.asarray(rows, dtype=np.int64)
