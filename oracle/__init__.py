"""fp64 CPU oracle for the attention forward + JVP.

TEST INFRASTRUCTURE ONLY.  Only ``tests/``, ``__graft_entry__.smoke()`` and the
CPU-baseline / reference legs of ``bench.py`` may import this package.  The
product path (``attention_jvp_fwd_b200``) never imports it and shares no code
with it; the two meet only in the seeded input generators, which hold none of
the method's arithmetic.

The arithmetic lives in ``attn_jvp_oracle.c`` (plain C, fp64, two-pass
softmax, no blocking).  This module only compiles it with gcc and marshals
numpy arrays through ctypes.
"""
from __future__ import annotations

import ctypes
import os
import subprocess
import threading

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "attn_jvp_oracle.c")
_LIB_PATH = os.path.join(_HERE, "liboracle_attn_jvp.so")

IN_BF16 = 0
IN_F64 = 1

_lock = threading.Lock()
_lib = None


def compile_oracle(src: str = _SRC, out: str = _LIB_PATH, force: bool = False) -> str:
    """Compile the C oracle with gcc (no fast-math, no FMA contraction)."""
    if (not force and os.path.exists(out)
            and os.path.getmtime(out) >= os.path.getmtime(src)):
        return out
    tmp = out + f".tmp{os.getpid()}"
    cmd = ["gcc", "-O2", "-ffp-contract=off", "-fno-fast-math", "-fopenmp",
           "-fPIC", "-shared", "-o", tmp, src, "-lm"]
    subprocess.run(cmd, check=True)
    os.replace(tmp, out)
    return out


def load_library(path: str | None = None):
    """Load (compiling first if needed) an oracle shared library."""
    global _lib
    if path is not None:
        return _bind(ctypes.CDLL(path))
    with _lock:
        if _lib is None:
            _lib = _bind(ctypes.CDLL(compile_oracle()))
    return _lib


def _bind(lib):
    f = lib.oracle_attn_jvp
    f.restype = ctypes.c_int
    f.argtypes = ([ctypes.c_int] + [ctypes.c_void_p] * 6 + [ctypes.c_int] * 5
                  + [ctypes.c_double, ctypes.c_void_p, ctypes.c_void_p, ctypes.c_int64]
                  + [ctypes.c_void_p] * 4 + [ctypes.c_int])
    lib.oracle_max_threads.restype = ctypes.c_int
    lib.oracle_max_threads.argtypes = []
    return lib


def max_threads() -> int:
    return int(load_library().oracle_max_threads())


def _ptr(a: np.ndarray) -> int:
    return a.ctypes.data


def attn_jvp(q, k, v, q_dot, k_dot, v_dot, scale, kv_len=None, rows=None,
             n_threads: int = 0, lib=None, lse_dot: bool = False):
    """Run the oracle.

    Inputs are either ``uint16`` arrays of bf16 bit patterns or ``float64``
    arrays, shaped ``[B, H, Lq, d]`` (q, q_dot) and ``[B, H, Lk, d]`` (k, v and
    their tangents).  ``kv_len`` is an int32 ``[B]`` array or None.  ``rows``
    selects flat query rows ``(b*H + h)*Lq + i``; the outputs then have a
    leading dimension ``len(rows)`` instead of ``[B, H, Lq]``.

    Returns ``(o, o_dot, lse)`` in float64, and ``lse_dot`` (the tangent of
    lse, mu = sum_j P S') as a fourth array when ``lse_dot`` is set.
    """
    lib = lib or load_library()
    arrs = [q, k, v, q_dot, k_dot, v_dot]
    dt = arrs[0].dtype
    if dt == np.uint16:
        dtype = IN_BF16
    elif dt == np.float64:
        dtype = IN_F64
    else:
        raise TypeError(f"oracle inputs must be uint16 (bf16 bits) or float64, got {dt}")
    arrs = [np.ascontiguousarray(a, dtype=dt) for a in arrs]
    B, H, Lq, d = arrs[0].shape
    Lk = arrs[1].shape[2]
    for a, L in zip(arrs, [Lq, Lk, Lk, Lq, Lk, Lk]):
        if a.shape != (B, H, L, d):
            raise ValueError(f"bad input shape {a.shape}")
    kvp = None
    if kv_len is not None:
        kv_len = np.ascontiguousarray(kv_len, dtype=np.int32)
        if kv_len.shape != (B,):
            raise ValueError("kv_len must have shape [B]")
        kvp = _ptr(kv_len)
    if rows is None:
        out_shape = (B, H, Lq)
        rp, nr = None, 0
    else:
        rows = np.ascontiguousarray(rows, dtype=np.int64)
        out_shape = (rows.shape[0],)
        rp, nr = _ptr(rows), rows.shape[0]
    o = np.empty(out_shape + (d,), np.float64)
    od = np.empty(out_shape + (d,), np.float64)
    lse = np.empty(out_shape, np.float64)
    mu = np.empty(out_shape, np.float64) if lse_dot else None
    if rows is not None and nr == 0:
        return (o, od, lse, mu) if lse_dot else (o, od, lse)
    rc = lib.oracle_attn_jvp(dtype, *[_ptr(a) for a in arrs], B, H, Lq, Lk, d,
                             float(scale), kvp, rp, nr, _ptr(o), _ptr(od), _ptr(lse),
                             _ptr(mu) if lse_dot else None, int(n_threads))
    if rc != 0:
        raise RuntimeError(f"oracle_attn_jvp failed with code {rc}")
    return (o, od, lse, mu) if lse_dot else (o, od, lse)
