"""The C ABI without a GPU: the library loads, exports every function the
header declares, and rejects bad arguments on the host before any CUDA call."""
import ctypes
import os
import re

import pytest

from attention_jvp_fwd_b200 import api
from attention_jvp_fwd_b200.build import build

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
HEADER = os.path.join(ROOT, "include", "attn_jvp.h")
HEADERS = [os.path.join(ROOT, "include", h) for h in sorted(os.listdir(os.path.join(ROOT, "include")))
           if h.endswith(".h")]


@pytest.fixture(scope="module")
def lib():
    build()
    return api.load_library()


def declared_functions():
    names = set()
    for h in HEADERS:
        text = re.sub(r"/\*.*?\*/", "", open(h).read(), flags=re.S)
        names.update(re.findall(r"^\s*(?:const\s+)?\w+\s*\*?\s*((?:attn_jvp|scm|qkv)_\w+)\s*\(", text, re.M))
    return sorted(names)


def test_header_declares_the_abi():
    assert set(declared_functions()) >= {"attn_jvp_fwd", "attn_jvp_check",
                                         "attn_jvp_status_string"}


def test_exports_every_declared_symbol(lib):
    for name in declared_functions():
        assert hasattr(lib, name), f"library does not export {name}"
    assert set(api.EXPORTED) == set(declared_functions())


def _call(lib, ptrs=None, B=1, H=1, Lq=1, Lk=1, d=64, scale=0.125, kv=None):
    if ptrs is None:
        ptrs = [0x10000 * (i + 1) for i in range(9)]
    return lib.attn_jvp_fwd(*[ctypes.c_void_p(p) for p in ptrs], B, H, Lq, Lk, d,
                            ctypes.c_float(scale), kv, None)


def test_argument_errors(lib):
    good = [0x100000 * (i + 1) for i in range(9)]
    for i in range(9):
        bad = list(good)
        bad[i] = 0
        assert _call(lib, bad) == api.ATTN_JVP_ERR_NULL
    for shape in [(0, 1, 1, 1), (1, 0, 1, 1), (1, 1, 0, 1), (1, 1, 1, 0), (1, 1, -5, 1)]:
        assert _call(lib, good, *shape) == api.ATTN_JVP_ERR_SHAPE
    assert _call(lib, good, 1 << 16, 1 << 16, 1, 1) == api.ATTN_JVP_ERR_SHAPE
    for d in (0, 32, 96, 256):
        assert _call(lib, good, d=d) == api.ATTN_JVP_ERR_HEADDIM
    for i in range(8):
        bad = list(good)
        bad[i] += 8
        assert _call(lib, bad) == api.ATTN_JVP_ERR_ALIGN
    bad = list(good)
    bad[8] += 2
    assert _call(lib, bad) == api.ATTN_JVP_ERR_ALIGN
    assert _call(lib, good, kv=ctypes.c_void_p(0x1002)) == api.ATTN_JVP_ERR_ALIGN
    for s in (float("nan"), float("inf")):
        assert _call(lib, good, scale=s) == api.ATTN_JVP_ERR_VALUE
    alias = list(good)
    alias[6] = alias[0]  # o == q
    assert _call(lib, alias) == api.ATTN_JVP_ERR_VALUE
    alias = list(good)
    alias[7] = alias[6] + 64  # o and o_dot overlap (each holds 1*1*1*64 bf16 = 128 bytes)
    assert _call(lib, alias) == api.ATTN_JVP_ERR_VALUE


def test_status_strings(lib):
    for code in range(-7, 1):
        s = api.attn_jvp_status_string(code)
        assert s and s != "unknown status"
    assert api.attn_jvp_status_string(42) == "unknown status"
    assert lib.attn_jvp_version() >= 100


def test_python_binding_rejects_cpu_tensors():
    import torch
    q = torch.zeros(1, 1, 4, 64, dtype=torch.bfloat16)
    with pytest.raises(ValueError):
        api.attn_jvp_fwd(q, q, q, q, q, q)
    with pytest.raises(TypeError):
        api.attn_jvp_fwd(q.float(), q, q, q, q, q)


def _call_ex(lib, ptrs, lse_dot=None, B=1, H=1, Lq=1, Lk=1, d=64, scale=0.125):
    return lib.attn_jvp_fwd_ex(*[ctypes.c_void_p(p) if p else None for p in ptrs],
                               ctypes.c_void_p(lse_dot) if lse_dot else None, B, H, Lq, Lk, d,
                               ctypes.c_float(scale), None, None)


def test_ex_argument_errors(lib):
    """attn_jvp_fwd_ex: k_dot and v_dot may be NULL together, not alone;
    lse_dot is checked for alignment and overlap like the other outputs."""
    good = [0x100000 * (i + 1) for i in range(9)]
    for i in (4, 5):  # exactly one of k_dot, v_dot missing
        bad = list(good)
        bad[i] = 0
        assert _call_ex(lib, bad) == api.ATTN_JVP_ERR_NULL
    for i in (0, 1, 2, 3, 6, 7, 8):
        bad = list(good)
        bad[i] = 0
        assert _call_ex(lib, bad) == api.ATTN_JVP_ERR_NULL
    assert _call_ex(lib, good, lse_dot=0x2000002) == api.ATTN_JVP_ERR_ALIGN
    assert _call_ex(lib, good, lse_dot=good[8]) == api.ATTN_JVP_ERR_VALUE  # lse_dot == lse
    assert _call_ex(lib, good, lse_dot=good[0]) == api.ATTN_JVP_ERR_VALUE  # overlaps q
    zero_kv = list(good)
    zero_kv[4] = zero_kv[5] = 0
    assert _call_ex(lib, zero_kv, d=96) == api.ATTN_JVP_ERR_HEADDIM  # reaches the later checks
    # the plain entry point keeps requiring both tangents
    assert _call(lib, zero_kv) == api.ATTN_JVP_ERR_NULL


def test_debug_rejects_unknown_flags(lib):
    good = [0x100000 * (i + 1) for i in range(9)]
    rc = lib.attn_jvp_fwd_debug(*[ctypes.c_void_p(p) for p in good], 1, 1, 1, 1, 64,
                                ctypes.c_float(0.125), None, None, ctypes.c_uint64(0), 1 << 5)
    assert rc == api.ATTN_JVP_ERR_VALUE


def test_python_binding_zero_tangent_arguments():
    import torch
    q = torch.zeros(1, 1, 4, 64, dtype=torch.bfloat16)
    with pytest.raises(ValueError):  # only one of k_dot, v_dot given
        api.attn_jvp_fwd(q, q, q, q, q, None)
    with pytest.raises(ValueError):  # CPU tensors, zero-tangent form
        api.attn_jvp_fwd(q, q, q, q, None, None)



def test_scm_loss_argument_errors(lib):
    good = [0x100000 * (i + 1) for i in range(5)]

    def call(p, B=2, N=64, c=0.1):
        return lib.scm_tangent_loss(*[ctypes.c_void_p(x) if x else None for x in p], B, N,
                                    ctypes.c_float(c), None)
    for i in range(4):
        bad = list(good)
        bad[i] = 0
        assert call(bad) == api.ATTN_JVP_ERR_NULL
    for B, N in [(0, 8), (2, 0), (70000, 8), (1, -1)]:
        assert call(good, B, N) == api.ATTN_JVP_ERR_SHAPE
    for i in (0, 1, 2, 4):
        bad = list(good)
        bad[i] += 8
        assert call(bad) == api.ATTN_JVP_ERR_ALIGN
    bad = list(good)
    bad[3] += 2
    assert call(bad) == api.ATTN_JVP_ERR_ALIGN
    for c in (float("nan"), float("inf"), -0.5):
        assert call(good, c=c) == api.ATTN_JVP_ERR_VALUE
    alias = list(good)
    alias[4] = alias[2]  # grad == g
    assert call(alias) == api.ATTN_JVP_ERR_VALUE
    alias = list(good)
    alias[3] = alias[0] + 16  # loss inside f
    assert call(alias) == api.ATTN_JVP_ERR_VALUE



def test_qkv_prologue_argument_errors(lib):
    good = [0x100000 * (i + 1) for i in range(11)]

    def call(p, B=1, L=128, H=2, D=256, d=128, eps=1e-6):
        return lib.qkv_rmsnorm_jvp(*[ctypes.c_void_p(x) if x else None for x in p], B, L, H, D, d,
                                   ctypes.c_float(eps), None)
    for i in range(11):
        bad = list(good)
        bad[i] = 0
        assert call(bad) == api.ATTN_JVP_ERR_NULL
    for kw in ({"B": 0}, {"L": 0}, {"H": 0}, {"D": 0}, {"D": 96}, {"D": 32}):
        assert call(good, **kw) == api.ATTN_JVP_ERR_SHAPE
    for d in (32, 96, 256):
        assert call(good, d=d) == api.ATTN_JVP_ERR_HEADDIM
    for i in (0, 1, 2, 5, 6, 7, 8, 9, 10):
        bad = list(good)
        bad[i] += 8
        assert call(bad) == api.ATTN_JVP_ERR_ALIGN
    for i in (3, 4):
        bad = list(good)
        bad[i] += 2
        assert call(bad) == api.ATTN_JVP_ERR_ALIGN
    for eps in (float("nan"), -1.0):
        assert call(good, eps=eps) == api.ATTN_JVP_ERR_VALUE
    alias = list(good)
    alias[5] = alias[0]  # q == x
    assert call(alias) == api.ATTN_JVP_ERR_VALUE
    alias = list(good)
    alias[6] = alias[5] + 16  # q and k overlap
    assert call(alias) == api.ATTN_JVP_ERR_VALUE
