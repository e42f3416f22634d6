"""The QKV projection + RMSNorm prologue kernel against its fp64 oracle.

Outputs are bf16 (about 2^-9 relative rounding) from fp32 accumulation over
D; the bar is the attention one: max|err| / max|ref| <= 1e-2 for q, k, v and
<= 2e-2 for their tangents (which subtract two terms of similar size)."""
import numpy as np
import pytest
import torch

from attention_jvp_fwd_b200 import qkv_prologue_check, qkv_rmsnorm_jvp
from attention_jvp_fwd_b200.workloads import bf16_round_bits
from oracle import qkv_prologue

pytestmark = pytest.mark.gpu

TOL = (1e-2, 1e-2, 1e-2, 2e-2, 2e-2, 2e-2)
NAMES = ("q", "k", "v", "q'", "k'", "v'")


@pytest.fixture(scope="module", autouse=True)
def _built():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    from attention_jvp_fwd_b200.build import build
    build()


def _inputs(B, L, H, D, d, seed):
    r = np.random.default_rng(seed)
    x = bf16_round_bits(r.standard_normal((B * L, D), dtype=np.float32))
    xd = bf16_round_bits(r.standard_normal((B * L, D), dtype=np.float32))
    w = bf16_round_bits((r.standard_normal((3 * H * d, D)) / np.sqrt(D)).astype(np.float32))
    gq = (1 + 0.1 * r.standard_normal(d)).astype(np.float32)
    gk = (1 + 0.1 * r.standard_normal(d)).astype(np.float32)
    return x, xd, w, gq, gk


def _dev16(bits):
    return torch.from_numpy(bits.view(np.int16)).cuda().view(torch.bfloat16)


def _run_and_check(B, L, H, D, d, seed, eps=1e-6):
    x, xd, w, gq, gk = _inputs(B, L, H, D, d, seed)
    outs = qkv_rmsnorm_jvp(_dev16(x), _dev16(xd), _dev16(w), torch.from_numpy(gq).cuda(),
                           torch.from_numpy(gk).cuda(), B, L, H, eps=eps)
    st, site = qkv_prologue_check()
    assert st == 0, f"device status {st} at site {site}"
    ref = qkv_prologue.qkv_rmsnorm_jvp(x, xd, w, gq.astype(np.float64), gk.astype(np.float64),
                                       B, L, H, d, eps=eps)
    errs = []
    for o, rf, tol, n in zip(outs, ref, TOL, NAMES):
        g = o.float().cpu().numpy().astype(np.float64)
        assert np.all(np.isfinite(g)), f"{n}: non-finite"
        e = float(np.max(np.abs(g - rf)) / np.max(np.abs(rf)))
        assert e <= tol, f"B{B} L{L} H{H} D{D} d{d} {n}: error {e:.3e} > {tol}"
        errs.append(e)
    return errs


@pytest.mark.parametrize("B,L,H,D,d", [(1, 128, 1, 64, 128), (2, 200, 2, 256, 128),
                                       (1, 333, 3, 512, 64), (3, 100, 4, 192, 64),
                                       (1, 1, 1, 64, 64)])
def test_shapes(B, L, H, D, d):
    _run_and_check(B, L, H, D, d, seed=B * 100 + L + D)


def test_t2i_sized():
    """A Cosmos-2B-like layer on the T2I token count: 2 x 4096 tokens, D = 2048,
    16 heads of 128."""
    print(_run_and_check(2, 4096, 16, 2048, 128, seed=7))


def test_feeds_attention():
    """The six outputs have exactly the layout attn_jvp_fwd takes."""
    from attention_jvp_fwd_b200 import attn_jvp_fwd
    B, L, H, D, d = 1, 256, 2, 256, 128
    x, xd, w, gq, gk = _inputs(B, L, H, D, d, seed=3)
    q, k, v, qd, kd, vd = qkv_rmsnorm_jvp(_dev16(x), _dev16(xd), _dev16(w), torch.from_numpy(gq).cuda(),
                                          torch.from_numpy(gk).cuda(), B, L, H)
    o, od, lse = attn_jvp_fwd(q, k, v, qd, kd, vd)
    torch.cuda.synchronize()
    assert o.shape == (B, H, L, d) and torch.isfinite(od.float()).all()
