"""The sCM tangent-normalised loss kernel against its fp64 oracle.

loss is an fp32 sum of squares, compared with relative error <= 1e-4 (fp32
summation of up to ~1e6 terms in a fixed tree order stays near 1e-6); grad =
2 r is rounded to bf16 on output, so max|err| / max|ref| <= 5e-3 (bf16 keeps
8 significant bits, a relative step of 2^-8 ~ 3.9e-3)."""
import numpy as np
import pytest
import torch

from attention_jvp_fwd_b200 import scm_tangent_loss
from attention_jvp_fwd_b200.workloads import bf16_round_bits
from oracle import scm_loss

pytestmark = pytest.mark.gpu

TOL_LOSS = 1e-4
TOL_GRAD = 5e-3


@pytest.fixture(scope="module", autouse=True)
def _built():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    from attention_jvp_fwd_b200.build import build
    build()


def _inputs(B, N, seed, g_scale=1.0, diff_scale=1.0):
    r = np.random.default_rng(seed)
    fe = r.standard_normal((B, N)).astype(np.float32)
    f = fe + diff_scale * r.standard_normal((B, N)).astype(np.float32)
    g = (g_scale * r.standard_normal((B, N))).astype(np.float32)
    return [bf16_round_bits(x) for x in (f, fe, g)]


def _dev(bits):
    return torch.from_numpy(bits.view(np.int16)).cuda().view(torch.bfloat16)


def _check(bits, c=0.1, what=""):
    loss, grad = scm_tangent_loss(*[_dev(b) for b in bits], c=c)
    torch.cuda.synchronize()
    rl, rg = scm_loss.scm_tangent_loss(*bits, c=c)
    gl = loss.cpu().numpy().astype(np.float64)
    el = float(np.max(np.abs(gl - rl) / np.maximum(np.abs(rl), 1e-30)))
    gg = grad.float().cpu().numpy().astype(np.float64)
    eg = float(np.max(np.abs(gg - rg)) / max(float(np.max(np.abs(rg))), 1e-30))
    assert el <= TOL_LOSS, f"{what}: loss error {el:.3e}"
    assert eg <= TOL_GRAD, f"{what}: grad error {eg:.3e}"
    return loss, grad


@pytest.mark.parametrize("B,N", [(1, 1), (1, 8), (3, 1000), (4, 4096), (2, 65544), (8, 262144),
                                 (2, 1000003), (17, 2048)])
def test_shapes(B, N):
    _check(_inputs(B, N, seed=B * 31 + N), what=f"B{B} N{N}")


@pytest.mark.parametrize("c", [0.0, 0.1, 10.0])
@pytest.mark.parametrize("g_scale", [1e-3, 1.0, 30.0])
def test_c_and_tangent_scale(c, g_scale):
    """Small tangents (the c term dominates) to large ones (g / |g|^2)."""
    _check(_inputs(3, 5000, seed=int(g_scale * 7) + 1, g_scale=g_scale), c=c, what=f"c{c} g{g_scale}")


def test_no_grad_and_determinism():
    bits = _inputs(6, 100000, seed=3)
    l1, g1 = _check(bits)
    l2, g2 = scm_tangent_loss(*[_dev(b) for b in bits])
    l3, none = scm_tangent_loss(*[_dev(b) for b in bits], grad=False)
    torch.cuda.synchronize()
    assert none is None
    assert torch.equal(l1, l2) and torch.equal(l1, l3), "loss differs between calls"
    assert torch.equal(g1, g2), "grad differs between calls"


def test_zero_tangent_is_plain_distance():
    bits = _inputs(2, 4096, seed=5)
    bits[2] = np.zeros_like(bits[2])
    loss, _ = _check(bits, what="g = 0")
    f, fe = (torch.from_numpy(((b.astype(np.uint32) << 16).view(np.float32))).double() for b in bits[:2])
    ref = ((f - fe) ** 2).sum(dim=1)
    assert torch.allclose(loss.double().cpu(), ref, rtol=TOL_LOSS)
