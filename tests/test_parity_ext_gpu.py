"""The zero-tangent kernel (K' = V' = 0, k_dot = v_dot = None) and the lse
tangent (lse' = sum_j P S', from attn_jvp_fwd_ex) against the fp64 oracle.

lse' has no tolerance of its own in the parity bar; it is a tangent like O'
and is held to the same max|err| / max|ref| <= 2e-2.  Its GPU value is
c + a / l, whose error comes from the bf16 rounding of P (sS' - c): random
per key, so it averages down over the row."""
import numpy as np
import pytest
import torch

from attention_jvp_fwd_b200 import attn_jvp_fwd
from attention_jvp_fwd_b200 import workloads as W
import oracle
from gpu_util import TOL_OD, compare, gpu_rows, oracle_ref, ratio, to_dev

pytestmark = pytest.mark.gpu

TOL_LSE_DOT = TOL_OD


@pytest.fixture(scope="module", autouse=True)
def _built():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    from attention_jvp_fwd_b200.build import build
    build()


def _run(w, zero_kv, lse_dot=True, scale=None):
    ins = [to_dev(x) for x in w.inputs()]
    if zero_kv:
        ins[4] = ins[5] = None
    kvt = torch.from_numpy(np.asarray(w.kv_len, np.int32)).cuda() if w.kv_len is not None else None
    out = attn_jvp_fwd(*ins, scale=w.scale if scale is None else scale, kv_len=kvt, lse_dot=lse_dot)
    torch.cuda.synchronize()
    return out


def _oracle_mu(w, rows=None):
    return oracle.attn_jvp(*w.inputs(), w.scale, kv_len=w.kv_len, rows=rows, lse_dot=True)[3]


def _check_mu(g, ref, what):
    g = np.asarray(g, np.float64).reshape(-1)
    ref = np.asarray(ref, np.float64).reshape(-1)
    assert np.all(np.isfinite(g)), f"{what}: non-finite lse'"
    e = ratio(float(np.max(np.abs(g - ref))), float(np.max(np.abs(ref))))
    assert e <= TOL_LSE_DOT, f"{what}: lse' error {e:.3e} > {TOL_LSE_DOT}"
    return e


@pytest.mark.parametrize("d", [64, 128])
@pytest.mark.parametrize("Lq,Lk", [(1, 1), (128, 64), (127, 129), (200, 1000), (64, 4099)])
def test_zero_kv_full(d, Lq, Lk):
    w = W.make_custom(2, 2, Lq, Lk, d, seed=3 * Lq + Lk, zero_kv_dot_from=0)
    o, od, lse, mu = _run(w, zero_kv=True)
    compare(gpu_rows(o, od, lse), oracle_ref(w), f"zero K'V' d{d} Lq{Lq} Lk{Lk}")
    _check_mu(mu.cpu().numpy(), _oracle_mu(w), f"zero K'V' lse' d{d} Lq{Lq} Lk{Lk}")


@pytest.mark.parametrize("d", [64, 128])
def test_zero_kv_kv_len(d):
    """Per-batch key lengths (0, tile edges, > Lk) on the zero-tangent kernel,
    with NaN in the padded keys of K and V."""
    B, H, Lq, Lk = 6, 2, 130, 200
    kv = np.array([0, 1, 64, 65, 199, 500], np.int32)
    w = W.make_custom(B, H, Lq, Lk, d, seed=17, kv_len=kv, zero_kv_dot_from=0)
    for t in (w.k, w.v):
        for b in range(B):
            t[b, :, max(int(kv[b]), 0):] = np.uint16(0x7FC0)
    o, od, lse, mu = _run(w, zero_kv=True)
    compare(gpu_rows(o, od, lse), oracle_ref(w), f"zero K'V' kv_len d{d}")
    mu = mu.cpu().numpy()
    assert np.all(mu[0] == 0.0), "lse' of rows without keys"
    _check_mu(mu, _oracle_mu(w), f"zero K'V' kv_len lse' d{d}")


@pytest.mark.parametrize("d", [64, 128])
def test_zero_kv_agrees_with_full_kernel(d):
    """With K' = V' = 0 given as tensors, the full kernel adds exact zeros;
    the zero-tangent kernel skips them.  Both must agree to rounding."""
    w = W.make_custom(1, 3, 300, 700, d, seed=23, zero_kv_dot_from=0)
    a = _run(w, zero_kv=True)
    b = _run(w, zero_kv=False)
    for x, y, n in zip(a, b, ("o", "o_dot", "lse", "lse_dot")):
        x, y = x.float(), y.float()
        err = float((x - y).abs().max()) / max(float(y.abs().max()), 1e-30)
        assert err <= 1e-2, f"{n}: zero-tangent vs full kernel {err:.3e}"


@pytest.mark.parametrize("d", [64, 128])
@pytest.mark.parametrize("Lq,Lk", [(1, 1), (127, 129), (200, 1000)])
def test_lse_dot_full_kernel(d, Lq, Lk):
    w = W.make_custom(2, 2, Lq, Lk, d, seed=5 * Lq + Lk)
    o, od, lse, mu = _run(w, zero_kv=False)
    compare(gpu_rows(o, od, lse), oracle_ref(w), f"with lse' d{d} Lq{Lq} Lk{Lk}")
    _check_mu(mu.cpu().numpy(), _oracle_mu(w), f"lse' d{d} Lq{Lq} Lk{Lk}")


def test_lse_dot_does_not_change_other_outputs():
    w = W.make_custom(1, 2, 256, 512, 128, seed=29)
    a = _run(w, zero_kv=False, lse_dot=True)
    b = _run(w, zero_kv=False, lse_dot=False)
    for x, y in zip(a[:3], b):
        assert torch.equal(x, y)


@pytest.mark.parametrize("name", ["cross_frozen", "stress_sharp_d128_L4099", "t2i_self"])
def test_named_workloads_row_sample(name):
    """Full-size workloads, sampled rows: the zero-tangent kernel where every
    batch is frozen, the full kernel with lse' elsewhere."""
    w = W.make(name, seed=0)
    rows = W.sample_rows(w, per_head=8)
    o, od, lse, mu = _run(w, zero_kv=w.zero_kv_dot)
    compare(gpu_rows(o, od, lse, rows), oracle_ref(w, rows=rows), name)
    mu = mu.reshape(-1)[torch.from_numpy(rows).cuda()].cpu().numpy()
    _check_mu(mu, _oracle_mu(w, rows=rows), f"{name} lse'")
