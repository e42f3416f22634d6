"""The last-wave key split (attn_jvp_fwd_ws) against the fp64 oracle.

The persistent kernel walks floor(T / n) waves of whole query tiles on n SMs;
the T mod n tiles left over are cut into key ranges, one per CTA, whose
partial softmax states are merged by the range that finishes last.  These
cases put every kind of item into that last wave: tiles whose batch has no
keys (range 0 writes zeros, the others skip), tiles with fewer key tiles
than ranges, ranges of a single key tile (at d = 64 only one softmax
warpgroup then has work), ranges ending in a masked tail, and CTAs that walk
whole tiles first and then one range."""
import ctypes

import numpy as np
import pytest
import torch

from attention_jvp_fwd_b200 import api, attn_jvp_fwd
from attention_jvp_fwd_b200 import workloads as W
from gpu_util import compare, gpu_rows, oracle_ref, to_dev

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def _built():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    from attention_jvp_fwd_b200.build import build
    build()


def _sms():
    return torch.cuda.get_device_properties(0).multi_processor_count


def _nan_pad(w, kv):
    for t in (w.k, w.v, w.k_dot, w.v_dot):
        for b in range(w.B):
            t[b, :, max(int(kv[b]), 0):] = np.uint16(0x7FC0)


def _run(w, split, zero_kv=False, lse_dot=False):
    ins = [to_dev(x) for x in w.inputs()]
    if zero_kv:
        ins[4] = ins[5] = None
    kvt = torch.from_numpy(np.asarray(w.kv_len, np.int32)).cuda() if w.kv_len is not None else None
    out = attn_jvp_fwd(*ins, scale=w.scale, kv_len=kvt, split=split, lse_dot=lse_dot)
    torch.cuda.synchronize()
    st, site = api.attn_jvp_check()
    assert st == 0, f"device status {st} at site {site}"
    return out


@pytest.mark.parametrize("d", [64, 128])
def test_split_small_grid_ragged(d):
    """18 query tiles, all in the last wave: cut into up to 6 ranges of one
    key tile; batch 1 has no keys, batch 2 two key tiles (the second with one
    key), padded keys hold NaN."""
    B, H, Lq, Lk = 3, 2, 300, 333
    kv = np.array([333, 0, 65], np.int32)
    assert api.attn_jvp_workspace_bytes(B, H, Lq, Lk, d) > 0
    w = W.make_custom(B, H, Lq, Lk, d, seed=51, kv_len=kv)
    _nan_pad(w, kv)
    ref = oracle_ref(w)
    for split in (True, False):
        compare(gpu_rows(*_run(w, split)), ref, f"split={split} d{d}")


@pytest.mark.parametrize("d", [64, 128])
def test_split_after_whole_waves(d):
    """More query tiles than SMs: every CTA walks whole tiles, then the tiles
    left over are cut into ranges of several key tiles; the oracle checks a
    row sample of every head, including all rows of the split tiles' edges."""
    n = _sms()
    nqt = 16
    H = n // nqt + 1                                # T = H * 16 tiles, a little over n
    Lq, Lk = nqt * 128 - 37, 1500
    T = H * nqt
    assert T > n and 0 < T % n and n // (T % n) >= 2, "shape must leave a split last wave"
    assert api.attn_jvp_workspace_bytes(1, H, Lq, Lk, d) > 0
    w = W.make_custom(1, H, Lq, Lk, d, seed=52)
    rows = W.sample_rows(w, per_head=24)
    ref = oracle_ref(w, rows=rows)
    o, od, lse = _run(w, True)
    compare(gpu_rows(o, od, lse, rows), ref, f"split after whole waves d{d}")
    whole = _run(w, False)
    for a, b, name, tol in zip((o, od), whole[:2], ("O", "O'"), (1e-2, 2e-2)):
        e = float((a.float() - b.float()).abs().max() / b.float().abs().max())
        assert e <= tol, f"{name}: split vs whole {e:.3e}"


@pytest.mark.parametrize("d", [64, 128])
def test_split_zero_tangents_and_lse_dot(d):
    """The zero-tangent kernel and lse' through the split."""
    import oracle
    B, H, Lq, Lk = 2, 3, 260, 700
    kv = np.array([700, 300], np.int32)
    w = W.make_custom(B, H, Lq, Lk, d, seed=53, kv_len=kv, zero_kv_dot_from=0)
    assert api.attn_jvp_workspace_bytes(B, H, Lq, Lk, d) > 0
    o, od, lse, mu = _run(w, True, zero_kv=True, lse_dot=True)
    compare(gpu_rows(o, od, lse), oracle_ref(w), f"split zero K'V' d{d}")
    rmu = oracle.attn_jvp(*w.inputs(), w.scale, kv_len=kv, lse_dot=True)[3]
    e = float(np.max(np.abs(mu.cpu().numpy() - rmu)) / np.max(np.abs(rmu)))
    assert e <= 2e-2, f"lse' {e:.3e}"


def test_split_deterministic():
    """Which range merges depends on timing; the merge order does not, so
    repeated calls give the same bits."""
    w = W.make_custom(2, 2, 300, 1000, 128, seed=54)
    a = _run(w, True)
    for _ in range(3):
        b = _run(w, True)
        for x, y in zip(a, b):
            assert torch.equal(x, y)


def test_workspace_argument_errors():
    """Too small, misaligned or missing workspace is refused on the host."""
    lib = api.load_library()
    B, H, Lq, Lk, d = 2, 2, 300, 1000, 128
    need = api.attn_jvp_workspace_bytes(B, H, Lq, Lk, d)
    assert need > 0
    w = W.make_custom(B, H, Lq, Lk, d, seed=55)
    ins = [to_dev(x) for x in w.inputs()]
    o = torch.empty_like(ins[0])
    od = torch.empty_like(ins[0])
    lse = torch.empty((B, H, Lq), dtype=torch.float32, device="cuda")
    ws = torch.empty(need + 512, dtype=torch.uint8, device="cuda")
    vp = ctypes.c_void_p

    def call(ptr, nbytes):
        return lib.attn_jvp_fwd_ws(*[vp(t.data_ptr()) for t in ins + [o, od, lse]], None, B, H, Lq, Lk, d,
                                   ctypes.c_float(w.scale), None, vp(ptr), nbytes,
                                   vp(torch.cuda.current_stream().cuda_stream))

    assert call(ws.data_ptr(), need - 1) == api.ATTN_JVP_ERR_VALUE
    assert call(ws.data_ptr() + 16, need) == api.ATTN_JVP_ERR_ALIGN
    assert call(0, 0) == api.ATTN_JVP_ERR_NULL
    assert call(ins[0].data_ptr(), need) == api.ATTN_JVP_ERR_VALUE  # overlaps q
    assert call(ws.data_ptr(), need) == api.ATTN_JVP_OK
    torch.cuda.synchronize()
    compare(gpu_rows(o, od, lse), oracle_ref(w), "workspace call")
