"""attn_jvp_fwd_noalloc: the split attention call for callers that cannot
allocate device memory (runtimes that own all device memory and give a
kernel library no allocator, and latency-critical loops that must not call
cudaMalloc, which can synchronise the device).  Its split workspace is the
library's own static device array instead of caller memory.

The test calls it through the C ABI and checks its outputs against the
existing entry point that takes caller-allocated workspace
(attn_jvp_fwd_ws, through the Python binding), within the parity tolerances,
on two calls in a row: the array keeps the previous call's contents, so the
second call also shows that what must start at zero is cleared.  It sits in
a file of its own that pytest collects last, and passes both alone in a
fresh process (where its first call looks up the array's address) and after
the other tests."""
import ctypes

import numpy as np
import pytest
import torch

from attention_jvp_fwd_b200 import api, attn_jvp_fwd
from attention_jvp_fwd_b200 import workloads as W
from gpu_util import TOL_LSE, TOL_O, TOL_OD, to_dev

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def _built():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    from attention_jvp_fwd_b200.build import build
    build()


def _noalloc(ins, w, kvt, lse_dot):
    """One call of attn_jvp_fwd_noalloc through ctypes; returns its outputs."""
    lib = api.load_library()
    B, H, Lq, d = w.B, w.H, w.Lq, w.d
    o = torch.empty((B, H, Lq, d), dtype=torch.bfloat16, device="cuda")
    od = torch.empty_like(o)
    lse = torch.empty((B, H, Lq), dtype=torch.float32, device="cuda")
    mu = torch.empty_like(lse) if lse_dot else None
    vp = ctypes.c_void_p
    ptr = lambda t: vp(None) if t is None else vp(t.data_ptr())  # noqa: E731
    rc = lib.attn_jvp_fwd_noalloc(*[ptr(t) for t in ins], ptr(o), ptr(od), ptr(lse), ptr(mu),
                                  B, H, Lq, w.Lk, d, ctypes.c_float(w.scale),
                                  ptr(kvt), vp(torch.cuda.current_stream().cuda_stream))
    assert rc == api.ATTN_JVP_OK, api.attn_jvp_status_string(rc)
    return (o, od, lse, mu) if lse_dot else (o, od, lse)


def _rel(a, b):
    a, b = a.float(), b.float()
    return float((a - b).abs().max()) / max(float(b.abs().max()), 1e-30)


@pytest.mark.parametrize("d", [64, 128])
def test_noalloc_matches_workspace_entry_point(d):
    # 12 query tiles on a 148-SM device: all of them in the split last wave
    B, H, Lq, Lk = 2, 2, 300, 1000
    assert api.attn_jvp_workspace_bytes(B, H, Lq, Lk, d) > 0, "the shape must use the split"
    kv = np.array([1000, 517], np.int32)
    kvt = torch.from_numpy(kv).cuda()
    for call, seed in enumerate((61, 62)):   # two calls in a row, different inputs
        w = W.make_custom(B, H, Lq, Lk, d, seed=seed + d, kv_len=kv)
        ins = [to_dev(x) for x in w.inputs()]
        got = _noalloc(ins, w, kvt, lse_dot=True)
        ref = attn_jvp_fwd(*ins, scale=w.scale, kv_len=kvt, lse_dot=True)
        torch.cuda.synchronize()
        st, site = api.attn_jvp_check()
        assert st == 0, f"device status {st} at site {site}"
        assert _rel(got[0], ref[0]) <= TOL_O, f"call {call}: O"
        assert _rel(got[1], ref[1]) <= TOL_OD, f"call {call}: O'"
        assert float((got[2] - ref[2]).abs().max()) <= TOL_LSE, f"call {call}: lse"
        assert _rel(got[3], ref[3]) <= TOL_OD, f"call {call}: lse'"


def test_noalloc_status_string():
    assert "static scratch" in api.attn_jvp_status_string(api.ATTN_JVP_ERR_SCRATCH)
