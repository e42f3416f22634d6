"""The failure path: a device-side wait that runs out returns an error status
instead of hanging, and the context stays usable.  The fault is made by a
test flag that stops the Q/Q' load, so the first wait on it can never
complete; every wait has a 2 ms limit here."""
import numpy as np
import pytest
import torch

import attention_jvp_fwd_b200 as A
from attention_jvp_fwd_b200 import api, workloads as W
from gpu_util import compare, gpu_rows, oracle_ref, to_dev

pytestmark = pytest.mark.gpu


@pytest.mark.parametrize("d", [64, 128])
@pytest.mark.parametrize("B,H,Lq", [(1, 2, 256), (2, 100, 300)])
def test_starved_wait_reports_timeout_and_recovers(d, B, H, Lq):
    """Both softmax splits (d = 64 by key tiles, d = 128 by columns); the
    second shape has 600 query tiles, so every persistent CTA has more tiles
    queued when the wait gives up."""
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    from attention_jvp_fwd_b200.build import build
    build()
    w = W.make_custom(B, H, Lq, 1024, d, seed=3)
    ins = [to_dev(x) for x in w.inputs()]
    assert A.attn_jvp_check()[0] == A.ATTN_JVP_OK
    A.attn_jvp_fwd(*ins, scale=w.scale, _debug_timeout_ns=2_000_000,
                   _debug_flags=api.ATTN_JVP_DEBUG_STARVE_Q)
    status, site = A.attn_jvp_check()
    assert status == A.ATTN_JVP_ERR_TIMEOUT and site != 0
    # the status word was cleared and the device still works
    assert A.attn_jvp_check()[0] == A.ATTN_JVP_OK
    o, od, lse = A.attn_jvp_fwd(*ins, scale=w.scale)
    assert A.attn_jvp_check()[0] == A.ATTN_JVP_OK
    compare(gpu_rows(o, od, lse), oracle_ref(w), f"after timeout d{d} B{B} H{H}")
