"""The trace build of the attention kernel: the same outputs as the normal
build, bit for bit, and stamps that respect the pipeline's order."""
import numpy as np
import pytest
import torch

from attention_jvp_fwd_b200 import attn_jvp_fwd, attn_jvp_fwd_trace, trace as T
from attention_jvp_fwd_b200 import workloads as W
from gpu_util import to_dev

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def _built():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    from attention_jvp_fwd_b200.build import build
    build()


@pytest.mark.parametrize("d", [64, 128])
def test_trace_build_matches_and_orders_events(d):
    B, H, Lq, Lk = 2, 8, 700, 333
    kv = np.array([333, 130], np.int32)
    w = W.make_custom(B, H, Lq, Lk, d, seed=21, kv_len=kv)
    ins = [to_dev(x) for x in w.inputs()]
    kvt = torch.from_numpy(kv).cuda()
    ref = attn_jvp_fwd(*ins, scale=w.scale, kv_len=kvt, split=False)  # the trace build walks tiles whole
    o, od, lse, tr = attn_jvp_fwd_trace(*ins, scale=w.scale, kv_len=kvt, tiles=24)
    torch.cuda.synchronize()
    for a, b in zip(ref, (o, od, lse)):
        assert torch.equal(a, b), "the trace build must not change any output"
    t = tr.cpu().numpy()
    # A stamp is taken a few instructions after its event, by a warp that the
    # SM schedules independently of the others: allow that much slack when
    # comparing stamps of different warps.
    slack = 200
    stamped = 0
    for c in range(t.shape[0]):
        for i in range(t.shape[1]):
            r = t[c, i]
            if not r[T.S_ISSUE]:
                continue
            stamped += 1
            assert 0 < r[T.K_LOAD] <= r[T.S_ISSUE] + slack
            owners = [g for g in (0, 1) if r[T.SM_S + 3 * g]]
            # d = 64: warpgroup g takes the key tiles with index % 2 == g
            assert owners == ([i % 2] if d == 64 else [0, 1])
            for g in owners:
                s, p, pd = r[T.SM_S + 3 * g], r[T.SM_P + 3 * g], r[T.SM_PD + 3 * g]
                assert r[T.S_ISSUE] <= s + slack and s <= p <= pd  # same warp: strict
                assert p <= r[T.PA_ISSUE] + slack and pd <= r[T.PB_ISSUE] + slack
            assert r[T.V_LOAD] <= r[T.PA_ISSUE] + slack and r[T.PA_ISSUE] <= r[T.PB_ISSUE]
    assert stamped > t.shape[0]  # most CTAs had several key tiles
    s = T.summarize(t)
    assert s["period"] > 0 and s["softmax_tile"] > s["softmax_p"] > 0
