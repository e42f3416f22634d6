"""Ulysses path on the GPU with one NCCL rank: the exchange is the identity,
so the context-parallel call must reproduce the plain kernel call bit for bit
(and so match the oracle).  More ranks need more GPUs; the exchange itself is
checked with 2 and 4 gloo ranks in test_ulysses_dist.py."""
import os
import socket

import numpy as np
import pytest
import torch
import torch.distributed as dist

from attention_jvp_fwd_b200 import attn_jvp_fwd, ulysses
from attention_jvp_fwd_b200 import workloads as W
from gpu_util import compare, gpu_rows, oracle_ref, to_dev

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def nccl_group():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    from attention_jvp_fwd_b200.build import build
    build()
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        port = s.getsockname()[1]
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    torch.cuda.set_device(0)
    dist.init_process_group("nccl", rank=0, world_size=1, device_id=torch.device("cuda", 0))
    yield None
    dist.destroy_process_group()


def test_single_rank_ulysses_is_the_kernel(nccl_group):
    w = W.make_custom(2, 4, 300, 300, 128, seed=41)
    ins = [to_dev(x) for x in w.inputs()]
    o, od, lse = ulysses.ulysses_attn_jvp(*ins, scale=w.scale)
    ro, rod, rlse = attn_jvp_fwd(*ins, scale=w.scale)
    torch.cuda.synchronize()
    assert torch.equal(o, ro) and torch.equal(od, rod) and torch.equal(lse, rlse)
    compare(gpu_rows(o, od, lse), oracle_ref(w), "ulysses P=1")


@pytest.mark.parametrize("zero_kv", [False, True])
def test_single_rank_ulysses_cross(nccl_group, zero_kv):
    """Cross-attention through the context-parallel call: text keys replicated
    (Lk = 77, ragged valid lengths including 0), with and without K' = V' = 0,
    with the lse tangent.  At P = 1 it must be the plain kernel call, bit for
    bit, and match the oracle."""
    kv = np.array([77, 0, 30], np.int32)
    w = W.make_custom(3, 4, 260, 77, 128, seed=43, kv_len=kv,
                      zero_kv_dot_from=0 if zero_kv else None)
    ins = [to_dev(x) for x in w.inputs()]
    if zero_kv:
        ins[4] = ins[5] = None
    kvt = torch.from_numpy(kv).cuda()
    got = ulysses.ulysses_attn_jvp(*ins, scale=w.scale, kv_len=kvt, lse_dot=True, kv_layout="replicated")
    ref = attn_jvp_fwd(*ins, scale=w.scale, kv_len=kvt, lse_dot=True)
    torch.cuda.synchronize()
    for a, b in zip(got, ref):
        assert torch.equal(a, b)
    compare(gpu_rows(*got[:3]), oracle_ref(w), f"ulysses cross P=1 zero_kv={zero_kv}")
