"""Ulysses context parallelism on CPU: gloo ranks exchange sequence shards for
head shards and back, with the fp64 oracle as each rank's local attention.
Rows are independent, so every rank's output shard must equal the oracle on
the whole, unsharded problem, bit for bit."""
import os
import socket

import numpy as np
import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp

from attention_jvp_fwd_b200 import ulysses


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _full_inputs(B, H, L, d, seed):
    r = np.random.default_rng(seed)
    return [r.standard_normal((B, H, L, d)) for _ in range(6)]


def _oracle_local(q, k, v, qd, kd, vd, scale=None):
    import oracle
    arrs = [t.numpy() for t in (q, k, v, qd, kd, vd)]
    o, od, lse = oracle.attn_jvp(*arrs, scale, n_threads=1)
    return torch.from_numpy(o), torch.from_numpy(od), torch.from_numpy(lse)


def _worker(rank, world, port, shape, out):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        B, H, L, d = shape
        full = _full_inputs(B, H, L, d, seed=7)
        Ls = L // world
        shards = [torch.from_numpy(np.ascontiguousarray(x[:, :, rank * Ls:(rank + 1) * Ls]))
                  for x in full]
        # the exchange alone: there and back again is the identity
        back = ulysses.heads_to_seq(ulysses.seq_to_heads(shards))
        assert all(torch.equal(a, b) for a, b in zip(shards, back))
        heads = ulysses.seq_to_heads(shards)
        Hp = H // world
        for x, h in zip(full, heads):
            assert torch.equal(h, torch.from_numpy(x[:, rank * Hp:(rank + 1) * Hp]))
        # the whole context-parallel call
        o, od, lse = ulysses.ulysses_attn_jvp(*shards, scale=0.3, local_fn=_oracle_local)
        out[rank] = (o.numpy(), od.numpy(), lse.numpy())
    finally:
        dist.destroy_process_group()


@pytest.mark.parametrize("world,shape", [(2, (2, 4, 10, 8)), (4, (1, 8, 12, 4))])
def test_ulysses_matches_unsharded_oracle(world, shape):
    import oracle
    port = _free_port()
    with mp.Manager() as m:
        out = m.dict()
        mp.spawn(_worker, args=(world, port, shape, out), nprocs=world, join=True)
        res = dict(out)
    B, H, L, d = shape
    ro, rod, rl = oracle.attn_jvp(*_full_inputs(B, H, L, d, seed=7), 0.3, n_threads=1)
    Ls = L // world
    for r in range(world):
        o, od, lse = res[r]
        sl = slice(r * Ls, (r + 1) * Ls)
        assert np.array_equal(o, ro[:, :, sl]), f"rank {r}: O"
        assert np.array_equal(od, rod[:, :, sl]), f"rank {r}: O'"
        assert np.array_equal(lse, rl[:, :, sl]), f"rank {r}: lse"


def test_shapes_must_split(monkeypatch):
    """Heads (inbound) and sequence (outbound) must split evenly over the
    ranks; both are checked before any communication."""
    monkeypatch.setattr(ulysses, "_world", lambda group: (2, 0))
    with pytest.raises(ValueError):
        ulysses.seq_to_heads([torch.zeros(1, 3, 4, 8)])
    with pytest.raises(ValueError):
        ulysses.heads_to_seq([torch.zeros(1, 2, 5, 8)])
