"""Ulysses context parallelism on CPU: gloo ranks exchange sequence shards for
head shards and back, with the fp64 oracle as each rank's local attention.
Rows are independent, so every rank's output shard must equal the oracle on
the whole, unsharded problem, bit for bit.

Cases: self-attention (keys sharded like the queries), cross-attention with
the text keys replicated on every rank (Lk free, ragged kv_len), cross-
attention with sequence-sharded keys of another length, zero key/value
tangents (k_dot = v_dot = None), and the lse tangent."""
import os
import socket

import numpy as np
import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp

from attention_jvp_fwd_b200 import ulysses

SCALE = 0.3


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _full_inputs(B, H, Lq, Lk, d, seed, zero_kv):
    r = np.random.default_rng(seed)
    ins = [r.standard_normal((B, H, L, d)) for L in (Lq, Lk, Lk, Lq, Lk, Lk)]
    if zero_kv:
        ins[4] = np.zeros_like(ins[4])
        ins[5] = np.zeros_like(ins[5])
    return ins


def _oracle_local(q, k, v, qd, kd, vd, scale=None, kv_len=None, lse_dot=False):
    import oracle
    if kd is None:  # K' = V' = 0
        kd = torch.zeros_like(k)
        vd = torch.zeros_like(v)
    arrs = [t.numpy() for t in (q, k, v, qd, kd, vd)]
    kv = None if kv_len is None else kv_len.numpy()
    res = oracle.attn_jvp(*arrs, scale, kv_len=kv, n_threads=1, lse_dot=lse_dot)
    return tuple(torch.from_numpy(x) for x in res)


def _worker(rank, world, port, case, out):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        B, H, Lq, Lk, d = case["shape"]
        layout, zero_kv, want_mu = case["layout"], case["zero_kv"], case["lse_dot"]
        full = _full_inputs(B, H, Lq, Lk, d, 7, zero_kv)
        Lqs = Lq // world
        Lks = Lk // world
        q_sh = [torch.from_numpy(np.ascontiguousarray(x[:, :, rank * Lqs:(rank + 1) * Lqs]))
                for x in (full[0], full[3])]
        if layout == "seq":
            kv_sh = [torch.from_numpy(np.ascontiguousarray(x[:, :, rank * Lks:(rank + 1) * Lks]))
                     for x in (full[1], full[2], full[4], full[5])]
        else:
            kv_sh = [torch.from_numpy(x.copy()) for x in (full[1], full[2], full[4], full[5])]
        k, v, kd, vd = kv_sh
        if zero_kv:
            kd = vd = None
        if case.get("check_exchange"):
            shards = q_sh + kv_sh
            back = ulysses.heads_to_seq(ulysses.seq_to_heads(shards))
            assert all(torch.equal(a, b) for a, b in zip(shards, back))
            heads = ulysses.seq_to_heads(shards)
            Hp = H // world
            for x, h in zip((full[0], full[3], full[1], full[2], full[4], full[5]), heads):
                assert torch.equal(h, torch.from_numpy(x[:, rank * Hp:(rank + 1) * Hp]))
            # mixed dtypes and lengths in one exchange
            mixed = [q_sh[0].float(), q_sh[1], torch.arange(B * H * Lqs, dtype=torch.int32).view(B, H, Lqs, 1)]
            back = ulysses.heads_to_seq(ulysses.seq_to_heads(mixed))
            assert all(a.dtype == b.dtype and torch.equal(a, b) for a, b in zip(mixed, back))
        kv_len = None if case["kv_len"] is None else torch.tensor(case["kv_len"], dtype=torch.int32)
        res = ulysses.ulysses_attn_jvp(q_sh[0], k, v, q_sh[1], kd, vd, scale=SCALE, kv_len=kv_len,
                                       lse_dot=want_mu, kv_layout=layout, local_fn=_oracle_local)
        out[rank] = tuple(x.numpy() for x in res)
    finally:
        dist.destroy_process_group()


CASES = [
    # self-attention, the exchange checked on its own too
    (2, dict(shape=(2, 4, 10, 10, 8), layout="seq", zero_kv=False, lse_dot=False, kv_len=None,
             check_exchange=True)),
    (4, dict(shape=(1, 8, 12, 12, 4), layout="seq", zero_kv=False, lse_dot=True, kv_len=None,
             check_exchange=True)),
    # cross-attention: text keys replicated, ragged valid lengths (0, short, > Lk)
    (2, dict(shape=(3, 4, 10, 7, 8), layout="replicated", zero_kv=False, lse_dot=True,
             kv_len=[7, 0, 3])),
    (4, dict(shape=(2, 8, 12, 5, 4), layout="replicated", zero_kv=False, lse_dot=False,
             kv_len=[2, 9])),
    # frozen text tokens: K' = V' = 0 given as None
    (2, dict(shape=(2, 4, 10, 7, 8), layout="replicated", zero_kv=True, lse_dot=True,
             kv_len=[5, 7])),
    (4, dict(shape=(1, 4, 8, 6, 4), layout="replicated", zero_kv=True, lse_dot=False, kv_len=None)),
    # keys sharded too, at another length than the queries
    (2, dict(shape=(2, 2, 10, 6, 8), layout="seq", zero_kv=True, lse_dot=True, kv_len=[6, 4])),
    (4, dict(shape=(1, 4, 8, 12, 4), layout="seq", zero_kv=False, lse_dot=True, kv_len=[11])),
]


@pytest.mark.parametrize("world,case", CASES)
def test_ulysses_matches_unsharded_oracle(world, case):
    import oracle
    port = _free_port()
    with mp.get_context("spawn").Manager() as m:
        out = m.dict()
        mp.spawn(_worker, args=(world, port, case, out), nprocs=world, join=True)
        res = dict(out)
    B, H, Lq, Lk, d = case["shape"]
    kv = None if case["kv_len"] is None else np.asarray(case["kv_len"], np.int32)
    ref = oracle.attn_jvp(*_full_inputs(B, H, Lq, Lk, d, 7, case["zero_kv"]), SCALE, kv_len=kv,
                          n_threads=1, lse_dot=case["lse_dot"])
    Ls = Lq // world
    names = ("O", "O'", "lse", "lse'")
    for r in range(world):
        assert len(res[r]) == len(ref)
        sl = slice(r * Ls, (r + 1) * Ls)
        for n, got, want in zip(names, res[r], ref):
            assert np.array_equal(got, want[:, :, sl]), f"rank {r}: {n}"


def test_shapes_must_split(monkeypatch):
    """Heads (inbound) and sequence (outbound) must split evenly over the
    ranks; both are checked before any communication, and so are the
    argument combinations the call refuses."""
    monkeypatch.setattr(ulysses, "_world", lambda group: (2, 0))
    with pytest.raises(ValueError):
        ulysses.seq_to_heads([torch.zeros(1, 3, 4, 8)])
    with pytest.raises(ValueError):
        ulysses.heads_to_seq([torch.zeros(1, 2, 5, 8)])
    z = torch.zeros(1, 2, 4, 8)
    with pytest.raises(ValueError):
        ulysses.ulysses_attn_jvp(z, z, z, z, z, None)
    with pytest.raises(ValueError):
        ulysses.ulysses_attn_jvp(z, z, z, z, z, z, kv_layout="ring")
    with pytest.raises(ValueError):
        ulysses.ulysses_attn_jvp(z, torch.zeros(1, 3, 4, 8), z, z, None, None, kv_layout="replicated",
                                 local_fn=lambda *a, **k: None)
