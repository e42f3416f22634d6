"""Ulysses context parallelism around the attention forward + JVP.

rCM extends the JVP to Ulysses context parallelism by distributing the QKV
tangents with the same all-to-all that Ulysses uses for Q, K and V ("Large
Scale Diffusion Distillation via Score-Regularized Continuous-Time
Consistency", ai.info AI summary, Key Contributions 1 and Methodology in Plain
English).  Each of P ranks holds a contiguous 1/P of the sequence for all H
heads.  One all-to-all turns that into all of the sequence for H/P heads; the
kernel runs locally; a second all-to-all returns O, O' and lse to sequence
shards.

Layout: every rank passes [B, H, L/P, d] shards of Q, K, V and their
tangents (self-attention: the same L/P for queries and keys) and gets back
[B, H, L/P, d] shards of O and O' and [B, H, L/P] of lse.  H must be a
multiple of P.  Rank r's shard holds sequence positions [r L/P, (r+1) L/P).

The exchange packs the six inputs into one buffer, [P, 6, B, H/P, L/P, d]
with the destination rank first, so a call costs one all-to-all in and two
out (O and O' together, lse on its own in fp32).  NCCL over NVLink is the
transport on GPUs; the functions are backend-agnostic, so the exchange can be
tested with gloo on the CPU.
"""
from __future__ import annotations

import torch
import torch.distributed as dist


def _world(group):
    return dist.get_world_size(group), dist.get_rank(group)


def seq_to_heads(xs: list[torch.Tensor], group=None) -> list[torch.Tensor]:
    """Sequence shards [B, H, Ls, d] (same shape, same dtype) -> head shards
    [B, H/P, P*Ls, d], all tensors in one all-to-all."""
    P, _ = _world(group)
    B, H, Ls, d = xs[0].shape
    if H % P:
        raise ValueError(f"H = {H} heads do not split over {P} ranks")
    Hp = H // P
    n = len(xs)
    # [n, B, P, Hp, Ls, d] -> [P, n, B, Hp, Ls, d]: destination rank j gets heads j*Hp..
    send = torch.stack(xs).reshape(n, B, P, Hp, Ls, d).permute(2, 0, 1, 3, 4, 5).contiguous()
    recv = torch.empty_like(send)
    dist.all_to_all_single(recv, send, group=group)
    # recv[i] came from rank i: its sequence shard i of our heads -> [n, B, Hp, P*Ls, d]
    out = recv.permute(1, 2, 3, 0, 4, 5).reshape(n, B, Hp, P * Ls, d)
    return [out[i].contiguous() for i in range(n)]


def heads_to_seq(xs: list[torch.Tensor], group=None) -> list[torch.Tensor]:
    """Head shards [B, H/P, L, d] -> sequence shards [B, H, L/P, d] (the
    inverse of seq_to_heads), all tensors in one all-to-all."""
    P, _ = _world(group)
    B, Hp, L, d = xs[0].shape
    if L % P:
        raise ValueError(f"L = {L} does not split over {P} ranks")
    Ls = L // P
    n = len(xs)
    # [n, B, Hp, P, Ls, d] -> [P, n, B, Hp, Ls, d]: destination rank j gets sequence shard j
    send = torch.stack(xs).reshape(n, B, Hp, P, Ls, d).permute(3, 0, 1, 2, 4, 5).contiguous()
    recv = torch.empty_like(send)
    dist.all_to_all_single(recv, send, group=group)
    # recv[i] came from rank i: heads i*Hp.. of our sequence shard -> [n, B, P*Hp, Ls, d]
    out = recv.permute(1, 2, 0, 3, 4, 5).reshape(n, B, P * Hp, Ls, d)
    return [out[i].contiguous() for i in range(n)]


def ulysses_attn_jvp(q, k, v, q_dot, k_dot, v_dot, group=None, scale=None, local_fn=None):
    """Context-parallel attention forward + JVP over `group`.

    Inputs are this rank's sequence shards [B, H, L/P, d] (bf16).  Returns
    this rank's shards (o, o_dot, lse).  ``local_fn(q, k, v, q_dot, k_dot,
    v_dot, scale)`` computes attention on head shards; it defaults to the CUDA
    kernel (``attn_jvp_fwd``).
    """
    if local_fn is None:
        from .api import attn_jvp_fwd

        def local_fn(*args, scale=None):
            return attn_jvp_fwd(*args, scale=scale)
    hq, hk, hv, hqd, hkd, hvd = seq_to_heads([q, k, v, q_dot, k_dot, v_dot], group)
    o, od, lse = local_fn(hq, hk, hv, hqd, hkd, hvd, scale=scale)
    so, sod = heads_to_seq([o, od], group)
    (slse,) = heads_to_seq([lse.unsqueeze(-1)], group)
    return so, sod, slse.squeeze(-1)
