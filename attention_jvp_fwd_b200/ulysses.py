"""Ulysses context parallelism around the attention forward + JVP.

rCM extends the JVP to Ulysses context parallelism by distributing the QKV
tangents with the same all-to-all that Ulysses uses for Q, K and V ("Large
Scale Diffusion Distillation via Score-Regularized Continuous-Time
Consistency", ai.info AI summary, Key Contributions 1 and Methodology in Plain
English).  Each of P ranks holds a contiguous 1/P of the query sequence for
all H heads.  One all-to-all turns that into all of the sequence for H/P
heads; the kernel runs locally; a second all-to-all returns O, O', lse (and
lse') to sequence shards.

Layout: every rank passes [B, H, Lq/P, d] shards of Q and Q' and gets back
[B, H, Lq/P, d] shards of O and O' and [B, H, Lq/P] of lse (and lse').  H
must be a multiple of P.  Rank r's shard holds query positions
[r Lq/P, (r+1) Lq/P).  The keys come in one of two layouts:

* ``kv_layout="seq"`` (self-attention): K, V, K', V' are sequence shards
  [B, H, Lk/P, d] like Q and travel in the same all-to-all.
* ``kv_layout="replicated"`` (cross-attention to text tokens): every rank
  holds the whole key sequence [B, H, Lk, d], as a text encoder's output is
  the same on every rank.  Nothing about the keys is exchanged; each rank
  takes its own H/P heads locally.  Lk is then free (e.g. 512 text tokens
  against thousands of image tokens).

``k_dot = v_dot = None`` means K' = V' = 0 (frozen text tokens): those
tangents are neither exchanged nor multiplied (the zero-tangent kernel).
``kv_len`` (int32 [B], positions in the whole key sequence) masks keys at and
past kv_len[b]; it is the same on every rank.

Every exchange packs all of its tensors, whatever their dtypes, as bytes into
one buffer laid out destination rank first, so a call costs one all-to-all in
and one out.  Each tensor is written into the send buffer by one strided copy
and read out of the receive buffer by one, with no staging copies.  NCCL over
NVLink is the transport on GPUs; the functions only use torch.distributed, so
the exchange is tested with gloo on the CPU.
"""
from __future__ import annotations

import torch
import torch.distributed as dist

_ALIGN = 16  # byte offset of every tensor inside a rank's chunk


def _world(group):
    return dist.get_world_size(group), dist.get_rank(group)


def _all_to_all_packed(sends, recvs, group):
    """One all-to-all of several tensors.  sends[t] and recvs[t] are [P, ...]
    views (any strides, any dtype): sends[t][j] goes to rank j, and
    recvs[t][i] receives what rank i sent as its sends[t][our rank]."""
    P = sends[0].shape[0]
    offs, off = [], 0
    for s in sends:
        offs.append(off)
        nb = s[0].numel() * s.element_size()
        off += (nb + _ALIGN - 1) // _ALIGN * _ALIGN
    chunk = max(off, _ALIGN)
    dev = sends[0].device
    send = torch.empty((P, chunk), dtype=torch.uint8, device=dev)
    recv = torch.empty_like(send)

    def slot(buf, t, like):
        nb = like[0].numel() * like.element_size()
        return buf[:, offs[t]:offs[t] + nb].view(like.dtype).unflatten(1, tuple(like.shape[1:]))

    for t, s in enumerate(sends):
        slot(send, t, s).copy_(s)
    dist.all_to_all_single(recv, send, group=group)
    for t, r in enumerate(recvs):
        r.copy_(slot(recv, t, r))


def seq_to_heads(xs: list[torch.Tensor], group=None) -> list[torch.Tensor]:
    """Sequence shards [B, H, Ls, d] -> head shards [B, H/P, P*Ls, d], all
    tensors in one all-to-all (shapes may differ in Ls and dtype)."""
    P, _ = _world(group)
    sends, outs, recvs = [], [], []
    for x in xs:
        B, H, Ls, d = x.shape
        if H % P:
            raise ValueError(f"H = {H} heads do not split over {P} ranks")
        Hp = H // P
        x = x.contiguous()
        # destination j gets heads [j Hp, (j+1) Hp)
        sends.append(x.view(B, P, Hp, Ls, d).permute(1, 0, 2, 3, 4))
        out = torch.empty((B, Hp, P * Ls, d), dtype=x.dtype, device=x.device)
        # source i sent its sequence shard i of our heads
        recvs.append(out.view(B, Hp, P, Ls, d).permute(2, 0, 1, 3, 4))
        outs.append(out)
    _all_to_all_packed(sends, recvs, group)
    return outs


def heads_to_seq(xs: list[torch.Tensor], group=None) -> list[torch.Tensor]:
    """Head shards [B, H/P, L, d] -> sequence shards [B, H, L/P, d] (the
    inverse of seq_to_heads), all tensors in one all-to-all."""
    P, _ = _world(group)
    sends, outs, recvs = [], [], []
    for x in xs:
        B, Hp, L, d = x.shape
        if L % P:
            raise ValueError(f"L = {L} does not split over {P} ranks")
        Ls = L // P
        x = x.contiguous()
        # destination j gets sequence shard j
        sends.append(x.view(B, Hp, P, Ls, d).permute(2, 0, 1, 3, 4))
        out = torch.empty((B, P * Hp, Ls, d), dtype=x.dtype, device=x.device)
        # source i sent heads [i Hp, (i+1) Hp) of our sequence shard
        recvs.append(out.view(B, P, Hp, Ls, d).permute(1, 0, 2, 3, 4))
        outs.append(out)
    _all_to_all_packed(sends, recvs, group)
    return outs


def _local_heads(x, P, r):
    """Heads [r H/P, (r+1) H/P) of a replicated [B, H, L, d] tensor, dense."""
    if x is None:
        return None
    H = x.shape[1]
    if H % P:
        raise ValueError(f"H = {H} heads do not split over {P} ranks")
    Hp = H // P
    return x[:, r * Hp:(r + 1) * Hp].contiguous()


def ulysses_attn_jvp(q, k, v, q_dot, k_dot, v_dot, group=None, scale=None, kv_len=None,
                     lse_dot: bool = False, kv_layout: str = "seq", local_fn=None):
    """Context-parallel attention forward + JVP over `group`.

    q, q_dot: this rank's query sequence shards [B, H, Lq/P, d] (bf16).
    k, v, k_dot, v_dot: sequence shards [B, H, Lk/P, d] (``kv_layout="seq"``)
    or the whole key sequence [B, H, Lk, d] on every rank
    (``kv_layout="replicated"``); k_dot = v_dot = None for K' = V' = 0.
    kv_len: optional int32 [B] valid key length over the whole key sequence.

    Returns this rank's shards (o, o_dot, lse), plus lse_dot with
    ``lse_dot=True``.  ``local_fn(q, k, v, q_dot, k_dot, v_dot, scale=,
    kv_len=, lse_dot=)`` computes attention on head shards; it defaults to the
    CUDA kernel (``attn_jvp_fwd``).
    """
    if kv_layout not in ("seq", "replicated"):
        raise ValueError("kv_layout must be 'seq' or 'replicated'")
    if (k_dot is None) != (v_dot is None):
        raise ValueError("k_dot and v_dot must both be given or both be None")
    if local_fn is None:
        from .api import attn_jvp_fwd as local_fn
    P, r = _world(group)
    zero_kv = k_dot is None
    if kv_layout == "seq":
        kv = [k, v] + ([] if zero_kv else [k_dot, v_dot])
        got = seq_to_heads([q, q_dot] + kv, group)
        hq, hqd, hk, hv = got[0], got[1], got[2], got[3]
        hkd, hvd = (None, None) if zero_kv else (got[4], got[5])
    else:
        hk, hv, hkd, hvd = (_local_heads(x, P, r) for x in (k, v, k_dot, v_dot))
        hq, hqd = seq_to_heads([q, q_dot], group)
    res = local_fn(hq, hk, hv, hqd, hkd, hvd, scale=scale, kv_len=kv_len, lse_dot=lse_dot)
    o, od, lse = res[0], res[1], res[2]
    backs = [o, od, lse.unsqueeze(-1)] + ([res[3].unsqueeze(-1)] if lse_dot else [])
    outs = heads_to_seq(backs, group)
    so, sod, slse = outs[0], outs[1], outs[2].squeeze(-1)
    if lse_dot:
        return so, sod, slse, outs[3].squeeze(-1)
    return so, sod, slse
