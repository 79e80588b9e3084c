"""Ulysses attention over real ranks: one process per GPU, the sequence <->
head all-to-all done by torch.distributed (NCCL over NVLink in production),
every byte rearrangement and all the attention arithmetic in the library's
kernels.

ringmaster, "Why": Ulysses wraps an attention kernel with an all-to-all on
the head dimension.  Before it each of the P ranks holds a sequence shard of
all H heads; after it each rank holds the whole sequence for H / P heads, so
P may not exceed the number of KV heads; K and V go through the exchange
beside Q.  Attention then runs on the whole sequence for the rank's heads,
and a second all-to-all returns O to sequence shards.

Exchange (rank r, P ranks, local shard [L, H, d] of one batch entry):

- seq -> head: the local pack (rm_seq_head_repack with P parts of L / P
  tokens, applied to the rank's own shard) lays the shard out as P blocks
  [L, H / P, d], block s holding head group s; all_to_all_single sends block
  s to rank s.  Rank r receives, in rank order, every rank's tokens for head
  group r: the whole sequence [P L, H / P, d] in rank-major token order.
- head -> seq: all_to_all_single sends the tokens of rank s (block s of the
  rank-major sequence) to rank s; the received blocks, one per head group,
  are unpacked (rm_seq_head_repack, head -> seq) into [L, H, d].

The attention over the rank-major sequence is the single-GPU ring over P
virtual ranks with the caller's layout, so zigzag / striped sequence
sharding and causal masks by global position carry over unchanged (with
P = 1 and the contiguous layout it is plain attention).  Every batch entry
is exchanged on its own.

Operands on rank r: q, dout [B, L, Hq, d], k, v [B, L, Hkv, d], its shard in
the layout's local order, dense; Hq % P == Hkv % P == L % P == 0.  The
arithmetic goes through an ``ops`` object (``KernelOps``, the CUDA kernels,
by default), so the exchange can also be exercised with another
implementation of the same operations.
"""

from __future__ import annotations

import torch
import torch.distributed as dist

__all__ = ["KernelOps", "seq_to_head", "head_to_seq", "ulysses_forward", "ulysses_backward"]


class KernelOps:
    """Pack / unpack and the attention on the library's CUDA kernels."""

    def __init__(self):
        from . import rm
        self.rm = rm

    def pack(self, x, P):
        """[L, H, d] -> [P, L, H / P, d], block s = head group s."""
        L, H, d = x.shape
        y = self.rm.seq_head_repack(x.contiguous().view(P, L // P, H, d), P)
        return y.view(P, L, H // P, d)

    def unpack(self, y, P):
        """[P, L, H / P, d], block s = head group s -> [L, H, d]."""
        _, L, HP, d = y.shape
        x = self.rm.seq_head_repack(y.contiguous().view(P, L, HP, d), P, head_to_seq=True)
        return x.view(L, HP * P, d)

    def attn_fwd(self, q, k, v, *, P, layout, causal, scale, segs):
        return self.rm.ring_attn_fwd(q, k, v, P=P, layout=layout, causal=causal, scale=scale,
                                     **segs)

    def attn_bwd(self, q, k, v, o, lse, dout, *, P, layout, causal, scale, segs):
        return self.rm.ring_attn_bwd(q, k, v, o, lse, dout, P=P, layout=layout, causal=causal,
                                     scale=scale, **segs)


def _check(x, P):
    B, L, H, d = x.shape
    if H % P or L % P:
        raise ValueError(f"Ulysses over {P} ranks needs heads ({H}) and local tokens ({L}) "
                         f"divisible by {P}")


def seq_to_head(x, *, group=None, ops=None):
    """[B, L, H, d] sequence shard -> [B, P L, H / P, d]: the whole sequence
    (rank-major order) for this rank's head group."""
    ops = KernelOps() if ops is None else ops
    P = dist.get_world_size(group)
    _check(x, P)
    B, L, H, d = x.shape
    out = torch.empty((B, P * L, H // P, d), dtype=x.dtype, device=x.device)
    for b in range(B):
        send = ops.pack(x[b], P)
        dist.all_to_all_single(out[b].view(P, L, H // P, d), send, group=group)
    return out


def head_to_seq(y, *, group=None, ops=None):
    """[B, P L, H / P, d] (this rank's head group, rank-major sequence) ->
    [B, L, H, d] (this rank's tokens, every head)."""
    ops = KernelOps() if ops is None else ops
    P = dist.get_world_size(group)
    B, N, HP, d = y.shape
    L = N // P
    out = torch.empty((B, L, HP * P, d), dtype=y.dtype, device=y.device)
    for b in range(B):
        recv = torch.empty((P, L, HP, d), dtype=y.dtype, device=y.device)
        dist.all_to_all_single(recv, y[b].contiguous().view(P, L, HP, d), group=group)
        out[b] = ops.unpack(recv, P)
    return out


def ulysses_forward(q, k, v, *, layout: str, causal: bool, scale=None, group=None, ops=None,
                    cu_seqlens=None, seq_lens=None):
    """(O [B, L, Hq, d] of this rank's tokens, ctx for ulysses_backward).

    ctx holds the head-sharded operands, O and LSE ([B, Hq / P, P L] fp32,
    rank-major tokens) of this rank's heads.  cu_seqlens / seq_lens: segment
    descriptions by global position, as in the single-GPU ring."""
    ops = KernelOps() if ops is None else ops
    P = dist.get_world_size(group)
    segs = {"cu_seqlens": cu_seqlens, "seq_lens": seq_lens}
    qh = seq_to_head(q, group=group, ops=ops)
    kh = seq_to_head(k, group=group, ops=ops)
    vh = seq_to_head(v, group=group, ops=ops)
    oh, lseh = ops.attn_fwd(qh, kh, vh, P=P, layout=layout, causal=causal, scale=scale, segs=segs)
    o = head_to_seq(oh, group=group, ops=ops)
    ctx = {"q": qh, "k": kh, "v": vh, "o": oh, "lse": lseh, "layout": layout, "causal": causal,
           "scale": scale, "segs": segs}
    return o, ctx


def ulysses_backward(dout, ctx, *, group=None, ops=None):
    """(dQ, dK, dV) of this rank's tokens, in the operands' dtypes."""
    ops = KernelOps() if ops is None else ops
    P = dist.get_world_size(group)
    doh = seq_to_head(dout, group=group, ops=ops)
    dqh, dkh, dvh = ops.attn_bwd(ctx["q"], ctx["k"], ctx["v"], ctx["o"], ctx["lse"], doh, P=P,
                                 layout=ctx["layout"], causal=ctx["causal"], scale=ctx["scale"],
                                 segs=ctx["segs"])
    return tuple(head_to_seq(g, group=group, ops=ops) for g in (dqh, dkh, dvh))
