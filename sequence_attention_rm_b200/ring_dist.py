"""Ring attention over real ranks: one process per GPU, KV shards passed
around the ring with point-to-point transfers (NCCL over NVLink in
production, any torch.distributed backend), every shard pair computed by the
library's block kernels.

Mosaic, "How Ring Attention Works": each of the P devices keeps its query
chunk and, at step k, attends to the KV chunk it received from its
neighbour, then passes that chunk on; after P steps every query chunk has
met every KV chunk, and the partial results are combined by the LSE merge.
ringmaster, "Status": the point-to-point ring keeps only O(S/P) KV resident,
overlaps the transfer of the next KV block with the current block's compute,
and runs the backward as a ring as well.

Schedule (rank r, P ranks, ``layout`` as in the single-GPU ring):

- forward: at step k rank r holds KV shard s = (r - k) mod P.  It posts the
  send of that shard to rank r + 1 and the receive of shard s - 1 from rank
  r - 1 into a second buffer, computes the block (q_rank r, kv_rank s) into
  an fp32 partial, folds it into its running (O, LSE) with the LSE merge, and
  waits for the transfer before the next step.  Shard pairs the causal rule
  empties are skipped (their KV is still passed on).
- backward: the KV shard travels with fp32 dK / dV accumulators.  At step k
  rank r adds the contributions of pair (r, s) to its own dQ and to the
  travelling dK_s / dV_s, then passes KV and accumulators on (KV is sent
  while the block computes; the accumulators once it is done).  Shard s has
  visited every rank after P steps and sits on rank s - 1; one last transfer
  returns its dK / dV to rank s.

Stream order: point-to-point transfers start after the work already queued
on the current stream and later work on it waits for them, so the block
kernels and the transfers need no host synchronisation.

Operands on rank r are its own shard in the layout's local order:
q, dout [B, L, Hq, d]; k, v [B, L, Hkv, d]; o and lse as the forward
returns them ([B, L, Hq, d] in the input dtype, fp32 [B, Hq, L]).  The
shard-pair arithmetic goes through a ``blocks`` object (``KernelBlocks``,
the library's CUDA kernels, by default), so that the communication schedule
can also be exercised with another implementation of the same operations.
"""

from __future__ import annotations

import torch
import torch.distributed as dist

__all__ = ["KernelBlocks", "ring_forward", "ring_backward", "pair_is_empty"]


class KernelBlocks:
    """The shard-pair operations on the library's CUDA kernels."""

    acc_dtype = torch.float32  # partial O and the gradient accumulators

    def __init__(self):
        from . import rm
        self.rm = rm

    def block_fwd(self, q, k, v, *, N, P, layout, causal, q_rank, kv_rank, scale, segs):
        return self.rm.attn_block_fwd(q, k, v, N=N, P=P, layout=layout, causal=causal,
                                      q_rank=q_rank, kv_rank=kv_rank, scale=scale, o_f32=True,
                                      **segs)

    def merge_into(self, o_acc, lse_acc, o_new, lse_new):
        self.rm.lse_merge([o_acc, o_new], [lse_acc, lse_new], torch.float32, out=o_acc,
                          lse_out=lse_acc)

    def finish(self, o_acc, lse_acc, dtype):
        if dtype == torch.float32:
            return o_acc
        return self.rm.convert_f32(o_acc, dtype)

    def delta(self, o, dout):
        return self.rm.attn_bwd_preprocess(o, dout)

    def block_bwd(self, q, k, v, dout, lse, delta, dq, dk, dv, *, N, P, layout, causal, q_rank,
                  kv_rank, scale, segs):
        self.rm.attn_block_bwd(q, k, v, dout, lse, delta, dq, dk, dv, N=N, P=P, layout=layout,
                               causal=causal, q_rank=q_rank, kv_rank=kv_rank, scale=scale, **segs)

    def cast(self, acc, dtype):
        if dtype == torch.float32:
            return acc
        return self.rm.convert_f32(acc, dtype)


def pair_is_empty(layout: str, N: int, P: int, q_rank: int, kv_rank: int, causal: bool) -> bool:
    """Whether the causal rule hides every key of shard kv_rank from every
    query of shard q_rank: only the contiguous layout has such pairs (a later
    shard's keys all follow an earlier shard's queries); zigzag and striped
    shards interleave, so every pair holds a visible key."""
    return causal and layout == "contiguous" and kv_rank > q_rank


def _exchange(send, recv, dst, src, group):
    """Post sends of `send` to dst and receives into `recv` from src."""
    ops = [dist.P2POp(dist.isend, t, dst, group) for t in send]
    ops += [dist.P2POp(dist.irecv, t, src, group) for t in recv]
    return dist.batch_isend_irecv(ops)


def _receive_buffers(k, v, P):
    """Two (K, V) receive buffers used in turn (one while P = 2): step t
    receives into buffer t mod 2 and computes on the one received at step
    t - 1.  The caller's own k and v are only ever sent, never written."""
    return [[torch.empty_like(k), torch.empty_like(v)] for _ in range(min(P - 1, 2))]


def _wait(reqs):
    for r in reqs:
        r.wait()


def ring_forward(q, k, v, *, layout: str, causal: bool, scale=None, group=None, blocks=None,
                 cu_seqlens=None, seq_lens=None):
    """This rank's (O [B, L, Hq, d] in q's dtype, LSE fp32 [B, Hq, L]).

    cu_seqlens (packing boundaries in global positions, B = 1) or seq_lens
    (right-padding lengths per batch entry), int32, on the operands' device,
    the same on every rank: as in the single-GPU ring, a key is visible only
    inside its query's segment."""
    segs = {"cu_seqlens": cu_seqlens, "seq_lens": seq_lens}
    blocks = KernelBlocks() if blocks is None else blocks
    P = dist.get_world_size(group)
    r = dist.get_rank(group)
    L = q.shape[1]
    N = P * L
    nxt, prv = (r + 1) % P, (r - 1) % P
    # global ranks of the ring neighbours (P2P ops take global ranks)
    dst = dist.get_global_rank(group, nxt) if group is not None else nxt
    src = dist.get_global_rank(group, prv) if group is not None else prv
    bufs = _receive_buffers(k, v, P)
    o_acc = lse_acc = None
    for step in range(P):
        s = (r - step) % P
        cur = [k, v] if step == 0 else bufs[(step - 1) % 2]
        reqs = _exchange(cur, bufs[step % 2], dst, src, group) if step + 1 < P else []
        if not pair_is_empty(layout, N, P, r, s, causal):
            o_s, lse_s = blocks.block_fwd(q, cur[0], cur[1], N=N, P=P, layout=layout,
                                          causal=causal, q_rank=r, kv_rank=s, scale=scale,
                                          segs=segs)
            if o_acc is None:
                o_acc, lse_acc = o_s, lse_s
            else:
                blocks.merge_into(o_acc, lse_acc, o_s, lse_s)
        _wait(reqs)
    # the pair (r, r) is never skipped, so o_acc is set
    return blocks.finish(o_acc, lse_acc, q.dtype), lse_acc


def ring_backward(q, k, v, o, lse, dout, *, layout: str, causal: bool, scale=None, group=None,
                  blocks=None, cu_seqlens=None, seq_lens=None):
    """This rank's (dQ, dK, dV) in the operands' dtypes, from the final O and
    LSE (segments as in ring_forward)."""
    segs = {"cu_seqlens": cu_seqlens, "seq_lens": seq_lens}
    blocks = KernelBlocks() if blocks is None else blocks
    P = dist.get_world_size(group)
    r = dist.get_rank(group)
    L = q.shape[1]
    N = P * L
    nxt, prv = (r + 1) % P, (r - 1) % P
    dst = dist.get_global_rank(group, nxt) if group is not None else nxt
    src = dist.get_global_rank(group, prv) if group is not None else prv
    delta = blocks.delta(o, dout)
    zeros = lambda t: torch.zeros(t.shape, dtype=blocks.acc_dtype, device=t.device)
    dq = zeros(q)
    bufs = _receive_buffers(k, v, P)
    acc = [zeros(k), zeros(v)]
    acc_spare = [zeros(k), zeros(v)] if P > 1 else None
    for step in range(P):
        s = (r - step) % P
        kv = [k, v] if step == 0 else bufs[(step - 1) % 2]
        # KV moves on while the block computes; the accumulators once it is done
        kv_reqs = _exchange(kv, bufs[step % 2], dst, src, group) if step + 1 < P else []
        if not pair_is_empty(layout, N, P, r, s, causal):
            blocks.block_bwd(q, kv[0], kv[1], dout, lse, delta, dq, acc[0], acc[1], N=N, P=P,
                             layout=layout, causal=causal, q_rank=r, kv_rank=s, scale=scale,
                             segs=segs)
        if P > 1:
            # after the last step shard s sits on rank s - 1: this transfer
            # returns every shard's dK / dV to its owner.  (The transfers are
            # ordered after the kernels already queued on the current stream,
            # and waiting on them orders later kernels after the transfers.)
            _wait(_exchange(acc, acc_spare, dst, src, group))
            acc, acc_spare = acc_spare, acc
        _wait(kv_reqs)
    return blocks.cast(dq, q.dtype), blocks.cast(acc[0], k.dtype), blocks.cast(acc[1], v.dtype)
