"""USP over real ranks: Ulysses inside each ring group, the ring across them,
one process per GPU (torch.distributed for the transfers, the library's
kernels for everything else).

ringmaster, "Why": USP combines the two schemes, a Ulysses all-to-all over
heads inside a group of ranks and a ring over the groups, so the Ulysses
degree stays within the number of KV heads while the ring takes the rest of
the ranks.  This is the multi-rank form of the single-GPU rm_usp_attn_*:

- the world of W = R * U ranks is R ring positions by U Ulysses positions;
  rank w is ring position w // U and Ulysses position w % U (``usp_groups``
  builds the U-rank Ulysses groups and the R-rank ring groups), so a Ulysses
  group is U consecutive ranks: inside one node when U divides the GPUs per
  node, the ring crossing nodes, as the page's 2D mesh places them;
- the sequence is cut into R ring shards by the layout (contiguous, zigzag
  or striped over R), and ring shard r into U contiguous pieces of its local
  order, piece u on rank (r, u);
- the Ulysses all-to-all (ulysses_dist) gives rank (r, u) the whole ring
  shard r for head group u; the ring (ring_dist) over the R ranks of ring
  group u runs on those shards; the reverse all-to-all returns O (and in the
  backward dQ, dK, dV) to the pieces.

Operands on rank (r, u): q, dout [B, L, Hq, d], k, v [B, L, Hkv, d] with
L = N / (R U), its piece in local order; Hq, Hkv divisible by U.
"""

from __future__ import annotations

import torch.distributed as dist

from . import ring_dist, ulysses_dist

__all__ = ["usp_groups", "rank_piece", "usp_forward", "usp_backward"]


def usp_groups(ulysses: int, backend=None):
    """(Ulysses group, ring group) of this rank.  Every rank must call this
    with the same degree: it creates all R + U groups in the same order."""
    W, me = dist.get_world_size(), dist.get_rank()
    if ulysses < 1 or W % ulysses:
        raise ValueError(f"the Ulysses degree {ulysses} must divide the world size {W}")
    R = W // ulysses
    u_group = r_group = None
    for r in range(R):
        g = dist.new_group([r * ulysses + u for u in range(ulysses)], backend=backend)
        if me // ulysses == r:
            u_group = g
    for u in range(ulysses):
        g = dist.new_group([r * ulysses + u for r in range(R)], backend=backend)
        if me % ulysses == u:
            r_group = g
    return u_group, r_group


def rank_piece(ring_shard_positions, ulysses: int, u: int):
    """The positions of Ulysses position u's piece of a ring shard (given in
    the shard's local order)."""
    L = len(ring_shard_positions) // ulysses
    return ring_shard_positions[u * L:(u + 1) * L]


def usp_forward(q, k, v, *, layout: str, causal: bool, ulysses_group, ring_group, scale=None,
                blocks=None, ops=None, cu_seqlens=None, seq_lens=None):
    """(O [B, L, Hq, d] of this rank's piece, ctx for usp_backward)."""
    segs = {"cu_seqlens": cu_seqlens, "seq_lens": seq_lens}
    qh = ulysses_dist.seq_to_head(q, group=ulysses_group, ops=ops)
    kh = ulysses_dist.seq_to_head(k, group=ulysses_group, ops=ops)
    vh = ulysses_dist.seq_to_head(v, group=ulysses_group, ops=ops)
    oh, lseh = ring_dist.ring_forward(qh, kh, vh, layout=layout, causal=causal, scale=scale,
                                      group=ring_group, blocks=blocks, **segs)
    o = ulysses_dist.head_to_seq(oh, group=ulysses_group, ops=ops)
    ctx = {"q": qh, "k": kh, "v": vh, "o": oh, "lse": lseh, "layout": layout, "causal": causal,
           "scale": scale, "segs": segs}
    return o, ctx


def usp_backward(dout, ctx, *, ulysses_group, ring_group, blocks=None, ops=None):
    """(dQ, dK, dV) of this rank's piece, in the operands' dtypes."""
    doh = ulysses_dist.seq_to_head(dout, group=ulysses_group, ops=ops)
    grads = ring_dist.ring_backward(ctx["q"], ctx["k"], ctx["v"], ctx["o"], ctx["lse"], doh,
                                    layout=ctx["layout"], causal=ctx["causal"],
                                    scale=ctx["scale"], group=ring_group, blocks=blocks,
                                    **ctx["segs"])
    return tuple(ulysses_dist.head_to_seq(g, group=ulysses_group, ops=ops) for g in grads)
