"""USP: the Ulysses head all-to-all composed with the ring, on one host, fp64.

TEST INFRASTRUCTURE ONLY (see ``oracle/__init__.py``).

ringmaster "Why": USP lays the ranks out on a 2-D mesh, Ulysses exchanging
heads along one axis and the ring passing KV along the other, and an
auto-selector chooses the (Ulysses degree x ring degree) split from the KV-head
count and the world size.

Readings of what the page leaves open:
- The sequence is first laid out over the p_ring ring ranks by the layout
  (tensors here are rank-major for p_ring, as in ``ring``); ring shard r is
  then cut into p_ulysses contiguous sub-shards, one per device (r, u).
- Ulysses inside ring group r: the seq->head repack of the group's
  [p_ulysses, L_r / p_ulysses, H, d] sub-shards (``repack.seq_to_head``), after
  which device (r, u) holds all of ring shard r for head group u.
- The ring then runs over r for every head group u (``ring``), on the query
  and KV heads of that group; grouped-query attention keeps its grouping
  because both head counts are divided by p_ulysses.
- The outputs go back with the head->seq repack inside every ring group.
- Auto-selection (``auto_select``): the largest Ulysses degree that divides the
  world size and the KV-head count (the Ulysses cap) and fits in one node;
  the ring degree is the rest of the world.
- Packed and right-padded batches (ringmaster "Status": packing by global
  position boundaries works whatever the context-parallel strategy): the
  head exchange moves whole heads and keeps every token's global position,
  so each head group's ring takes the same segment ids (``seg``, by global
  position, as in ``attention``) as the unsharded problem.
"""

from __future__ import annotations

import numpy as np

from . import repack, ring


def auto_select(hq: int, hkv: int, world: int, node_size: int = 8) -> tuple[int, int]:
    """(ulysses, ring) with ulysses * ring == world."""
    if hq % hkv:
        raise ValueError("Hq must be a multiple of Hkv")
    best = 1
    for u in range(1, world + 1):
        if world % u == 0 and hkv % u == 0 and u <= node_size:
            best = u
    return best, world // best


def _check(n: int, hq: int, hkv: int, p_ring: int, p_ulysses: int) -> None:
    if n % p_ring or (n // p_ring) % p_ulysses:
        raise ValueError("N must split into p_ring shards of p_ulysses sub-shards")
    if hq % p_ulysses or hkv % p_ulysses:
        raise ValueError("p_ulysses must divide the query and the KV head counts")


def _seq_to_head(x, p_ring: int, p_ulysses: int):
    """[B, N, H, d] -> [B, p_ulysses, N, H / p_ulysses, d]: the Ulysses repack
    inside every ring group, ring shards kept in rank order."""
    x = np.asarray(x)
    b_, n, h, d = x.shape
    lr = n // p_ring
    out = np.empty((b_, p_ulysses, n, h // p_ulysses, d), dtype=x.dtype)
    for b in range(b_):
        for r in range(p_ring):
            shard = x[b, r * lr:(r + 1) * lr].reshape(p_ulysses, lr // p_ulysses, h, d)
            out[b, :, r * lr:(r + 1) * lr] = repack.seq_to_head(shard, p_ulysses)
    return out


def _head_to_seq(y, p_ring: int, p_ulysses: int):
    """Inverse of ``_seq_to_head``."""
    y = np.asarray(y)
    b_, _, n, hp, d = y.shape
    lr = n // p_ring
    out = np.empty((b_, n, hp * p_ulysses, d), dtype=y.dtype)
    for b in range(b_):
        for r in range(p_ring):
            seq = repack.head_to_seq(y[b, :, r * lr:(r + 1) * lr], p_ulysses)
            out[b, r * lr:(r + 1) * lr] = seq.reshape(lr, hp * p_ulysses, d)
    return out


def _seg_of(seg, b):
    """Segment ids of batch entry b: seg is None, [N] (shared) or [B, N]."""
    if seg is None:
        return None
    seg = np.asarray(seg)
    return seg[b] if seg.ndim == 2 else seg


def usp_forward(q, k, v, layout: str, p_ring: int, p_ulysses: int, causal: bool, scale=None,
                seg=None):
    """(o, lse): o [B, N, Hq, d] rank-major for p_ring, lse [B, Hq, N]."""
    q = np.asarray(q, dtype=np.float64)
    b_, n, hq, d = q.shape
    hkv = np.shape(k)[2]
    _check(n, hq, hkv, p_ring, p_ulysses)
    yq, yk, yv = (_seq_to_head(x, p_ring, p_ulysses) for x in (q, k, v))
    hg = hq // p_ulysses
    yo = np.empty_like(yq)
    lse = np.empty((b_, hq, n))
    for b in range(b_):
        for u in range(p_ulysses):
            o_u, l_u = ring.ring_forward(yq[b, u][None], yk[b, u][None], yv[b, u][None], layout,
                                         p_ring, causal, scale, seg=_seg_of(seg, b))
            yo[b, u] = o_u[0]
            lse[b, u * hg:(u + 1) * hg] = l_u[0]
    return _head_to_seq(yo, p_ring, p_ulysses), lse


def usp_backward(q, k, v, o, lse, dout, layout: str, p_ring: int, p_ulysses: int, causal: bool,
                 scale=None, seg=None):
    """(dq, dk, dv) rank-major for p_ring, from the final o and lse."""
    q = np.asarray(q, dtype=np.float64)
    b_, n, hq, d = q.shape
    hkv = np.shape(k)[2]
    _check(n, hq, hkv, p_ring, p_ulysses)
    yq, yk, yv, yo, ydo = (_seq_to_head(np.asarray(x, dtype=np.float64), p_ring, p_ulysses)
                           for x in (q, k, v, o, dout))
    hg = hq // p_ulysses
    lse = np.asarray(lse, dtype=np.float64)
    ydq, ydk, ydv = np.empty_like(yq), np.empty_like(yk), np.empty_like(yv)
    for b in range(b_):
        for u in range(p_ulysses):
            gq, gk, gv = ring.ring_backward(yq[b, u][None], yk[b, u][None], yv[b, u][None],
                                            yo[b, u][None], lse[b, u * hg:(u + 1) * hg][None],
                                            ydo[b, u][None], layout, p_ring, causal, scale,
                                            seg=_seg_of(seg, b))
            ydq[b, u], ydk[b, u], ydv[b, u] = gq[0], gk[0], gv[0]
    return (_head_to_seq(ydq, p_ring, p_ulysses), _head_to_seq(ydk, p_ring, p_ulysses),
            _head_to_seq(ydv, p_ring, p_ulysses))
