"""The ring over P ranks on one host: forward and backward, fp64.

TEST INFRASTRUCTURE ONLY (see ``oracle/__init__.py``).

Schedule (Mosaic page, "How Ring Attention Works"): rank r starts with its own
KV shard and, at each step, receives the shard of the rank before it in the
ring (in the page's 4-GPU example, GPU 0's second chunk is GPU 3's), so at
step k = 0..P-1 rank r works
with KV shard (r - k) mod P.  Each step produces a partial (O, LSE) for the
rank's query shard; the partials are merged with the LSE merge.

Backward (ringmaster "Status" says the p2p ring has a FlashAttention-like
backward that runs the ring in the opposite direction): every
(query shard, KV shard) pair rebuilds its probabilities from the final LSE of
its query rows and uses the row term D_t = dO_t . O_t of the final O; dQ of a
rank sums over its steps, dK / dV of a shard sum over all ranks that used it
(on real hardware they travel back round the ring; here it is a sum).

``seg`` (segment ids by global position, see ``attention``) restricts every
pair to same-segment keys: packed and right-padded batches.

Tensors are in rank-major order along the token axis (see ``layouts``):
q, dout [B, N, Hq, d]; k, v [B, N, Hkv, d]; lse [B, Hq, N].
"""

from __future__ import annotations

import numpy as np

from . import attention, layouts, merge


def schedule(p: int) -> list[list[int]]:
    """table[r][k] = KV shard used by rank r at ring step k."""
    return [[(r - k) % p for k in range(p)] for r in range(p)]


def _shard(x, r, local):
    return x[:, r * local:(r + 1) * local]


def ring_forward(q, k, v, layout: str, p: int, causal: bool, scale=None, return_partials=False,
                 seg=None):
    """(o, lse) for all ranks; o [B, N, Hq, dv], lse [B, Hq, N], rank-major order.

    With return_partials, also returns partials[r][k] = (o, lse) of rank r at
    step k before merging.
    """
    q = np.asarray(q, dtype=np.float64)
    n = q.shape[1]
    layouts.check(layout, n, p)
    local = n // p
    table = schedule(p)
    pos = [layouts.rank_positions(layout, n, p, r) for r in range(p)]
    o_out, lse_out, partials = [], [], []
    for r in range(p):
        parts = []
        for step in range(p):
            s = table[r][step]
            parts.append(attention.attention_forward(
                _shard(q, r, local), _shard(k, s, local), _shard(v, s, local),
                scale=scale, causal=causal, q_pos=pos[r], k_pos=pos[s], seg=seg))
        o_r, lse_r = merge.lse_merge([a for a, _ in parts], [b for _, b in parts])
        o_out.append(o_r)
        lse_out.append(lse_r)
        partials.append(parts)
    o = np.concatenate(o_out, axis=1)
    lse = np.concatenate(lse_out, axis=2)
    if return_partials:
        return o, lse, partials
    return o, lse


def ring_backward(q, k, v, o, lse, dout, layout: str, p: int, causal: bool, scale=None,
                  seg=None):
    """(dq, dk, dv) in rank-major order, from the final o and lse of the forward."""
    q = np.asarray(q, dtype=np.float64)
    k = np.asarray(k, dtype=np.float64)
    v = np.asarray(v, dtype=np.float64)
    n = q.shape[1]
    layouts.check(layout, n, p)
    local = n // p
    table = schedule(p)
    pos = [layouts.rank_positions(layout, n, p, r) for r in range(p)]
    delta = attention.delta_from_output(dout, o)  # [B, Hq, N]
    dq = np.zeros(q.shape)
    dk = np.zeros(k.shape)
    dv = np.zeros(v.shape)
    for r in range(p):
        rows = slice(r * local, (r + 1) * local)
        for step in range(p):
            s = table[r][step]
            cols = slice(s * local, (s + 1) * local)
            gq, gk, gv = attention.attention_backward_block(
                q[:, rows], k[:, cols], v[:, cols], np.asarray(dout, dtype=np.float64)[:, rows],
                np.asarray(lse)[:, :, rows], delta[:, :, rows],
                scale=scale, causal=causal, q_pos=pos[r], k_pos=pos[s], seg=seg)
            dq[:, rows] += gq
            dk[:, cols] += gk
            dv[:, cols] += gv
    return dq, dk, dv
