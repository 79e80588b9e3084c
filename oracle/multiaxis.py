"""Multi-axis attention over a tabular tensor (batch, rows, features, embed), fp64.

TEST INFRASTRUCTURE ONLY (see ``oracle/__init__.py``).

Mosaic page ("Mosaic: Multi-Axis Attention Sharding", "The Implementation"):
attention runs along one chosen axis of a (batch, rows, features, embed)
tensor; the axis is moved to the sequence position, the remaining axes are
flattened into the batch, attention runs, and the original shape is restored.
The embed axis is split into heads of embed / heads channels.

Readings: the learned QKV / output projections of that page are model weights
and are not part of the path, so q, k, v are given directly, each shaped like
the tabular tensor; both axes are non-causal; the scale is 1/sqrt(head dim)
with the true head dimension (24 for embed 96 and 4 heads).

Outputs:
- row axis: o [B, R, F, E]; lse [B, F * heads, R] (head index f * heads + h);
- feature axis: o [B, R, F, E]; lse [B * R, heads, F].
"""

from __future__ import annotations

import numpy as np

from . import attention


def _split_heads(x, heads):
    x = np.asarray(x, dtype=np.float64)
    b, r, f, e = x.shape
    if e % heads != 0:
        raise ValueError("embed must be a multiple of heads")
    return x.reshape(b, r, f, heads, e // heads)


def row_axis_attention(q, k, v, heads: int):
    """Attention along the rows axis; every (batch, feature, head) is one sequence."""
    qs, ks, vs = (_split_heads(t, heads) for t in (q, k, v))
    b, r, f, hh, dh = qs.shape
    # move rows to the sequence position, fold (batch, feature) into the batch
    to_seq = lambda t: np.transpose(t, (0, 2, 1, 3, 4)).reshape(b * f, r, hh, dh)
    o, lse = attention.attention_forward(to_seq(qs), to_seq(ks), to_seq(vs), causal=False)
    o = np.transpose(o.reshape(b, f, r, hh, dh), (0, 2, 1, 3, 4)).reshape(b, r, f, hh * dh)
    lse = lse.reshape(b, f * hh, r)
    return o, lse


def feature_axis_attention(q, k, v, heads: int):
    """Attention along the features axis; every (batch, row, head) is one sequence."""
    qs, ks, vs = (_split_heads(t, heads) for t in (q, k, v))
    b, r, f, hh, dh = qs.shape
    to_seq = lambda t: t.reshape(b * r, f, hh, dh)
    o, lse = attention.attention_forward(to_seq(qs), to_seq(ks), to_seq(vs), causal=False)
    return o.reshape(b, r, f, hh * dh), lse
