"""Ulysses sequence<->head repack as explicit index loops.

TEST INFRASTRUCTURE ONLY (see ``oracle/__init__.py``).

Ulysses (ringmaster "Why") wraps an attention kernel with an all-to-all on the
head dimension: before attention each of the P ranks holds a sequence shard
of all H heads; after the all-to-all each rank holds the whole sequence for
H / P heads (so P may not exceed the head count; the page limits the
Ulysses degree by the number of KV heads).  On one device the all-to-all is a local pack:

    seq -> head:  out[r][s * L + t][h] = in[s][t][r * (H / P) + h]

for ranks r, s in [0, P), local token t in [0, L), head h in [0, H / P): the
output of rank r is the concatenation, in rank order, of every rank's tokens
for head group r.  head -> seq is the inverse.

Shapes: seq-sharded [P, L, H, d]; head-sharded [P, P * L, H / P, d].
"""

from __future__ import annotations

import numpy as np


def seq_to_head(x, p: int):
    x = np.asarray(x)
    if x.ndim != 4 or x.shape[0] != p:
        raise ValueError("input must be [P, L, H, d]")
    _, local, heads, d = x.shape
    if heads % p != 0:
        raise ValueError("H must be a multiple of P")
    hp = heads // p
    out = np.empty((p, p * local, hp, d), dtype=x.dtype)
    for r in range(p):
        for s in range(p):
            for h in range(hp):
                out[r, s * local:(s + 1) * local, h, :] = x[s, :, r * hp + h, :]
    return out


def head_to_seq(y, p: int):
    y = np.asarray(y)
    if y.ndim != 4 or y.shape[0] != p or y.shape[1] % p != 0:
        raise ValueError("input must be [P, P * L, H / P, d]")
    _, n, hp, d = y.shape
    local = n // p
    x = np.empty((p, local, hp * p, d), dtype=y.dtype)
    for r in range(p):
        for s in range(p):
            for h in range(hp):
                x[s, :, r * hp + h, :] = y[r, s * local:(s + 1) * local, h, :]
    return x
