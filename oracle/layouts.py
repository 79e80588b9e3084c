"""Token layouts over P ranks: global position of each rank-local token.

TEST INFRASTRUCTURE ONLY (see ``oracle/__init__.py``).

Three layouts, each a bijection between global positions t in [0, N) and
(rank r, local index j) pairs, L = N / P tokens per rank:
- contiguous (ringmaster "Layout": shard.py, dense contiguous sequence
  sharding): t = r * L + j;
- zigzag / head_tail (ringmaster "Layout": balancers.py; the rank holding
  chunks i and 2P-1-i): the sequence is cut into 2P chunks of C = N / (2P)
  tokens; rank r holds chunk r, then chunk 2P-1-r, each in increasing order;
- striped ("Ring Attention & Friends", slide "Striped Attention"; token t on
  rank t mod P): local j of rank r is t = j * P + r.

"Rank-major order" is the token axis holding rank 0's local tokens, then rank
1's, and so on; it is how a single device stores the P shards side by side.
"""

from __future__ import annotations

import numpy as np

CONTIGUOUS = "contiguous"
ZIGZAG = "zigzag"
STRIPED = "striped"
LAYOUTS = (CONTIGUOUS, ZIGZAG, STRIPED)


def check(layout: str, n: int, p: int) -> None:
    if layout not in LAYOUTS:
        raise ValueError(f"unknown layout {layout!r}")
    if p < 1 or n % p != 0:
        raise ValueError("N must be a multiple of P")
    if layout == ZIGZAG and n % (2 * p) != 0:
        raise ValueError("zigzag needs N to be a multiple of 2P")


def global_position(layout: str, n: int, p: int, r: int, j: int) -> int:
    """Global position of local token j of rank r (scalar form, the definition)."""
    check(layout, n, p)
    return _position(layout, n, p, r, j)


def _position(layout: str, n: int, p: int, r: int, j: int) -> int:
    local = n // p
    if not (0 <= r < p and 0 <= j < local):
        raise IndexError("rank or local index out of range")
    if layout == CONTIGUOUS:
        return r * local + j
    if layout == STRIPED:
        return j * p + r
    chunk = n // (2 * p)
    if j < chunk:
        return r * chunk + j
    return (2 * p - 1 - r) * chunk + (j - chunk)


def rank_positions(layout: str, n: int, p: int, r: int) -> np.ndarray:
    """Global positions of rank r's local tokens, in local order."""
    check(layout, n, p)
    local = n // p
    return np.array([_position(layout, n, p, r, j) for j in range(local)], dtype=np.int64)


def rank_major_positions(layout: str, n: int, p: int) -> np.ndarray:
    """pos[r * L + j] = global position of local token j of rank r."""
    return np.concatenate([rank_positions(layout, n, p, r) for r in range(p)])


def permute(x, layout: str, p: int, axis: int = 1):
    """Global order -> rank-major order along ``axis`` (a pure gather)."""
    x = np.asarray(x)
    n = x.shape[axis]
    pos = rank_major_positions(layout, n, p)
    return np.take(x, pos, axis=axis)


def unpermute(y, layout: str, p: int, axis: int = 1):
    """Rank-major order -> global order along ``axis`` (a pure scatter)."""
    y = np.asarray(y)
    n = y.shape[axis]
    pos = rank_major_positions(layout, n, p)
    out = np.empty_like(y)
    index = [slice(None)] * y.ndim
    index[axis] = pos
    out[tuple(index)] = y
    return out
