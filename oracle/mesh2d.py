"""Mesh2D: attention over a grid of (query chunk, key chunk) tiles, fp64.

TEST INFRASTRUCTURE ONLY (see ``oracle/__init__.py``).

Mosaic page, "Beyond 1D: Mesh2D Attention": both Q and K are sharded, and on
a grid of devices the device at (i, j) computes the tile of QK^T between
query chunk i and key chunk j (the page draws a 2 x 2 mesh, Q0/Q1 down,
K0/K1 across, and names an 8 x 8 one); per-device memory falls with the
product of the grid sizes.

Readings of what the page leaves open:
- Chunks are contiguous in sequence order: query chunk i holds global
  positions [i * N / grid_q, (i + 1) * N / grid_q), key chunk j (and the
  value rows that go with it) [j * N / grid_k, (j + 1) * N / grid_k).  The
  grid may be rectangular; both sizes must divide N.
- Tile (i, j) produces the partial (O_ij, LSE_ij) of its query rows against
  its keys alone (``attention.attention_forward`` with the tile's global
  positions, so the causal rule is the usual u <= t).  The page shows the
  tiles but not how a row's tiles are combined; the reading taken is the LSE
  merge of the grid_k partials of each query chunk (``merge``), the exact
  identity the ring uses.  A tile with no visible pair has LSE = -inf and
  weight 0.
- Backward (the page shows only the forward): every tile rebuilds its
  probabilities from the final LSE of its rows and uses D_t = dO_t . O_t of
  the final O (as in ``ring``); dQ of chunk i sums over the tiles of row i,
  dK / dV of chunk j over the tiles of column j.
- Packed and right-padded batches: every tile takes the segment ids of its
  global positions (``seg``, as in ``attention``), so a key is visible only
  inside its query's segment; a row with no visible key in a tile has a
  -inf partial there, and one with none in any tile ends with O = 0 and
  LSE = -inf.

Tensors are in global token order: q, dout [B, N, Hq, d]; k, v [B, N, Hkv, d];
lse [B, Hq, N].
"""

from __future__ import annotations

import numpy as np

from . import attention, merge


def check(n: int, grid_q: int, grid_k: int) -> None:
    if grid_q < 1 or grid_k < 1 or n % grid_q or n % grid_k:
        raise ValueError("both grid sizes must be >= 1 and divide N")


def chunk(n: int, grid: int, i: int) -> np.ndarray:
    """Global positions of chunk i of a sequence of n tokens cut into `grid`."""
    size = n // grid
    return np.arange(i * size, (i + 1) * size)


def tile_has_pairs(n: int, grid_q: int, grid_k: int, i: int, j: int, causal: bool) -> bool:
    """Whether tile (i, j) holds a visible (query, key) pair: without the
    causal rule always; with it, when the first key of chunk j is not after
    the last query of chunk i."""
    return (not causal) or chunk(n, grid_k, j)[0] <= chunk(n, grid_q, i)[-1]


def mesh2d_forward(q, k, v, grid_q: int, grid_k: int, causal: bool, scale=None,
                   return_partials=False, seg=None):
    """(o [B, N, Hq, dv], lse [B, Hq, N]); with return_partials also
    partials[i][j] = (o, lse) of tile (i, j) before merging."""
    q = np.asarray(q, dtype=np.float64)
    k = np.asarray(k, dtype=np.float64)
    v = np.asarray(v, dtype=np.float64)
    n = q.shape[1]
    check(n, grid_q, grid_k)
    o = np.zeros(q.shape[:3] + (v.shape[3],))
    lse = np.full((q.shape[0], q.shape[2], n), -np.inf)
    partials = []
    for i in range(grid_q):
        qp = chunk(n, grid_q, i)
        row = []
        for j in range(grid_k):
            kp = chunk(n, grid_k, j)
            row.append(attention.attention_forward(
                q[:, qp], k[:, kp], v[:, kp], scale=scale, causal=causal, q_pos=qp, k_pos=kp,
                seg=seg))
        o_i, lse_i = merge.lse_merge([a for a, _ in row], [b for _, b in row])
        o[:, qp] = o_i
        lse[:, :, qp] = lse_i
        partials.append(row)
    if return_partials:
        return o, lse, partials
    return o, lse


def mesh2d_backward(q, k, v, o, lse, dout, grid_q: int, grid_k: int, causal: bool, scale=None,
                    seg=None):
    """(dq, dk, dv) in global token order, from the final o and lse."""
    q = np.asarray(q, dtype=np.float64)
    k = np.asarray(k, dtype=np.float64)
    v = np.asarray(v, dtype=np.float64)
    dout = np.asarray(dout, dtype=np.float64)
    lse = np.asarray(lse, dtype=np.float64)
    n = q.shape[1]
    check(n, grid_q, grid_k)
    delta = attention.delta_from_output(dout, o)
    dq = np.zeros(q.shape)
    dk = np.zeros(k.shape)
    dv = np.zeros(v.shape)
    for i in range(grid_q):
        qp = chunk(n, grid_q, i)
        for j in range(grid_k):
            kp = chunk(n, grid_k, j)
            gq, gk, gv = attention.attention_backward_block(
                q[:, qp], k[:, kp], v[:, kp], dout[:, qp], lse[:, :, qp], delta[:, :, qp],
                scale=scale, causal=causal, q_pos=qp, k_pos=kp, seg=seg)
            dq[:, qp] += gq
            dk[:, kp] += gk
            dv[:, kp] += gv
    return dq, dk, dv
