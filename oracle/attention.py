"""Exact attention on one (query set, key set) pair, forward and backward, fp64.

TEST INFRASTRUCTURE ONLY (see ``oracle/__init__.py``).

Definition followed (Mosaic page, "The Problem"): Attention(Q, K, V) =
softmax(Q K^T / sqrt(d)) V, where the softmax runs over the key axis of each
query row; the per-row normaliser of that softmax ("Ring Attention & Friends",
slide "Vanilla Transformer", which names the per-row constant that normalises
the softmax) is
reported as its natural logarithm, the LSE.

Tensor layout (tokens-major, "bshd"): q [B, Nq, Hq, d], k [B, Nk, Hkv, d],
v [B, Nk, Hkv, dv]; outputs o [B, Nq, Hq, dv], lse [B, Hq, Nq].

Readings of points the pages leave open:
- scale is 1/sqrt(d) with d the true head dimension;
- LSE is the natural log of sum_u exp(s_tu) over the visible keys;
- causal: key at global position u is visible to the query at global position
  t iff u <= t (diagonal inclusive; ringmaster "Status" accepts causal
  sequences without holes or arbitrary masks).  Global positions are passed in explicitly so that the same
  function serves any shard pair of any layout;
- grouped-query attention: query head h reads KV head h // (Hq // Hkv)
  (contiguous groups; ringmaster "Quickstart" only names num_kv_heads);
- a query row with no visible key has o = 0 and lse = -inf;
- packed and right-padded batches (ringmaster "Status": attention takes dense
  causal sequences or globally right-padded batches; packed attention uses
  global position boundaries): ``seg`` gives every global position of every
  batch entry a segment id, -1 for padding.  A key is visible to a query only
  inside the query's segment (and, if causal, not after it); padding tokens
  see nothing and are seen by nothing.

The full score row of each query is materialised; queries are processed in
row blocks only to bound host memory.  No online softmax is used.
"""

from __future__ import annotations

import math

import numpy as np

_ELEMS_PER_BLOCK = 1 << 24  # score elements per row block (128 MiB of fp64)


def default_scale(d: int) -> float:
    """1/sqrt(d) (Mosaic page, "The Problem")."""
    return 1.0 / math.sqrt(d)


def kv_head_of(h: int, hq: int, hkv: int) -> int:
    """KV head read by query head h under grouped-query attention."""
    if hq % hkv != 0:
        raise ValueError("Hq must be a multiple of Hkv")
    return h // (hq // hkv)


def visible(q_pos: np.ndarray, k_pos: np.ndarray, causal: bool, q_seg=None,
            k_seg=None) -> np.ndarray:
    """Boolean [Nq, Nk]: may query at global position q_pos[i] see key k_pos[j].
    q_seg / k_seg: segment ids of those positions (-1 = padding), or None."""
    if not causal:
        vis = np.ones((len(q_pos), len(k_pos)), dtype=bool)
    else:
        vis = k_pos[None, :] <= q_pos[:, None]
    if q_seg is not None:
        vis = vis & (k_seg[None, :] == q_seg[:, None]) & (k_seg[None, :] >= 0)
    return vis


def segments_from_boundaries(cu, n: int) -> np.ndarray:
    """Segment id of each of n global positions from boundaries
    0 = cu[0] < cu[1] < ... < cu[S] <= n (packing); positions >= cu[S] are
    padding (-1).  Shape [n]."""
    cu = np.asarray(cu, dtype=np.int64)
    seg = np.full(n, -1, dtype=np.int64)
    for i in range(len(cu) - 1):
        seg[cu[i]:cu[i + 1]] = i
    return seg


def segments_from_lengths(lengths, n: int) -> np.ndarray:
    """Right padding: batch entry b holds lengths[b] valid tokens, then
    padding.  Shape [B, n]."""
    lengths = np.asarray(lengths, dtype=np.int64)
    seg = np.full((len(lengths), n), -1, dtype=np.int64)
    for b, length in enumerate(lengths):
        seg[b, :length] = 0
    return seg


def _segs(seg, b, q_pos, k_pos):
    if seg is None:
        return None, None
    row = np.asarray(seg)[b] if np.ndim(seg) == 2 else np.asarray(seg)
    return row[q_pos], row[k_pos]


def _prepare(q, k, v, scale, q_pos, k_pos):
    q = np.asarray(q, dtype=np.float64)
    k = np.asarray(k, dtype=np.float64)
    v = np.asarray(v, dtype=np.float64)
    if q.ndim != 4 or k.ndim != 4 or v.ndim != 4:
        raise ValueError("q, k, v must be [B, N, H, d]")
    B, nq, hq, d = q.shape
    if k.shape[0] != B or v.shape[0] != B or k.shape[1] != v.shape[1]:
        raise ValueError("batch / key-length mismatch")
    if k.shape[3] != d or k.shape[2] != v.shape[2]:
        raise ValueError("head-dim / kv-head mismatch")
    nk = k.shape[1]
    if scale is None:
        scale = default_scale(d)
    q_pos = np.arange(nq, dtype=np.int64) if q_pos is None else np.asarray(q_pos, dtype=np.int64)
    k_pos = np.arange(nk, dtype=np.int64) if k_pos is None else np.asarray(k_pos, dtype=np.int64)
    if q_pos.shape != (nq,) or k_pos.shape != (nk,):
        raise ValueError("position arrays must match the token axes")
    return q, k, v, float(scale), q_pos, k_pos


def _row_blocks(nq: int, nk: int):
    step = max(1, _ELEMS_PER_BLOCK // max(nk, 1))
    for r0 in range(0, nq, step):
        yield r0, min(nq, r0 + step)


def _softmax_rows(s: np.ndarray, vis: np.ndarray):
    """Softmax of each row of s over its visible entries, plus the row LSE.

    Two passes over the materialised row: the max shift, then the sum.  Rows
    with no visible entry get probabilities 0 and LSE -inf.
    """
    s = np.where(vis, s, -np.inf)
    any_vis = vis.any(axis=1)
    m = np.where(any_vis, s.max(axis=1, initial=-np.inf), 0.0)
    e = np.exp(s - m[:, None])  # exp(-inf) == 0 for hidden keys
    den = e.sum(axis=1)
    safe_den = np.where(any_vis, den, 1.0)
    probs = e / safe_den[:, None]
    lse = np.where(any_vis, m + np.log(safe_den), -np.inf)
    return probs, lse


def attention_forward(q, k, v, scale=None, causal=False, q_pos=None, k_pos=None, seg=None):
    """(o, lse) of softmax(q k^T * scale) v with optional causal mask.

    seg: segment ids [B, N] or [N] by global position (see the module
    docstring), or None.  Returns o [B, Nq, Hq, dv] float64 and lse
    [B, Hq, Nq] float64.
    """
    q, k, v, scale, q_pos, k_pos = _prepare(q, k, v, scale, q_pos, k_pos)
    B, nq, hq, _ = q.shape
    nk, hkv, dv = k.shape[1], k.shape[2], v.shape[3]
    o = np.zeros((B, nq, hq, dv))
    lse = np.full((B, hq, nq), -np.inf)
    for b in range(B):
        qs, ks = _segs(seg, b, q_pos, k_pos)
        for h in range(hq):
            g = kv_head_of(h, hq, hkv)
            kk, vv = k[b, :, g, :], v[b, :, g, :]
            for r0, r1 in _row_blocks(nq, nk):
                s = (q[b, r0:r1, h, :] @ kk.T) * scale
                vis = visible(q_pos[r0:r1], k_pos, causal,
                              None if qs is None else qs[r0:r1], ks)
                probs, row_lse = _softmax_rows(s, vis)
                o[b, r0:r1, h, :] = probs @ vv
                lse[b, h, r0:r1] = row_lse
    return o, lse


def attention_probabilities(q, k, scale=None, causal=False, q_pos=None, k_pos=None):
    """The full softmax matrix [B, Hq, Nq, Nk] (small inputs only)."""
    v = np.zeros(np.shape(k)[:3] + (1,))
    q, k, v, scale, q_pos, k_pos = _prepare(q, k, v, scale, q_pos, k_pos)
    B, nq, hq, _ = q.shape
    nk, hkv = k.shape[1], k.shape[2]
    out = np.zeros((B, hq, nq, nk))
    for b in range(B):
        for h in range(hq):
            g = kv_head_of(h, hq, hkv)
            s = (q[b, :, h, :] @ k[b, :, g, :].T) * scale
            out[b, h], _ = _softmax_rows(s, visible(q_pos, k_pos, causal))
    return out


def delta_from_output(dout, o):
    """D[b, h, t] = sum_c dO[b, t, h, c] * O[b, t, h, c], shape [B, Hq, Nq].

    Equal to sum_u P_tu dP_tu (the row term of the softmax derivative) because
    O_t = sum_u P_tu v_u; the ring backward uses this form with the final O.
    """
    dout = np.asarray(dout, dtype=np.float64)
    o = np.asarray(o, dtype=np.float64)
    return np.einsum("bthc,bthc->bht", dout, o)


def attention_backward_block(q, k, v, dout, lse, delta, scale=None, causal=False,
                             q_pos=None, k_pos=None, seg=None):
    """Gradient contributions of one (query set, key set) pair.

    The probabilities are rebuilt from the given row LSE (the LSE of the whole
    key set of each query, not of this block), P_tu = exp(s_tu - lse_t), and
    delta is the given row term D_t.  Then, for this pair:
        dV_u += sum_t P_tu dO_t
        dP_tu = dO_t . v_u
        dS_tu = P_tu (dP_tu - D_t)
        dQ_t += scale * sum_u dS_tu k_u
        dK_u += scale * sum_t dS_tu q_t
    dK / dV of a KV head sum over the query heads of its group.
    Returns dq [B,Nq,Hq,d], dk [B,Nk,Hkv,d], dv [B,Nk,Hkv,dv] (float64).
    """
    q, k, v, scale, q_pos, k_pos = _prepare(q, k, v, scale, q_pos, k_pos)
    dout = np.asarray(dout, dtype=np.float64)
    lse = np.asarray(lse, dtype=np.float64)
    delta = np.asarray(delta, dtype=np.float64)
    B, nq, hq, _ = q.shape
    nk, hkv = k.shape[1], k.shape[2]
    if dout.shape != q.shape[:3] + (v.shape[3],):
        raise ValueError("dout must have the shape of o")
    if lse.shape != (B, hq, nq) or delta.shape != (B, hq, nq):
        raise ValueError("lse / delta must be [B, Hq, Nq]")
    dq = np.zeros(q.shape)
    dk = np.zeros(k.shape)
    dv = np.zeros(v.shape)
    for b in range(B):
        qs, ks = _segs(seg, b, q_pos, k_pos)
        for h in range(hq):
            g = kv_head_of(h, hq, hkv)
            kk, vv = k[b, :, g, :], v[b, :, g, :]
            for r0, r1 in _row_blocks(nq, nk):
                qq = q[b, r0:r1, h, :]
                do = dout[b, r0:r1, h, :]
                s = (qq @ kk.T) * scale
                vis = visible(q_pos[r0:r1], k_pos, causal,
                              None if qs is None else qs[r0:r1], ks)
                with np.errstate(over="ignore", invalid="ignore"):
                    probs = np.where(vis, np.exp(s - lse[b, h, r0:r1, None]), 0.0)
                dv[b, :, g, :] += probs.T @ do
                dp = do @ vv.T
                ds = probs * (dp - delta[b, h, r0:r1, None])
                dq[b, r0:r1, h, :] += scale * (ds @ kk)
                dk[b, :, g, :] += scale * (ds.T @ qq)
    return dq, dk, dv


def attention_backward(q, k, v, dout, scale=None, causal=False, q_pos=None, k_pos=None,
                       seg=None):
    """(dq, dk, dv) of sum(dout * attention_forward(q, k, v)[0]).

    D_t is taken straight from the definition, D_t = sum_u P_tu dP_tu, with the
    probabilities of the full key set; no shortcut through O is used here.
    """
    q, k, v, scale, q_pos, k_pos = _prepare(q, k, v, scale, q_pos, k_pos)
    dout = np.asarray(dout, dtype=np.float64)
    B, nq, hq, _ = q.shape
    nk, hkv = k.shape[1], k.shape[2]
    _, lse = attention_forward(q, k, v, scale, causal, q_pos, k_pos, seg)
    delta = np.zeros((B, hq, nq))
    for b in range(B):
        qs, ks = _segs(seg, b, q_pos, k_pos)
        for h in range(hq):
            g = kv_head_of(h, hq, hkv)
            for r0, r1 in _row_blocks(nq, nk):
                s = (q[b, r0:r1, h, :] @ k[b, :, g, :].T) * scale
                vis = visible(q_pos[r0:r1], k_pos, causal,
                              None if qs is None else qs[r0:r1], ks)
                probs, _ = _softmax_rows(s, vis)
                dp = dout[b, r0:r1, h, :] @ v[b, :, g, :].T
                delta[b, h, r0:r1] = (probs * dp).sum(axis=1)
    return attention_backward_block(q, k, v, dout, lse, delta, scale, causal, q_pos, k_pos, seg)
