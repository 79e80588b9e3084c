"""LSE merge of partial (O, LSE) results, fp64.

TEST INFRASTRUCTURE ONLY (see ``oracle/__init__.py``).

Ring attention computes, for one query shard, a partial result against each
KV shard and combines them at the end (Mosaic page, "How Ring Attention
Works": compute partial attention, accumulate, normalise at the end;
ringmaster "Layout": ring/merge.py, the online-softmax LSE merge).  The pages
do not print the merge formula (the slide formulas were lost); the reading
taken is the exact identity that follows from the definition of the LSE:

    LSE = m + ln sum_i exp(LSE_i - m),   m = max_i LSE_i
    O   = sum_i exp(LSE_i - LSE) * O_i

A partial with LSE_i = -inf (no visible key) has weight 0; if every partial is
-inf the result is O = 0, LSE = -inf.
"""

from __future__ import annotations

import numpy as np


def lse_merge(o_parts, lse_parts):
    """Merge n partials.

    o_parts: sequence of arrays [B, Nq, H, d]; lse_parts: sequence of [B, H, Nq].
    Returns (o [B, Nq, H, d], lse [B, H, Nq]) in float64.
    """
    if len(o_parts) != len(lse_parts) or len(o_parts) == 0:
        raise ValueError("need the same, non-zero number of O and LSE parts")
    o_parts = [np.asarray(o, dtype=np.float64) for o in o_parts]
    lse_parts = [np.asarray(l, dtype=np.float64) for l in lse_parts]
    lse_stack = np.stack(lse_parts)                         # [n, B, H, Nq]
    m = lse_stack.max(axis=0)                                # [B, H, Nq]
    finite = np.isfinite(m)
    m_safe = np.where(finite, m, 0.0)
    total = np.exp(lse_stack - m_safe[None]).sum(axis=0)     # exp(-inf) == 0
    lse = np.where(finite, m_safe + np.log(np.where(finite, total, 1.0)), -np.inf)
    o = np.zeros_like(o_parts[0])
    for o_i, lse_i in zip(o_parts, lse_parts):
        w = np.where(finite, np.exp(lse_i - np.where(finite, lse, 0.0)), 0.0)  # [B, H, Nq]
        o += np.transpose(w, (0, 2, 1))[..., None] * o_i
    return o, lse
