"""Pins of the oracle's Ulysses repack and multi-axis routing."""

import math

import numpy as np
import pytest

from oracle import attention, multiaxis, repack

RNG = np.random.default_rng(5)


def test_repack_matches_hand_fixture(golden_dir):
    p, local, heads = 2, 2, 4
    x = np.zeros((p, local, heads, 1), dtype=np.int64)
    for s in range(p):
        for t in range(local):
            for h in range(heads):
                x[s, t, h, 0] = 1000 * s + 100 * t + h
    y = repack.seq_to_head(x, p)
    seen = 0
    for line in open(f"{golden_dir}/repack_p2.txt"):
        if line.startswith("#") or not line.strip():
            continue
        head, vals = line.split(":")
        _, r, row = head.split()
        assert y[int(r), int(row), :, 0].tolist() == [int(v) for v in vals.split()]
        seen += 1
    assert seen == 8


@pytest.mark.parametrize("p,local,heads", [(1, 3, 2), (2, 5, 4), (4, 3, 8), (8, 2, 16)])
def test_repack_roundtrip_and_full_sequence_view(p, local, heads):
    x = RNG.standard_normal((p, local, heads, 3))
    y = repack.seq_to_head(x, p)
    np.testing.assert_array_equal(repack.head_to_seq(y, p), x)
    # rank r holds the whole sequence (shards concatenated in rank order) for head group r
    full = x.reshape(p * local, heads, 3)
    hp = heads // p
    for r in range(p):
        np.testing.assert_array_equal(y[r], full[:, r * hp:(r + 1) * hp])


def test_repack_rejects_head_count_not_multiple_of_p():
    with pytest.raises(ValueError):
        repack.seq_to_head(np.zeros((4, 2, 6, 1)), 4)


def test_row_axis_is_attention_per_feature_and_head():
    b, r, f, e, heads = 1, 12, 3, 8, 2
    q, k, v = (RNG.standard_normal((b, r, f, e)) for _ in range(3))
    o, lse = multiaxis.row_axis_attention(q, k, v, heads)
    dh = e // heads
    for ff in range(f):
        for h in range(heads):
            sl = (slice(None), slice(None), ff, slice(h * dh, (h + 1) * dh))
            oo, ll = attention.attention_forward(q[sl][:, :, None], k[sl][:, :, None], v[sl][:, :, None])
            np.testing.assert_allclose(o[sl], oo[:, :, 0], rtol=1e-13)
            np.testing.assert_allclose(lse[:, ff * heads + h], ll[:, 0], rtol=1e-13)


def test_feature_axis_brute_force():
    b, r, f, e, heads = 1, 3, 5, 6, 2
    q, k, v = (RNG.standard_normal((b, r, f, e)) for _ in range(3))
    o, lse = multiaxis.feature_axis_attention(q, k, v, heads)
    dh = e // heads
    for row in range(r):
        for h in range(heads):
            cs = slice(h * dh, (h + 1) * dh)
            for t in range(f):
                s = [float(q[0, row, t, cs] @ k[0, row, u, cs]) / math.sqrt(dh) for u in range(f)]
                z = sum(math.exp(x) for x in s)
                expect = sum(math.exp(s[u]) / z * v[0, row, u, cs] for u in range(f))
                np.testing.assert_allclose(o[0, row, t, cs], expect, rtol=1e-12)
                assert abs(lse[row, h, t] - math.log(z)) < 1e-12


def test_zero_padding_head_dim_leaves_attention_unchanged():
    q, k, v = (RNG.standard_normal((1, 9, 2, 24)) for _ in range(3))
    pad = lambda x: np.concatenate([x, np.zeros((1, 9, 2, 8))], axis=-1)
    o, lse = attention.attention_forward(q, k, v)
    op, lsep = attention.attention_forward(pad(q), pad(k), pad(v), scale=1 / math.sqrt(24))
    np.testing.assert_allclose(op[..., :24], o, rtol=1e-13)
    assert np.all(op[..., 24:] == 0)
    np.testing.assert_allclose(lsep, lse, rtol=1e-13)
