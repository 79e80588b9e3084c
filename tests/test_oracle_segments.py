"""Pins of the oracle's packed and right-padded batches (ringmaster "Status":
dense causal sequences or globally right-padded batches; packing by global
position boundaries).  Each is checked against plain attention on the pieces,
computed without any segment mechanism: a packed sequence is the
concatenation of its segments' own attentions; a right-padded entry's valid
rows are the attention of the truncated sequence and its padded rows are
empty (O = 0, LSE = -inf, zero gradients); the ring with segments over any
layout equals the plain function with segments after un-permuting."""

import numpy as np
import pytest

from oracle import attention, layouts, ring

RNG = np.random.default_rng(31)


def _rand(*shape):
    return RNG.standard_normal(shape)


@pytest.mark.parametrize("causal", [True, False])
def test_packed_is_concatenation_of_segments(causal):
    cu = [0, 5, 6, 17, 30]
    n = 32  # positions 30, 31: trailing padding
    q, k, v, do = _rand(1, n, 4, 8), _rand(1, n, 2, 8), _rand(1, n, 2, 8), _rand(1, n, 4, 8)
    seg = attention.segments_from_boundaries(cu, n)
    assert list(seg[28:]) == [3, 3, -1, -1]
    o, l = attention.attention_forward(q, k, v, causal=causal, seg=seg)
    g = attention.attention_backward(q, k, v, do, causal=causal, seg=seg)
    for a, b in zip(cu[:-1], cu[1:]):
        o_s, l_s = attention.attention_forward(q[:, a:b], k[:, a:b], v[:, a:b], causal=causal)
        np.testing.assert_allclose(o[:, a:b], o_s, rtol=1e-12, atol=1e-14)
        np.testing.assert_allclose(l[:, :, a:b], l_s, rtol=1e-12)
        g_s = attention.attention_backward(q[:, a:b], k[:, a:b], v[:, a:b], do[:, a:b], causal=causal)
        for x, y in zip(g, g_s):
            np.testing.assert_allclose(x[:, a:b], y, rtol=1e-10, atol=1e-12)
    assert np.all(o[:, 30:] == 0) and np.all(np.isneginf(l[:, :, 30:]))
    for x in g:
        assert np.all(x[:, 30:] == 0)


@pytest.mark.parametrize("causal", [True, False])
def test_right_padding_is_truncation(causal):
    n, lengths = 24, [24, 17, 1]
    q, k, v, do = _rand(3, n, 2, 8), _rand(3, n, 2, 8), _rand(3, n, 2, 8), _rand(3, n, 2, 8)
    seg = attention.segments_from_lengths(lengths, n)
    o, l = attention.attention_forward(q, k, v, causal=causal, seg=seg)
    g = attention.attention_backward(q, k, v, do, causal=causal, seg=seg)
    for b, m in enumerate(lengths):
        o_t, l_t = attention.attention_forward(q[b:b + 1, :m], k[b:b + 1, :m], v[b:b + 1, :m],
                                               causal=causal)
        np.testing.assert_allclose(o[b:b + 1, :m], o_t, rtol=1e-12, atol=1e-14)
        np.testing.assert_allclose(l[b:b + 1, :, :m], l_t, rtol=1e-12)
        assert np.all(o[b, m:] == 0) and np.all(np.isneginf(l[b, :, m:]))
        g_t = attention.attention_backward(q[b:b + 1, :m], k[b:b + 1, :m], v[b:b + 1, :m],
                                           do[b:b + 1, :m], causal=causal)
        for x, y in zip(g, g_t):
            np.testing.assert_allclose(x[b:b + 1, :m], y, rtol=1e-10, atol=1e-12)
            assert np.all(x[b, m:] == 0)


@pytest.mark.parametrize("layout", layouts.LAYOUTS)
@pytest.mark.parametrize("p", [2, 4])
def test_ring_with_segments_equals_plain(layout, p):
    n = 32
    q, k, v, do = _rand(1, n, 2, 4), _rand(1, n, 1, 4), _rand(1, n, 1, 4), _rand(1, n, 2, 4)
    seg = attention.segments_from_boundaries([0, 3, 11, 12, 29], n)
    o_ref, l_ref = attention.attention_forward(q, k, v, causal=True, seg=seg)
    g_ref = attention.attention_backward(q, k, v, do, causal=True, seg=seg)
    perm = lambda x: layouts.permute(x, layout, p)
    o, l = ring.ring_forward(perm(q), perm(k), perm(v), layout, p, True, seg=seg)
    np.testing.assert_allclose(layouts.unpermute(o, layout, p), o_ref, rtol=1e-12, atol=1e-14)
    np.testing.assert_allclose(layouts.unpermute(l, layout, p, axis=2), l_ref, rtol=1e-12)
    g = ring.ring_backward(perm(q), perm(k), perm(v), o, l, perm(do), layout, p, True, seg=seg)
    for a, b in zip(g, g_ref):
        np.testing.assert_allclose(layouts.unpermute(a, layout, p), b, rtol=1e-10, atol=1e-12)


@pytest.mark.parametrize("kind", ["packed", "padded"])
@pytest.mark.parametrize("layout", layouts.LAYOUTS)
def test_usp_with_segments_equals_plain(kind, layout):
    """USP (Ulysses 2 x ring 2) with segment ids = the plain function with the
    same ids, after un-permuting: the head exchange keeps global positions."""
    from oracle import usp
    p, u, n = 2, 2, 32
    b_ = 1 if kind == "packed" else 2
    q, k, v, do = _rand(b_, n, 4, 4), _rand(b_, n, 2, 4), _rand(b_, n, 2, 4), _rand(b_, n, 4, 4)
    seg = (attention.segments_from_boundaries([0, 3, 11, 12, 29], n) if kind == "packed"
           else attention.segments_from_lengths([n, 13], n))
    o_ref, l_ref = attention.attention_forward(q, k, v, causal=True, seg=seg)
    g_ref = attention.attention_backward(q, k, v, do, causal=True, seg=seg)
    perm = lambda x: layouts.permute(x, layout, p)
    o, l = usp.usp_forward(perm(q), perm(k), perm(v), layout, p, u, True, seg=seg)
    np.testing.assert_allclose(layouts.unpermute(o, layout, p), o_ref, rtol=1e-12, atol=1e-14)
    np.testing.assert_allclose(layouts.unpermute(l, layout, p, axis=2), l_ref, rtol=1e-12)
    g = usp.usp_backward(perm(q), perm(k), perm(v), o, l, perm(do), layout, p, u, True, seg=seg)
    for a, b in zip(g, g_ref):
        np.testing.assert_allclose(layouts.unpermute(a, layout, p), b, rtol=1e-10, atol=1e-12)


@pytest.mark.parametrize("kind", ["packed", "padded"])
@pytest.mark.parametrize("grid", [(2, 2), (4, 2), (2, 4), (3, 1)])
@pytest.mark.parametrize("causal", [True, False])
def test_mesh2d_with_segments_equals_plain(kind, grid, causal):
    """Mesh2D tiles with segment ids, merged per query chunk = the plain
    function with the same ids; rows that see no key at all (padding) end
    with O = 0 and LSE = -inf and get zero gradients."""
    from oracle import mesh2d
    gq, gk = grid
    n = 24
    b_ = 1 if kind == "packed" else 2
    q, k, v, do = _rand(b_, n, 4, 4), _rand(b_, n, 2, 4), _rand(b_, n, 2, 4), _rand(b_, n, 4, 4)
    seg = (attention.segments_from_boundaries([0, 5, 6, 17, 21], n) if kind == "packed"
           else attention.segments_from_lengths([19, 7], n))
    o_ref, l_ref = attention.attention_forward(q, k, v, causal=causal, seg=seg)
    g_ref = attention.attention_backward(q, k, v, do, causal=causal, seg=seg)
    o, l = mesh2d.mesh2d_forward(q, k, v, gq, gk, causal, seg=seg)
    np.testing.assert_allclose(o, o_ref, rtol=1e-12, atol=1e-14)
    np.testing.assert_allclose(l, l_ref, rtol=1e-12)
    g = mesh2d.mesh2d_backward(q, k, v, o, l, do, gq, gk, causal, seg=seg)
    for a, b in zip(g, g_ref):
        np.testing.assert_allclose(a, b, rtol=1e-10, atol=1e-12)
    pad = np.asarray(seg).reshape(b_, n) < 0
    assert np.all(np.isneginf(np.moveaxis(l, 1, 2)[pad]))
    assert np.all(o[pad] == 0) and np.all(g[0][pad] == 0)
