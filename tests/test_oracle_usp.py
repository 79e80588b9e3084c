"""Pins of the oracle's USP composition (ringmaster "Why": Ulysses x ring on
a 2-D mesh): whatever the (ring, Ulysses) split, the composition must give
plain attention (the unsharded definition) forward and backward; with one
Ulysses rank it is the ring itself; the selector follows its stated rule,
checked by brute force."""

import numpy as np
import pytest

from oracle import attention, layouts, ring, usp

RNG = np.random.default_rng(23)


def _rand(*shape):
    return RNG.standard_normal(shape)


@pytest.mark.parametrize("layout", layouts.LAYOUTS)
@pytest.mark.parametrize("p_ring,p_ulysses", [(1, 2), (2, 2), (4, 1), (2, 4), (1, 4)])
@pytest.mark.parametrize("causal", [False, True])
def test_usp_equals_plain_attention(layout, p_ring, p_ulysses, causal):
    n, hq, hkv, d = 32, 8, 4, 8
    if p_ulysses > hkv:
        pytest.skip("Ulysses degree above the KV heads")
    q, k, v, do = _rand(2, n, hq, d), _rand(2, n, hkv, d), _rand(2, n, hkv, d), _rand(2, n, hq, d)
    o_ref, l_ref = attention.attention_forward(q, k, v, causal=causal)
    g_ref = attention.attention_backward(q, k, v, do, causal=causal)
    perm = lambda x: layouts.permute(x, layout, p_ring)
    o, l = usp.usp_forward(perm(q), perm(k), perm(v), layout, p_ring, p_ulysses, causal)
    np.testing.assert_allclose(layouts.unpermute(o, layout, p_ring), o_ref, rtol=1e-12, atol=1e-13)
    np.testing.assert_allclose(layouts.unpermute(l, layout, p_ring, axis=2), l_ref, rtol=1e-12)
    g = usp.usp_backward(perm(q), perm(k), perm(v), o, l, perm(do), layout, p_ring, p_ulysses,
                         causal)
    for a, b in zip(g, g_ref):
        np.testing.assert_allclose(layouts.unpermute(a, layout, p_ring), b, rtol=1e-10, atol=1e-12)


def test_usp_with_one_ulysses_rank_is_the_ring():
    q, k, v = _rand(1, 24, 4, 8), _rand(1, 24, 2, 8), _rand(1, 24, 2, 8)
    o, l = usp.usp_forward(q, k, v, layouts.ZIGZAG, 3, 1, True)
    o2, l2 = ring.ring_forward(q, k, v, layouts.ZIGZAG, 3, True)
    assert np.array_equal(o, o2) and np.array_equal(l, l2)


def test_usp_head_groups_are_independent():
    """Changing the inputs of one head group leaves the other groups' outputs
    unchanged (the Ulysses exchange moves whole heads, no mixing)."""
    n, hq, hkv, d = 16, 4, 2, 4
    q, k, v = _rand(1, n, hq, d), _rand(1, n, hkv, d), _rand(1, n, hkv, d)
    o1, _ = usp.usp_forward(q, k, v, layouts.CONTIGUOUS, 2, 2, True)
    k2 = k.copy()
    k2[:, :, 1] *= 2.0  # KV head 1 belongs to head group 1 (query heads 2, 3)
    o2, _ = usp.usp_forward(q, k2, v, layouts.CONTIGUOUS, 2, 2, True)
    assert np.array_equal(o1[:, :, :2], o2[:, :, :2])
    assert not np.allclose(o1[:, :, 2:], o2[:, :, 2:])


def test_auto_select_rule_by_brute_force():
    for hkv in (1, 2, 3, 4, 8, 16):
        for group in (1, 2, 4):
            for world in (1, 2, 4, 6, 8, 12, 16, 32):
                u, r = usp.auto_select(hkv * group, hkv, world)
                assert u * r == world
                ok = [x for x in range(1, world + 1) if world % x == 0 and hkv % x == 0 and x <= 8]
                assert u == max(ok)
    assert usp.auto_select(16, 8, 8) == (8, 1)
    assert usp.auto_select(32, 4, 16) == (4, 4)
    assert usp.auto_select(64, 16, 32, node_size=8) == (8, 4)


def test_usp_rejects_bad_splits():
    q = _rand(1, 12, 4, 4)
    with pytest.raises(ValueError):
        usp.usp_forward(q, q[:, :, :2], q[:, :, :2], layouts.CONTIGUOUS, 2, 4, False)  # 4 > Hkv
    with pytest.raises(ValueError):
        usp.usp_forward(q, q, q, layouts.CONTIGUOUS, 5, 1, False)  # 12 % 5
