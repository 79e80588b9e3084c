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


# (Hq, Hkv, world, node_size) -> (ulysses, ring), worked out by hand from the
# reading of ringmaster "Why" (an auto-selector driven by the KV-head count and
# the world size; the Ulysses degree is capped by the KV heads): the Ulysses
# degree is the largest u that divides both the world and the KV-head count
# and fits in one node; the ring takes the rest of the world.
SELECTOR_TABLE = [
    ((16, 8, 8, 8), (8, 1)),      # the whole world fits the 8 KV heads
    ((16, 8, 16, 8), (8, 2)),
    ((32, 4, 16, 8), (4, 4)),     # capped by 4 KV heads
    ((64, 16, 32, 8), (8, 4)),    # capped by the node size
    ((64, 16, 32, 16), (16, 2)),
    ((8, 1, 8, 8), (1, 8)),       # one KV head: ring only
    ((16, 8, 1, 8), (1, 1)),      # one device
    ((12, 3, 6, 8), (3, 2)),      # non-power-of-two world and head count
    ((12, 3, 4, 8), (1, 4)),      # 3 and 4 share no factor
    ((24, 6, 12, 8), (6, 2)),
    ((24, 6, 12, 4), (3, 4)),     # 6 divides both but exceeds the node
    ((16, 8, 6, 8), (2, 3)),
    ((10, 5, 10, 8), (5, 2)),
    ((14, 7, 7, 8), (7, 1)),
    ((2, 2, 3, 8), (1, 3)),
    ((48, 12, 24, 8), (6, 4)),
]


@pytest.mark.parametrize("args,want", SELECTOR_TABLE, ids=lambda x: str(x))
def test_auto_select_hand_table(args, want):
    hq, hkv, world, node = args
    assert usp.auto_select(hq, hkv, world, node_size=node) == want


def test_auto_select_split_covers_the_world():
    for hkv in (1, 2, 3, 4, 8, 16):
        for world in (1, 2, 4, 6, 8, 12, 16, 32):
            u, r = usp.auto_select(hkv * 2, hkv, world)
            assert u * r == world and hkv % u == 0 and u <= 8


def test_usp_rejects_bad_splits():
    q = _rand(1, 12, 4, 4)
    with pytest.raises(ValueError):
        usp.usp_forward(q, q[:, :, :2], q[:, :, :2], layouts.CONTIGUOUS, 2, 4, False)  # 4 > Hkv
    with pytest.raises(ValueError):
        usp.usp_forward(q, q, q, layouts.CONTIGUOUS, 5, 1, False)  # 12 % 5
