"""Pins of the oracle's layouts, LSE merge and ring: hand-written fixtures
from the pages, and the invariants the method fixes (merging the ring over
any P gives unsharded attention; permute + causal ring + un-permute gives plain
causal attention)."""

import math

import numpy as np
import pytest

from oracle import attention, layouts, merge, ring

RNG = np.random.default_rng(11)


def _rand(*shape, scale=1.0):
    return RNG.standard_normal(shape) * scale


def _read_layouts(golden_dir):
    rows = {}
    for line in open(f"{golden_dir}/layouts_n16.txt"):
        if line.startswith("#") or not line.strip():
            continue
        head, vals = line.split(":")
        name, p, r = head.split()
        rows[(name, int(p), int(r))] = [int(x) for x in vals.split()]
    return rows


def test_layout_positions_match_hand_fixture(golden_dir):
    rows = _read_layouts(golden_dir)
    assert len(rows) == 18
    for (name, p, r), expect in rows.items():
        assert list(layouts.rank_positions(name, 16, p, r)) == expect


@pytest.mark.parametrize("layout", layouts.LAYOUTS)
@pytest.mark.parametrize("n,p", [(24, 1), (24, 2), (24, 3), (24, 4), (48, 8), (40, 4)])
def test_layout_is_bijection_and_permute_roundtrip(layout, n, p):
    if layout == layouts.ZIGZAG and n % (2 * p):
        pytest.skip("zigzag needs 2P | N")
    pos = layouts.rank_major_positions(layout, n, p)
    assert sorted(pos.tolist()) == list(range(n))
    x = _rand(2, n, 3, 4)
    y = layouts.permute(x, layout, p)
    np.testing.assert_array_equal(y[:, 5], x[:, pos[5]])
    np.testing.assert_array_equal(layouts.unpermute(y, layout, p), x)


def test_striped_token_on_rank_t_mod_p():
    n, p = 64, 8
    pos = layouts.rank_major_positions(layouts.STRIPED, n, p)
    for idx, t in enumerate(pos):
        assert idx // (n // p) == t % p


def test_zigzag_balances_causal_work():
    # every rank sees the same number of causal (query, key) pairs: sum_t (t + 1)
    n, p = 64, 4
    work = [sum(t + 1 for t in layouts.rank_positions(layouts.ZIGZAG, n, p, r)) for r in range(p)]
    assert len(set(work)) == 1
    work_c = [sum(t + 1 for t in layouts.rank_positions(layouts.CONTIGUOUS, n, p, r)) for r in range(p)]
    assert len(set(work_c)) == p


def test_layout_validation():
    with pytest.raises(ValueError):
        layouts.check(layouts.ZIGZAG, 12, 4)
    with pytest.raises(ValueError):
        layouts.check(layouts.CONTIGUOUS, 10, 4)
    with pytest.raises(ValueError):
        layouts.check("diagonal", 8, 2)


def test_schedule_matches_walkthrough(golden_dir):
    table = {}
    for line in open(f"{golden_dir}/ring_schedule_p4.txt"):
        if line.startswith("#") or not line.strip():
            continue
        r, vals = line.split(":")
        table[int(r)] = [int(x) for x in vals.split()]
    assert ring.schedule(4) == [table[r] for r in range(4)]


def test_merge_closed_forms():
    o1, o2 = _rand(1, 5, 2, 3), _rand(1, 5, 2, 3)
    l1, l2 = _rand(1, 2, 5), _rand(1, 2, 5)
    o, l = merge.lse_merge([o1], [l1])
    np.testing.assert_allclose(o, o1, rtol=1e-15)
    np.testing.assert_allclose(l, l1, rtol=1e-15)
    # equal LSEs: plain average, LSE + ln 2
    o, l = merge.lse_merge([o1, o2], [l1, l1])
    np.testing.assert_allclose(o, (o1 + o2) / 2, rtol=1e-13)
    np.testing.assert_allclose(l, l1 + math.log(2), rtol=1e-13)
    # order does not matter
    oa, la = merge.lse_merge([o1, o2], [l1, l2])
    ob, lb = merge.lse_merge([o2, o1], [l2, l1])
    np.testing.assert_allclose(oa, ob, rtol=1e-13)
    np.testing.assert_allclose(la, lb, rtol=1e-13)


def test_merge_handles_empty_partials():
    o1, o2 = _rand(1, 4, 1, 3), _rand(1, 4, 1, 3)
    l1 = _rand(1, 1, 4)
    empty = np.full((1, 1, 4), -np.inf)
    o, l = merge.lse_merge([o1, np.zeros_like(o2)], [l1, empty])
    np.testing.assert_allclose(o, o1, rtol=1e-15)
    np.testing.assert_allclose(l, l1, rtol=1e-15)
    o, l = merge.lse_merge([np.zeros_like(o1), np.zeros_like(o2)], [empty, empty])
    assert np.all(o == 0) and np.all(l == -np.inf)


def test_merge_of_key_halves_is_attention_over_all_keys():
    q, k, v = _rand(1, 7, 2, 4), _rand(1, 10, 2, 4), _rand(1, 10, 2, 4)
    full = attention.attention_forward(q, k, v)
    a = attention.attention_forward(q, k[:, :3], v[:, :3])
    b = attention.attention_forward(q, k[:, 3:], v[:, 3:])
    o, l = merge.lse_merge([a[0], b[0]], [a[1], b[1]])
    np.testing.assert_allclose(o, full[0], rtol=1e-12)
    np.testing.assert_allclose(l, full[1], rtol=1e-13)


@pytest.mark.parametrize("p", [1, 2, 3, 4, 6, 8, 12, 24])
def test_ring_over_any_p_equals_unsharded(p):
    q, k, v = _rand(1, 24, 4, 8), _rand(1, 24, 2, 8), _rand(1, 24, 2, 8)
    ref = attention.attention_forward(q, k, v)
    o, l = ring.ring_forward(q, k, v, layouts.CONTIGUOUS, p, causal=False)
    np.testing.assert_allclose(o, ref[0], rtol=1e-12, atol=1e-13)
    np.testing.assert_allclose(l, ref[1], rtol=1e-13)


@pytest.mark.parametrize("layout", layouts.LAYOUTS)
@pytest.mark.parametrize("p", [1, 2, 4])
@pytest.mark.parametrize("causal", [False, True])
def test_permuted_ring_equals_plain(layout, p, causal):
    n = 32
    q, k, v = _rand(1, n, 4, 8), _rand(1, n, 2, 8), _rand(1, n, 2, 8)
    dout = _rand(1, n, 4, 8)
    o_ref, l_ref = attention.attention_forward(q, k, v, causal=causal)
    perm = lambda x: layouts.permute(x, layout, p)
    o, l = ring.ring_forward(perm(q), perm(k), perm(v), layout, p, causal)
    np.testing.assert_allclose(layouts.unpermute(o, layout, p), o_ref, rtol=1e-12, atol=1e-13)
    np.testing.assert_allclose(layouts.unpermute(l, layout, p, axis=2), l_ref, rtol=1e-12)
    g_ref = attention.attention_backward(q, k, v, dout, causal=causal)
    g = ring.ring_backward(perm(q), perm(k), perm(v), o, l, perm(dout), layout, p, causal)
    for a, b in zip(g, g_ref):
        np.testing.assert_allclose(layouts.unpermute(a, layout, p), b, rtol=1e-10, atol=1e-12)


def test_causal_contiguous_future_shards_are_empty():
    q, k, v = _rand(1, 16, 1, 4), _rand(1, 16, 1, 4), _rand(1, 16, 1, 4)
    _, _, parts = ring.ring_forward(q, k, v, layouts.CONTIGUOUS, 4, causal=True, return_partials=True)
    for r in range(4):
        for step in range(4):
            s = (r - step) % 4
            assert np.all(np.isneginf(parts[r][step][1])) == (s > r)
