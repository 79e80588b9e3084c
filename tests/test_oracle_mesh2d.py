"""Pins of the oracle's Mesh2D tiling (Mosaic page, "Beyond 1D: Mesh2D
Attention"): for any grid, square or rectangular, the merged tiles must give
plain attention (the unsharded definition, itself pinned by brute force and
finite differences) forward and backward; a tile past the causal diagonal
holds no pair; a 1 x 1 grid is the unsharded call; and a brute-force loop
over one small grid checks the tile partials themselves."""

import math

import numpy as np
import pytest

from oracle import attention, mesh2d

RNG = np.random.default_rng(31)


def _rand(*shape):
    return RNG.standard_normal(shape)


@pytest.mark.parametrize("grid_q,grid_k", [(1, 1), (2, 2), (4, 4), (2, 4), (4, 2), (3, 1), (1, 6)])
@pytest.mark.parametrize("causal", [False, True])
def test_mesh2d_equals_plain_attention(grid_q, grid_k, causal):
    n, hq, hkv, d = 24, 4, 2, 8
    q, k, v, do = _rand(2, n, hq, d), _rand(2, n, hkv, d), _rand(2, n, hkv, d), _rand(2, n, hq, d)
    o_ref, l_ref = attention.attention_forward(q, k, v, causal=causal)
    g_ref = attention.attention_backward(q, k, v, do, causal=causal)
    o, l = mesh2d.mesh2d_forward(q, k, v, grid_q, grid_k, causal)
    np.testing.assert_allclose(o, o_ref, rtol=1e-12, atol=1e-13)
    np.testing.assert_allclose(l, l_ref, rtol=1e-12)
    g = mesh2d.mesh2d_backward(q, k, v, o, l, do, grid_q, grid_k, causal)
    for a, b in zip(g, g_ref):
        np.testing.assert_allclose(a, b, rtol=1e-10, atol=1e-12)


def test_tiles_past_the_diagonal_hold_no_pair():
    n, grid_q, grid_k = 24, 4, 3
    q, k, v = _rand(1, n, 2, 4), _rand(1, n, 2, 4), _rand(1, n, 2, 4)
    _, _, parts = mesh2d.mesh2d_forward(q, k, v, grid_q, grid_k, True, return_partials=True)
    seen = 0
    for i in range(grid_q):
        for j in range(grid_k):
            o_ij, l_ij = parts[i][j]
            has = mesh2d.tile_has_pairs(n, grid_q, grid_k, i, j, True)
            # chunk i = [6i, 6i + 6), chunk j = [8j, 8j + 8): pairs iff 8j <= 6i + 5
            assert has == (8 * j <= 6 * i + 5)
            if has:
                assert np.isfinite(l_ij).any()
                seen += 1
            else:
                assert np.all(np.isneginf(l_ij)) and np.all(o_ij == 0)
    assert seen == 9  # (0,0) (1,0) (1,1) (2,0) (2,1) (2,2) (3,0) (3,1) (3,2)


def test_tile_partials_by_brute_force():
    """Tile (1, 0) of a 2 x 2 causal grid: the second half of the queries
    against the first half of the keys, by scalar loops."""
    n, d = 8, 4
    q, k, v = _rand(1, n, 1, d), _rand(1, n, 1, d), _rand(1, n, 1, d)
    _, _, parts = mesh2d.mesh2d_forward(q, k, v, 2, 2, True, return_partials=True)
    o_t, l_t = parts[1][0]
    for t in range(4, 8):
        s = [sum(q[0, t, 0, c] * k[0, u, 0, c] for c in range(d)) / math.sqrt(d) for u in range(4)]
        z = sum(math.exp(x) for x in s)
        assert abs(l_t[0, 0, t - 4] - math.log(z)) < 1e-12
        for c in range(d):
            ref = sum(math.exp(s[u]) / z * v[0, u, 0, c] for u in range(4))
            assert abs(o_t[0, t - 4, 0, c] - ref) < 1e-12
    # tile (0, 1): every key after every query
    assert np.all(np.isneginf(parts[0][1][1]))


def test_one_by_one_grid_is_the_unsharded_call():
    q, k, v = _rand(1, 12, 2, 4), _rand(1, 12, 1, 4), _rand(1, 12, 1, 4)
    o, l = mesh2d.mesh2d_forward(q, k, v, 1, 1, True)
    o_ref, l_ref = attention.attention_forward(q, k, v, causal=True)
    assert np.array_equal(o, o_ref) and np.array_equal(l, l_ref)


def test_rejects_grids_that_do_not_divide_n():
    q = _rand(1, 10, 1, 4)
    with pytest.raises(ValueError):
        mesh2d.mesh2d_forward(q, q, q, 3, 1, False)
    with pytest.raises(ValueError):
        mesh2d.mesh2d_forward(q, q, q, 2, 0, False)
