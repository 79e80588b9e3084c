"""Pins of the oracle's exact attention (forward and backward) to things other
than itself: a brute-force loop written from the definition, closed forms,
invariants, fp64 finite differences and a library cross-check."""

import math

import numpy as np
import pytest
import torch

from oracle import attention

RNG = np.random.default_rng(7)


def _rand(*shape, scale=1.0):
    return RNG.standard_normal(shape) * scale


def brute_force(q, k, v, causal, q_pos, k_pos):
    """softmax(QK^T/sqrt(d))V by scalar loops and math.exp (Mosaic page, "The Problem")."""
    B, nq, hq, d = q.shape
    hkv = k.shape[2]
    o = np.zeros((B, nq, hq, v.shape[3]))
    lse = np.full((B, hq, nq), -math.inf)
    for b in range(B):
        for h in range(hq):
            g = h // (hq // hkv)
            for t in range(nq):
                keys = [u for u in range(k.shape[1]) if (not causal) or k_pos[u] <= q_pos[t]]
                if not keys:
                    continue
                s = {u: sum(q[b, t, h, c] * k[b, u, g, c] for c in range(d)) / math.sqrt(d) for u in keys}
                z = sum(math.exp(s[u]) for u in keys)
                lse[b, h, t] = math.log(z)
                for c in range(v.shape[3]):
                    o[b, t, h, c] = sum(math.exp(s[u]) / z * v[b, u, g, c] for u in keys)
    return o, lse


@pytest.mark.parametrize("causal", [False, True])
def test_forward_matches_brute_force(causal):
    q, k, v = _rand(2, 5, 4, 3), _rand(2, 6, 2, 3), _rand(2, 6, 2, 2)
    q_pos = np.array([3, 0, 7, 5, 1])
    k_pos = np.array([0, 2, 4, 6, 1, 5])
    o, lse = attention.attention_forward(q, k, v, causal=causal, q_pos=q_pos, k_pos=k_pos)
    o_bf, lse_bf = brute_force(q, k, v, causal, q_pos, k_pos)
    np.testing.assert_allclose(o, o_bf, rtol=1e-12, atol=1e-12)
    np.testing.assert_allclose(lse, lse_bf, rtol=1e-12, atol=1e-12)


def test_forward_hand_example():
    # d = 2, one query, two keys: s = (q.k0, q.k1)/sqrt(2) = (1/sqrt 2, 0)
    q = np.array([1.0, 0.0]).reshape(1, 1, 1, 2)
    k = np.array([[1.0, 0.0], [0.0, 1.0]]).reshape(1, 2, 1, 2)
    v = np.array([[1.0, 2.0], [3.0, 4.0]]).reshape(1, 2, 1, 2)
    o, lse = attention.attention_forward(q, k, v)
    a = math.exp(1 / math.sqrt(2))
    w0, w1 = a / (a + 1), 1 / (a + 1)
    np.testing.assert_allclose(o.ravel(), [w0 * 1 + w1 * 3, w0 * 2 + w1 * 4], rtol=1e-14)
    np.testing.assert_allclose(lse.ravel(), [math.log(a + 1)], rtol=1e-14)


def test_zero_query_gives_mean_and_log_count():
    n = 9
    q = np.zeros((1, n, 2, 4))
    k, v = _rand(1, n, 1, 4), _rand(1, n, 1, 4)
    o, lse = attention.attention_forward(q, k, v, causal=True)
    for t in range(n):
        np.testing.assert_allclose(o[0, t, 0], v[0, :t + 1, 0].mean(axis=0), rtol=1e-12, atol=1e-14)
        np.testing.assert_allclose(lse[0, :, t], math.log(t + 1), rtol=1e-13)
    o, lse = attention.attention_forward(q, k, v, causal=False)
    np.testing.assert_allclose(o[0, :, 1], np.broadcast_to(v[0, :, 0].mean(axis=0), (n, 4)), rtol=1e-12)
    np.testing.assert_allclose(lse, math.log(n), rtol=1e-13)


def test_single_visible_key():
    q, k, v = _rand(1, 4, 1, 8), _rand(1, 4, 1, 8), _rand(1, 4, 1, 8)
    o, lse = attention.attention_forward(q, k, v, causal=True)
    np.testing.assert_allclose(o[0, 0, 0], v[0, 0, 0], rtol=1e-14)
    np.testing.assert_allclose(lse[0, 0, 0], q[0, 0, 0] @ k[0, 0, 0] / math.sqrt(8), rtol=1e-13)


def test_ones_value_gives_ones():
    q, k = _rand(1, 17, 2, 8, scale=3.0), _rand(1, 17, 2, 8, scale=3.0)
    o, _ = attention.attention_forward(q, k, np.ones((1, 17, 2, 8)), causal=True)
    np.testing.assert_allclose(o, 1.0, rtol=1e-13)


def test_rows_sum_to_one():
    q, k = _rand(2, 11, 4, 8, scale=2.0), _rand(2, 11, 2, 8, scale=2.0)
    for causal in (False, True):
        p = attention.attention_probabilities(q, k, causal=causal)
        np.testing.assert_allclose(p.sum(axis=-1), 1.0, rtol=1e-13)
        assert (p >= 0).all()
        if causal:
            assert np.all(np.triu(p, k=1) == 0.0)


def test_no_visible_key_row():
    q, k, v = _rand(1, 2, 1, 4), _rand(1, 3, 1, 4), _rand(1, 3, 1, 4)
    o, lse = attention.attention_forward(q, k, v, causal=True, q_pos=np.array([0, 5]),
                                         k_pos=np.array([3, 4, 5]))
    assert np.all(o[0, 0] == 0) and lse[0, 0, 0] == -np.inf
    assert np.isfinite(lse[0, 0, 1])


def test_explicit_scale_is_used():
    q, k, v = _rand(1, 6, 1, 4), _rand(1, 6, 1, 4), _rand(1, 6, 1, 4)
    # doubling q at scale 1/2 is the same score matrix as q at scale 1
    o1, l1 = attention.attention_forward(2 * q, k, v, scale=0.5)
    o2, l2 = attention.attention_forward(q, k, v, scale=1.0)
    np.testing.assert_allclose(o1, o2, rtol=1e-13)
    np.testing.assert_allclose(l1, l2, rtol=1e-13)


@pytest.mark.parametrize("causal", [False, True])
def test_forward_matches_torch_sdpa_fp64(causal):
    q, k, v = _rand(2, 33, 4, 16), _rand(2, 33, 2, 16), _rand(2, 33, 2, 16)
    o, lse = attention.attention_forward(q, k, v, causal=causal)
    tq = torch.from_numpy(q).permute(0, 2, 1, 3)
    tk = torch.from_numpy(k).permute(0, 2, 1, 3).repeat_interleave(2, dim=1)
    tv = torch.from_numpy(v).permute(0, 2, 1, 3).repeat_interleave(2, dim=1)
    ref = torch.nn.functional.scaled_dot_product_attention(tq, tk, tv, is_causal=causal)
    np.testing.assert_allclose(o, ref.permute(0, 2, 1, 3).numpy(), rtol=1e-11, atol=1e-12)
    s = (tq @ tk.transpose(-1, -2)) / math.sqrt(16)
    if causal:
        s = s.masked_fill(torch.ones(33, 33, dtype=torch.bool).triu(1), -math.inf)
    np.testing.assert_allclose(lse, torch.logsumexp(s, dim=-1).numpy(), rtol=1e-12)


def _loss(q, k, v, dout, causal):
    o, _ = attention.attention_forward(q, k, v, causal=causal)
    return float((o * dout).sum())


@pytest.mark.parametrize("causal", [False, True])
def test_backward_matches_finite_differences(causal):
    q, k, v = _rand(1, 6, 2, 3), _rand(1, 6, 1, 3), _rand(1, 6, 1, 3)
    dout = _rand(1, 6, 2, 3)
    dq, dk, dv = attention.attention_backward(q, k, v, dout, causal=causal)
    eps = 1e-6
    for x, g in ((q, dq), (k, dk), (v, dv)):
        num = np.zeros_like(x)
        for idx in np.ndindex(x.shape):
            old = x[idx]
            x[idx] = old + eps
            lp = _loss(q, k, v, dout, causal)
            x[idx] = old - eps
            lm = _loss(q, k, v, dout, causal)
            x[idx] = old
            num[idx] = (lp - lm) / (2 * eps)
        np.testing.assert_allclose(g, num, rtol=1e-6, atol=1e-8)


@pytest.mark.parametrize("causal", [False, True])
def test_backward_invariants(causal):
    q, k, v = _rand(2, 20, 4, 8), _rand(2, 20, 2, 8), _rand(2, 20, 2, 8)
    dout = _rand(2, 20, 4, 8)
    dq, dk, dv = attention.attention_backward(q, k, v, dout, causal=causal)
    # sum_u dK_u = 0 (each softmax row's derivative sums to zero)
    np.testing.assert_allclose(dk.sum(axis=1), 0.0, atol=1e-11)
    # sum_u dV_u = sum over the group's query heads and all t of dO_t
    grouped = dout.reshape(2, 20, 2, 2, 8).sum(axis=3)
    np.testing.assert_allclose(dv.sum(axis=1), grouped.sum(axis=1), rtol=1e-11, atol=1e-11)


def test_delta_two_routes_agree_and_block_equals_full():
    q, k, v = _rand(1, 12, 2, 4), _rand(1, 12, 1, 4), _rand(1, 12, 1, 4)
    dout = _rand(1, 12, 2, 4)
    o, lse = attention.attention_forward(q, k, v, causal=True)
    p = attention.attention_probabilities(q, k, causal=True)
    dp = np.einsum("bthc,buhc->bhtu", dout, np.repeat(v, 2, axis=2))
    np.testing.assert_allclose(attention.delta_from_output(dout, o), (p * dp).sum(-1), rtol=1e-12)
    full = attention.attention_backward(q, k, v, dout, causal=True)
    blk = attention.attention_backward_block(q, k, v, dout, lse, attention.delta_from_output(dout, o),
                                             causal=True)
    for a, b in zip(full, blk):
        np.testing.assert_allclose(a, b, rtol=1e-11, atol=1e-12)


def test_gqa_equals_mha_with_repeated_kv():
    q, k, v = _rand(1, 10, 6, 4), _rand(1, 10, 2, 4), _rand(1, 10, 2, 4)
    o, lse = attention.attention_forward(q, k, v, causal=True)
    o2, lse2 = attention.attention_forward(q, np.repeat(k, 3, axis=2), np.repeat(v, 3, axis=2), causal=True)
    np.testing.assert_allclose(o, o2, rtol=1e-14)
    np.testing.assert_allclose(lse, lse2, rtol=1e-14)
    with pytest.raises(ValueError):
        attention.kv_head_of(0, 5, 2)


def test_row_blocking_does_not_change_results(monkeypatch):
    q, k, v = _rand(1, 40, 2, 4), _rand(1, 40, 2, 4), _rand(1, 40, 2, 4)
    ref = attention.attention_forward(q, k, v, causal=True)
    monkeypatch.setattr(attention, "_ELEMS_PER_BLOCK", 7 * 40)
    got = attention.attention_forward(q, k, v, causal=True)
    np.testing.assert_array_equal(ref[0], got[0])
    np.testing.assert_array_equal(ref[1], got[1])
