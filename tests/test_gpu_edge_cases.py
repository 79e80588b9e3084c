"""Degenerate sizes on the GPU: empty batches, empty sequences, empty merge
rows and repacks of no tokens return at once with empty outputs (nothing
launched, no error), on every entry point that takes them.  Also the
smallest non-empty sequence, one token, checked against the oracle on every
attention path: a single visible key, so O is its value row and the LSE is
its scaled score."""

import numpy as np
import pytest
import torch

from oracle import attention as oatt
from sequence_attention_rm_b200 import synthetic
from tests._helpers import BF16_LSE_TOL, BF16_O_TOL, F32_TOL, assert_max_abs, gpu, np64

pytestmark = gpu


@pytest.fixture(scope="module")
def rm():
    from sequence_attention_rm_b200 import rm as mod
    return mod


def _zeros(B, N, H, d, dtype=torch.bfloat16):
    return torch.zeros(B, N, H, d, dtype=dtype, device="cuda")


@pytest.mark.parametrize("B,N", [(0, 1024), (1, 0), (0, 0)])
@pytest.mark.parametrize("layout,P", [("zigzag", 2), ("striped", 4), ("contiguous", 1)])
def test_ring_empty(rm, B, N, layout, P):
    q, k, v = _zeros(B, N, 4, 128), _zeros(B, N, 2, 128), _zeros(B, N, 2, 128)
    for order in ("rank", "global"):
        o, lse = rm.ring_attn_fwd(q, k, v, P=P, layout=layout, causal=True, order=order)
        assert o.shape == q.shape and lse.shape == (B, 4, N)
        dq, dk, dv = rm.ring_attn_bwd(q, k, v, o, lse, q, P=P, layout=layout, causal=True,
                                      order=order)
        assert dq.shape == q.shape and dk.shape == k.shape and dv.shape == v.shape
    torch.cuda.synchronize()
    assert rm.get_device_status() == rm.RM_OK


def test_block_and_short_sequence_empty(rm):
    q = _zeros(0, 5, 4, 24)
    o, lse = rm.attn_block_fwd(q, q, q, N=5, P=1, layout="contiguous", causal=False, q_rank=0,
                               kv_rank=0)
    assert o.shape == (0, 5, 4, 24) and lse.shape == (0, 4, 5)
    q = _zeros(3, 0, 4, 128)
    o, lse = rm.attn_block_fwd(q, q, q, N=0, P=2, layout="zigzag", causal=True, q_rank=0,
                               kv_rank=1)
    assert o.numel() == 0 and lse.numel() == 0
    torch.cuda.synchronize()


def test_merge_repack_permute_empty(rm):
    parts = [torch.zeros(1, 0, 2, 64, device="cuda") for _ in range(3)]
    lses = [torch.zeros(1, 2, 0, device="cuda") for _ in range(3)]
    o, lse = rm.lse_merge(parts, lses, torch.bfloat16)
    assert o.shape == (1, 0, 2, 64) and lse.shape == (1, 2, 0)
    x = _zeros(4, 0, 8, 128)
    y = rm.seq_head_repack(x, 4)
    assert y.shape == (4, 0, 2, 128)
    z = rm.layout_permute(_zeros(2, 0, 4, 32), "striped", 4)
    assert z.shape == (2, 0, 4, 32)
    torch.cuda.synchronize()


@pytest.mark.parametrize("dtype", [torch.bfloat16, torch.float32])
def test_one_token(rm, dtype):
    """N = 1: the only key is the token itself (visible under the causal rule
    too), so O = V and LSE = q.k / sqrt(d)."""
    w = synthetic.Workload(77, "one-token", B=3, Hq=4, Hkv=2, N=1, d=64, P=1, layout="contiguous",
                           causal=True, dtype=dtype, qkv_scale=0.5)
    q, k, v, _ = synthetic.attention_inputs(w, with_dout=False)
    o_ref, l_ref = oatt.attention_forward(np64(q), np64(k), np64(v), causal=True)
    # the closed form, independent of the oracle's softmax
    group = w.Hq // w.Hkv
    v_rep = np.repeat(np64(v), group, axis=2)
    assert np.allclose(o_ref, v_rep, atol=1e-12)
    qk = np.einsum("bthd,bthd->bht", np64(q), np.repeat(np64(k), group, axis=2)) / np.sqrt(w.d)
    assert np.allclose(l_ref, qk, atol=1e-12)
    to, tl = (F32_TOL, F32_TOL) if dtype == torch.float32 else (BF16_O_TOL, BF16_LSE_TOL)
    for mode in ("fused", "stepwise"):
        o, lse = rm.ring_attn_fwd(q.cuda(), k.cuda(), v.cuda(), P=1, layout="contiguous",
                                  causal=True, mode=mode)
        assert_max_abs(np64(o), o_ref, to, f"O {mode}")
        assert_max_abs(np64(lse), l_ref, tl, f"LSE {mode}")
