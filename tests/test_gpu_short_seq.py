"""GPU parity of short-sequence attention (at most 16 tokens per shard)
against the fp64 oracle: the local feature-axis attention of the Mosaic page
("The Implementation": attention along a short axis of a multi-axis tensor),
and every ring shard pair whose shards are that short.

bf16 operands with a bf16 output run on the staged kernel (a block copies
whole sequences into shared memory first); fp32 operands and fp32 partial
outputs run on the one-thread-per-row kernel.  Both are checked here, including batches that
leave the last block of sequences partly empty, GQA, the causal rule across
shard pairs of every layout, the longest supported sequence and strided
views."""

import numpy as np
import pytest
import torch

from oracle import attention as oatt
from oracle import layouts as olay
from sequence_attention_rm_b200 import synthetic
from tests._helpers import BF16_LSE_TOL, BF16_O_TOL, F32_TOL, assert_max_abs, gpu, np64

pytestmark = gpu


@pytest.fixture(scope="module")
def rm():
    from sequence_attention_rm_b200 import rm as mod
    return mod


def _inputs(dtype, B, Hq, Hkv, N, d, seed):
    w = synthetic.Workload(seed, "short", B=B, Hq=Hq, Hkv=Hkv, N=N, d=d, P=1, layout="contiguous",
                           causal=True, dtype=dtype, qkv_scale=1.0)
    q, k, v, _ = synthetic.attention_inputs(w, with_dout=False)
    return q, k, v


def _tols(dtype):
    return (F32_TOL, F32_TOL) if dtype == torch.float32 else (BF16_O_TOL, BF16_LSE_TOL)


# dtype, B, Hq, Hkv, N, d, causal
UNSHARDED = [
    (torch.bfloat16, 1, 4, 4, 5, 24, False),      # one sequence, the tabular head size
    (torch.bfloat16, 1001, 4, 4, 5, 24, False),   # last block of sequences partly empty
    (torch.bfloat16, 333, 8, 2, 7, 32, True),     # GQA, causal
    (torch.bfloat16, 65, 2, 1, 16, 64, True),     # the longest sequence, d = 64
    (torch.bfloat16, 70, 3, 3, 1, 24, False),     # one token
    (torch.bfloat16, 40, 4, 2, 9, 64, True),
    (torch.float32, 90, 4, 2, 6, 24, True),       # fp32: unstaged kernel
]


@pytest.mark.parametrize("case", UNSHARDED,
                         ids=lambda c: f"{str(c[0])[6:]}-B{c[1]}H{c[2]}/{c[3]}-N{c[4]}-d{c[5]}-{'c' if c[6] else 'nc'}")
def test_short_sequences_unsharded(rm, case):
    dtype, B, Hq, Hkv, N, d, causal = case
    q, k, v = _inputs(dtype, B, Hq, Hkv, N, d, 300 + B + N + d)
    o_ref, l_ref = oatt.attention_forward(np64(q), np64(k), np64(v), causal=causal)
    to, tl = _tols(dtype)
    o, l = rm.ring_attn_fwd(q.cuda(), k.cuda(), v.cuda(), P=1, layout="contiguous", causal=causal)
    assert o.dtype == dtype
    assert_max_abs(np64(o), o_ref, to, "O")
    assert_max_abs(np64(l), l_ref, tl, "LSE")
    # the block entry point, bf16 output and fp32 output
    for o_f32 in (False, True):
        o, l = rm.attn_block_fwd(q.cuda(), k.cuda(), v.cuda(), N=N, P=1, layout="contiguous",
                                 causal=causal, q_rank=0, kv_rank=0, o_f32=o_f32)
        assert_max_abs(np64(o), o_ref, to, f"block O (o_f32={o_f32})")
        assert_max_abs(np64(l), l_ref, tl, f"block LSE (o_f32={o_f32})")


@pytest.mark.parametrize("layout,P,N", [("contiguous", 2, 24), ("zigzag", 2, 32),
                                        ("striped", 4, 48)])
def test_short_shards_every_pair(rm, layout, P, N):
    """Every (query shard, KV shard) pair of a causal ring with shards of at
    most 16 tokens, bf16 output (staged kernel), against the oracle with the
    shards' global positions."""
    dtype, B, Hq, Hkv, d = torch.bfloat16, 37, 4, 2, 32
    q, k, v = _inputs(dtype, B, Hq, Hkv, N, d, 400 + N)
    L = N // P
    perm = lambda x: np64(x) if layout == "contiguous" else olay.permute(np64(x), layout, P)
    qr, kr, vr = perm(q), perm(k), perm(v)
    dev = lambda x: torch.from_numpy(x.astype(np.float32)).to(dtype).cuda()
    qg, kg, vg = dev(qr), dev(kr), dev(vr)
    for r in range(P):
        for s in range(P):
            o, l = rm.attn_block_fwd(qg[:, r * L:(r + 1) * L], kg[:, s * L:(s + 1) * L],
                                     vg[:, s * L:(s + 1) * L], N=N, P=P, layout=layout,
                                     causal=True, q_rank=r, kv_rank=s)
            o_ref, l_ref = oatt.attention_forward(
                qr[:, r * L:(r + 1) * L], kr[:, s * L:(s + 1) * L], vr[:, s * L:(s + 1) * L],
                causal=True, q_pos=olay.rank_positions(layout, N, P, r),
                k_pos=olay.rank_positions(layout, N, P, s))
            assert_max_abs(np64(o), o_ref, BF16_O_TOL, f"O pair ({r},{s})")
            assert_max_abs(np64(l), l_ref, BF16_LSE_TOL, f"LSE pair ({r},{s})")


def test_short_sequences_strided_views(rm):
    """Head views of a wider tensor (the feature-axis routing of a tabular
    tensor): rows of 3 heads x 32 inside a 160-wide embedding, no copy."""
    B, F, E, H, d = 257, 6, 160, 3, 32
    g = torch.Generator().manual_seed(77)
    base = [torch.randn(B, F, E, generator=g).to(torch.bfloat16) for _ in range(3)]
    views = [x[:, :, 32:32 + H * d].reshape(B, F, H, d) for x in base]   # host copies for the oracle
    o_ref, l_ref = oatt.attention_forward(*(np64(x) for x in views), causal=False)
    dev = [x.cuda()[:, :, 32:32 + H * d].unflatten(2, (H, d)) for x in base]  # strided device views
    assert not dev[0].is_contiguous()
    o, l = rm.attn_block_fwd(*dev, N=F, P=1, layout="contiguous", causal=False, q_rank=0,
                             kv_rank=0)
    assert_max_abs(np64(o), o_ref, BF16_O_TOL, "O")
    assert_max_abs(np64(l), l_ref, BF16_LSE_TOL, "LSE")
