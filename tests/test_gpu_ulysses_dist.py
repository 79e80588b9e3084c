"""Ulysses attention over real ranks (``ulysses_dist``) with its pack /
unpack and attention on the CUDA kernels, on one GPU: the ranks are threads
of this process and all_to_all_single goes through the in-process stand-in
of ``tests/_thread_ranks.py`` (host hand-offs of stream-ordered copies).
What this checks is the kernel side: the local pack that lays a shard out
for the all-to-all, the attention over the rank-major sequence of a head
group, the unpack; the exchange itself is checked over real gloo ranks on
the CPU.  Results are compared with the unsharded fp64 oracle."""

import numpy as np
import pytest
import torch

from oracle import attention as oatt
from oracle import layouts as olay
from sequence_attention_rm_b200 import synthetic, ulysses_dist
from tests._helpers import (BF16_O_TOL, F32_TOL, assert_grad_close, assert_max_abs, gpu, np64)
from tests._thread_ranks import run_ranks

pytestmark = gpu

CASES = [
    # dtype, B, Hq, Hkv, N, d, P, layout, causal, segments
    (torch.bfloat16, 1, 4, 2, 2048, 128, 2, "zigzag", True, None),
    (torch.bfloat16, 1, 8, 4, 2048, 128, 4, "striped", True, None),
    (torch.bfloat16, 2, 4, 4, 1024, 64, 4, "contiguous", True, None),
    (torch.float32, 1, 2, 2, 512, 64, 2, "contiguous", False, None),
    (torch.bfloat16, 1, 4, 2, 2048, 128, 2, "zigzag", True, ("packed", [0, 1, 700, 1300, 2040, 2048])),
]


@pytest.mark.parametrize("dtype,B,Hq,Hkv,N,d,P,layout,causal,segments", CASES)
def test_ulysses_dist_on_the_kernels(dtype, B, Hq, Hkv, N, d, P, layout, causal, segments):
    seed = 8100 + N + P
    q = synthetic.tensor(seed, (B, N, Hq, d), dtype)
    k = synthetic.tensor(seed + 1, (B, N, Hkv, d), dtype)
    v = synthetic.tensor(seed + 2, (B, N, Hkv, d), dtype)
    do = synthetic.tensor(seed + 3, (B, N, Hq, d), dtype)
    pos = [olay.rank_positions(layout, N, P, r) for r in range(P)]
    segs, seg = {}, None
    if segments is not None:
        vals = segments[1]
        segs = {"cu_seqlens": torch.tensor(vals, dtype=torch.int32, device="cuda")}
        seg = oatt.segments_from_boundaries(np.array(vals), N)
    shard = lambda x, r: x[:, torch.from_numpy(pos[r])].contiguous().cuda()

    def rank(r):
        qr, kr, vr, dor = shard(q, r), shard(k, r), shard(v, r), shard(do, r)
        o, ctx = ulysses_dist.ulysses_forward(qr, kr, vr, layout=layout, causal=causal, **segs)
        return o, ulysses_dist.ulysses_backward(dor, ctx)

    out = run_ranks(ulysses_dist, P, rank)
    o_ref, _ = oatt.attention_forward(np64(q), np64(k), np64(v), causal=causal, seg=seg)
    g_ref = oatt.attention_backward(np64(q), np64(k), np64(v), np64(do), causal=causal, seg=seg)
    o_tol = F32_TOL if dtype == torch.float32 else BF16_O_TOL
    kw = {"tol": F32_TOL} if dtype == torch.float32 else {}
    for r, (o, grads) in enumerate(out):
        assert o.dtype == dtype and all(g.dtype == dtype for g in grads)
        assert_max_abs(np64(o), o_ref[:, pos[r]], o_tol, f"O rank {r}")
        for name, g, ref in zip(("dQ", "dK", "dV"), grads, g_ref):
            assert_grad_close(np64(g), ref[:, pos[r]], what=f"{name} rank {r}", **kw)


@pytest.mark.parametrize("P,L,H", [(2, 6, 4), (4, 8, 8), (8, 16, 16)])
def test_seq_to_head_round_trip_is_the_identity(P, L, H):
    """seq -> head then head -> seq over P thread ranks returns every rank's
    shard bit for bit, and rank r's head-sharded tensor holds head group r of
    every rank's tokens in rank order."""
    shards = [synthetic.tensor(8200 + r, (1, L, H, 128), torch.bfloat16).cuda() for r in range(P)]

    def rank(r):
        y = ulysses_dist.seq_to_head(shards[r])
        return y, ulysses_dist.head_to_seq(y)

    out = run_ranks(ulysses_dist, P, rank)
    hp = H // P
    for r, (y, back) in enumerate(out):
        assert torch.equal(back, shards[r])
        want = torch.cat([s[:, :, r * hp:(r + 1) * hp] for s in shards], dim=1)
        assert torch.equal(y, want)


def test_real_nccl_group_of_one():
    """ring_dist and ulysses_dist on a real NCCL process group of one rank
    (this GPU): the all-to-all runs through NCCL itself and the results
    equal the single-GPU ring's bit for bit (one rank: the same kernels on
    the same operands)."""
    import os
    import socket

    import torch.distributed as dist

    from sequence_attention_rm_b200 import ring_dist, rm
    with socket.socket(socket.AF_INET, socket.SOCK_STREAM) as s:
        s.bind(("127.0.0.1", 0))
        port = s.getsockname()[1]
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("nccl", rank=0, world_size=1, device_id=torch.device("cuda", 0))
    try:
        q, k, v, do = (synthetic.tensor(8300 + i, (1, 512, h, 128), torch.bfloat16).cuda()
                       for i, h in enumerate((4, 2, 2, 4)))
        o_ref, lse_ref = rm.ring_attn_fwd(q, k, v, P=1, layout="contiguous", causal=True)
        g_ref = rm.ring_attn_bwd(q, k, v, o_ref, lse_ref, do, P=1, layout="contiguous",
                                 causal=True)
        o, ctx = ulysses_dist.ulysses_forward(q, k, v, layout="contiguous", causal=True)
        grads = ulysses_dist.ulysses_backward(do, ctx)
        torch.cuda.synchronize()
        assert torch.equal(o, o_ref) and torch.equal(ctx["lse"], lse_ref)
        assert all(torch.equal(a, b) for a, b in zip(grads, g_ref))
        o2, lse2 = ring_dist.ring_forward(q, k, v, layout="contiguous", causal=True)
        g2 = ring_dist.ring_backward(q, k, v, o2, lse2, do, layout="contiguous", causal=True)
        torch.cuda.synchronize()
        # the block path (fp32 partial, then the cast) against the fused ring
        assert_max_abs(np64(o2), np64(o_ref), BF16_O_TOL, "ring_dist O")
        for name, a, b in zip(("dQ", "dK", "dV"), g2, g_ref):
            assert_grad_close(np64(a), np64(b), what=f"ring_dist {name}")
    finally:
        dist.destroy_process_group()
