"""The multi-rank ring (``ring_dist``) with its shard pairs on the CUDA
kernels, on one GPU.

The ranks are threads of this process and the point-to-point transfers go
through an in-process stand-in for torch.distributed's P2P calls
(``tests/_thread_ranks.py``: host hand-offs of stream-ordered copies, so no
kernel ever waits for another rank's kernel).  What this checks is the kernel
side of the schedule (the fp32 partials merged in place, the travelling fp32
dK / dV accumulators, the final casts); the transfers themselves are checked
over real gloo ranks on the CPU.  Results are compared with the unsharded
fp64 oracle."""

import numpy as np
import pytest
import torch

from oracle import attention as oatt
from oracle import layouts as olay
from sequence_attention_rm_b200 import ring_dist, synthetic
from tests._helpers import (BF16_LSE_TOL, BF16_O_TOL, F32_TOL, assert_grad_close, assert_max_abs,
                            gpu, np64)
from tests._thread_ranks import run_ranks

pytestmark = gpu


CASES = [
    # dtype, B, Hq, Hkv, N, d, P, layout, causal, segments
    (torch.bfloat16, 1, 4, 2, 2048, 128, 4, "zigzag", True, None),
    (torch.bfloat16, 1, 4, 2, 2048, 128, 2, "zigzag", True, None),
    (torch.bfloat16, 2, 2, 1, 1536, 128, 3, "striped", True, None),
    (torch.bfloat16, 1, 2, 2, 1024, 128, 4, "contiguous", True, None),
    (torch.bfloat16, 1, 4, 2, 768, 64, 2, "contiguous", False, None),
    (torch.float32, 1, 2, 1, 512, 64, 4, "zigzag", True, None),
    # packed: boundaries inside shards and across them; right padding with a
    # one-token entry
    (torch.bfloat16, 1, 4, 2, 2048, 128, 4, "zigzag", True, ("packed", [0, 1, 700, 1300, 2040, 2048])),
    (torch.float32, 3, 2, 1, 512, 64, 2, "striped", True, ("padded", [1, 512, 300])),
]


@pytest.mark.parametrize("dtype,B,Hq,Hkv,N,d,P,layout,causal,segments", CASES)
def test_ring_dist_schedule_on_the_kernels(dtype, B, Hq, Hkv, N, d, P, layout, causal, segments):
    seed = 7000 + N + P
    q = synthetic.tensor(seed, (B, N, Hq, d), dtype)
    k = synthetic.tensor(seed + 1, (B, N, Hkv, d), dtype)
    v = synthetic.tensor(seed + 2, (B, N, Hkv, d), dtype)
    do = synthetic.tensor(seed + 3, (B, N, Hq, d), dtype)
    pos = [olay.rank_positions(layout, N, P, r) for r in range(P)]
    segs, seg = {}, None
    if segments is not None:
        kind, vals = segments
        t32 = torch.tensor(vals, dtype=torch.int32, device="cuda")
        if kind == "packed":
            segs, seg = {"cu_seqlens": t32}, oatt.segments_from_boundaries(np.array(vals), N)
        else:
            segs, seg = {"seq_lens": t32}, oatt.segments_from_lengths(np.array(vals), N)
    shard = lambda x, r: x[:, torch.from_numpy(pos[r])].contiguous().cuda()

    def rank(r):
        qr, kr, vr, dor = shard(q, r), shard(k, r), shard(v, r), shard(do, r)
        kept = [x.clone() for x in (qr, kr, vr, dor)]
        o, lse = ring_dist.ring_forward(qr, kr, vr, layout=layout, causal=causal, **segs)
        grads = ring_dist.ring_backward(qr, kr, vr, o, lse, dor, layout=layout, causal=causal,
                                        **segs)
        assert all(torch.equal(a, b) for a, b in zip((qr, kr, vr, dor), kept)), "inputs written"
        return o, lse, grads

    out = run_ranks(ring_dist, P, rank)
    o_ref, l_ref = oatt.attention_forward(np64(q), np64(k), np64(v), causal=causal, seg=seg)
    g_ref = oatt.attention_backward(np64(q), np64(k), np64(v), np64(do), causal=causal, seg=seg)
    o_tol, l_tol = (F32_TOL, F32_TOL) if dtype == torch.float32 else (BF16_O_TOL, BF16_LSE_TOL)
    g_tol = F32_TOL if dtype == torch.float32 else None
    for r, (o, lse, grads) in enumerate(out):
        assert o.dtype == dtype and all(g.dtype == dtype for g in grads)
        assert_max_abs(np64(o), o_ref[:, pos[r]], o_tol, f"O rank {r}")
        assert_max_abs(np64(lse), l_ref[:, :, pos[r]], l_tol, f"LSE rank {r}")
        for name, g, ref in zip(("dQ", "dK", "dV"), grads, g_ref):
            kw = {} if g_tol is None else {"tol": g_tol}
            assert_grad_close(np64(g), ref[:, pos[r]], what=f"{name} rank {r}", **kw)


def test_convert_f32_rounds_to_nearest_even():
    """rm_convert_f32 against torch's own fp32 -> bf16 cast (round to nearest
    even), on values that include exact ties and the fp32 -> fp32 copy."""
    from sequence_attention_rm_b200 import rm
    x = synthetic.tensor(99, (2, 300, 3, 40), torch.float32, scale=3.0)
    ties = torch.tensor([1 + 2 ** -8, 1 + 3 * 2 ** -8, -(1 + 2 ** -8), 2 ** -130], dtype=torch.float32)
    x.view(-1)[:4] = ties
    xd = x.cuda()
    assert torch.equal(rm.convert_f32(xd, torch.bfloat16).cpu(), x.to(torch.bfloat16))
    assert torch.equal(rm.convert_f32(xd, torch.float32).cpu(), x)
