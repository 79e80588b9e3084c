"""USP over real ranks (``usp_dist``) with its kernels on one GPU: 4 ranks as
threads of this process (``tests/_thread_ranks.py``), split 2 ring x 2
Ulysses and 1 x 4, compared with the unsharded fp64 oracle.  The two-level
exchange itself is checked over real gloo ranks on the CPU."""

import pytest
import torch

from oracle import attention as oatt
from oracle import layouts as olay
from sequence_attention_rm_b200 import ring_dist, synthetic, ulysses_dist, usp_dist
from tests._helpers import BF16_O_TOL, F32_TOL, assert_grad_close, assert_max_abs, gpu, np64
from tests._thread_ranks import ThreadRanks, run_ranks

pytestmark = gpu


@pytest.mark.parametrize("dtype,ulysses,Hq,Hkv,N,d,layout,causal", [
    (torch.bfloat16, 2, 4, 2, 2048, 128, "zigzag", True),
    (torch.bfloat16, 4, 8, 4, 2048, 128, "contiguous", True),
    (torch.float32, 2, 2, 2, 512, 64, "striped", False),
])
def test_usp_dist_on_the_kernels(dtype, ulysses, Hq, Hkv, N, d, layout, causal):
    world = 4
    R = world // ulysses
    seed = 8400 + N + ulysses
    q = synthetic.tensor(seed, (1, N, Hq, d), dtype)
    k = synthetic.tensor(seed + 1, (1, N, Hkv, d), dtype)
    v = synthetic.tensor(seed + 2, (1, N, Hkv, d), dtype)
    do = synthetic.tensor(seed + 3, (1, N, Hq, d), dtype)
    pos = [usp_dist.rank_piece(olay.rank_positions(layout, N, R, w // ulysses), ulysses,
                               w % ulysses) for w in range(world)]
    fake = ThreadRanks(world)
    u_groups = [fake.new_group([r * ulysses + u for u in range(ulysses)]) for r in range(R)]
    r_groups = [fake.new_group([r * ulysses + u for r in range(R)]) for u in range(ulysses)]

    def rank(w):
        kw = dict(ulysses_group=u_groups[w // ulysses], ring_group=r_groups[w % ulysses])
        sh = lambda x: x[:, torch.from_numpy(pos[w])].contiguous().cuda()
        o, ctx = usp_dist.usp_forward(sh(q), sh(k), sh(v), layout=layout, causal=causal, **kw)
        return o, usp_dist.usp_backward(sh(do), ctx, **kw)

    out = run_ranks([ring_dist, ulysses_dist, usp_dist], world, rank, fake=fake)
    o_ref, _ = oatt.attention_forward(np64(q), np64(k), np64(v), causal=causal)
    g_ref = oatt.attention_backward(np64(q), np64(k), np64(v), np64(do), causal=causal)
    o_tol = F32_TOL if dtype == torch.float32 else BF16_O_TOL
    kw = {"tol": F32_TOL} if dtype == torch.float32 else {}
    for w, (o, grads) in enumerate(out):
        assert_max_abs(np64(o), o_ref[:, pos[w]], o_tol, f"O rank {w}")
        for name, g, ref in zip(("dQ", "dK", "dV"), grads, g_ref):
            assert_grad_close(np64(g), ref[:, pos[w]], what=f"{name} rank {w}", **kw)
