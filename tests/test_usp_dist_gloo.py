"""USP over real ranks (``usp_dist``) on CPU: 4 gloo ranks split as 2 ring x
2 Ulysses, 4 x 1 and 1 x 4, with the arithmetic from the fp64 oracle (the
blocks of ``test_ring_dist_gloo`` and the ops of ``test_ulysses_dist_gloo``),
so that what is checked is the two-level exchange: ringmaster, "Why": a
Ulysses all-to-all inside each group, the ring across the groups.  Every
rank compares its piece of O, dQ, dK and dV with the unsharded oracle."""

import json
import os
import socket
import sys

import numpy as np
import pytest
import torch
import torch.multiprocessing as mp

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _free_port() -> int:
    with socket.socket(socket.AF_INET, socket.SOCK_STREAM) as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _rank_main(rank, world, port, out_dir, ulysses, layout, causal, hq, hkv, packed):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    sys.path.insert(0, ROOT)
    import torch.distributed as dist

    from oracle import attention, layouts
    from sequence_attention_rm_b200 import usp_dist
    from tests.test_ring_dist_gloo import OracleBlocks
    from tests.test_ulysses_dist_gloo import OracleOps
    dist.init_process_group("gloo", rank=rank, world_size=world)
    u_group, r_group = usp_dist.usp_groups(ulysses)
    R = world // ulysses
    N = 16 * world
    g = torch.Generator().manual_seed(5151)
    q, k, v, do = (torch.randn(1, N, h, 8, generator=g, dtype=torch.float64)
                   for h in (hq, hkv, hkv, hq))
    segs = {"cu_seqlens": None, "seq_lens": None}
    seg = None
    if packed:
        cuts = [0, 1, N // 3, N // 3 + 5, N - 2, N]
        segs["cu_seqlens"] = torch.tensor(cuts, dtype=torch.int32)
        seg = attention.segments_from_boundaries(np.array(cuts), N)
    ring_pos = layouts.rank_positions(layout, N, R, rank // ulysses)
    pos = usp_dist.rank_piece(ring_pos, ulysses, rank % ulysses)
    shard = lambda x: x[:, torch.from_numpy(pos)].contiguous()
    mine = [shard(x) for x in (q, k, v, do)]
    kw = dict(ulysses_group=u_group, ring_group=r_group, blocks=OracleBlocks(), ops=OracleOps())
    o, ctx = usp_dist.usp_forward(*mine[:3], layout=layout, causal=causal, **kw, **segs)
    grads = usp_dist.usp_backward(mine[3], ctx, **kw)
    o_ref, _ = attention.attention_forward(q.numpy(), k.numpy(), v.numpy(), causal=causal,
                                           seg=seg)
    g_ref = attention.attention_backward(q.numpy(), k.numpy(), v.numpy(), do.numpy(),
                                         causal=causal, seg=seg)
    err = {"o": float(np.abs(o.numpy() - o_ref[:, pos]).max())}
    for name, got, ref in zip(("dq", "dk", "dv"), grads, g_ref):
        err[name] = float(np.abs(got.numpy() - ref[:, pos]).max())
    dist.barrier()
    dist.destroy_process_group()
    with open(os.path.join(out_dir, f"rank{rank}.json"), "w") as f:
        json.dump(err, f)


@pytest.mark.timeout(300)
@pytest.mark.parametrize("ulysses,layout,causal,hq,hkv,packed", [
    (2, "zigzag", True, 4, 2, False), (1, "striped", True, 2, 1, False),
    (4, "contiguous", True, 8, 4, False), (2, "contiguous", False, 2, 2, True)])
def test_usp_over_gloo_ranks_equals_unsharded(tmp_path, ulysses, layout, causal, hq, hkv, packed):
    world = 4
    mp.spawn(_rank_main, args=(world, _free_port(), str(tmp_path), ulysses, layout, causal, hq,
                               hkv, packed), nprocs=world, join=True)
    for r in range(world):
        err = json.load(open(tmp_path / f"rank{r}.json"))
        for name, e in err.items():
            assert e < 1e-10, f"rank {r} {name}: {e:.3e}"
