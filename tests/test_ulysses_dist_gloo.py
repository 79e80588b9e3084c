"""Ulysses attention over real ranks (``ulysses_dist``) on CPU: 1, 2 and 4 gloo
ranks exchange with all_to_all_single, with the pack / unpack and the
attention supplied by the fp64 oracle (``oracle/repack.py`` index loops and
the rank-major ``oracle/ring.py``), so that what is checked is the exchange:
ringmaster, "Why": after the all-to-all each rank holds the whole sequence
for its heads, and the reverse all-to-all returns O to sequence shards.
Every rank compares its shard of O, dQ, dK and dV with the unsharded oracle."""

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


class OracleOps:
    """ulysses_dist's pack / unpack / attention in fp64 numpy (CPU tensors)."""

    def __init__(self):
        from oracle import attention, repack, ring
        self.att, self.rep, self.ring = attention, repack, ring

    def pack(self, x, P):
        L, H, d = x.shape
        y = self.rep.seq_to_head(x.numpy().reshape(P, L // P, H, d), P)
        return torch.from_numpy(np.ascontiguousarray(y)).view(P, L, H // P, d)

    def unpack(self, y, P):
        _, L, HP, d = y.shape
        x = self.rep.head_to_seq(y.numpy().reshape(P, L, HP, d), P)
        return torch.from_numpy(np.ascontiguousarray(x)).view(L, HP * P, d)

    def _seg(self, segs, N):
        if segs["cu_seqlens"] is not None:
            return self.att.segments_from_boundaries(segs["cu_seqlens"].numpy(), N)
        if segs["seq_lens"] is not None:
            return self.att.segments_from_lengths(segs["seq_lens"].numpy(), N)
        return None

    def attn_fwd(self, q, k, v, *, P, layout, causal, scale, segs):
        o, l = self.ring.ring_forward(q.numpy(), k.numpy(), v.numpy(), layout, P, causal, scale,
                                      seg=self._seg(segs, q.shape[1]))
        return torch.from_numpy(o), torch.from_numpy(l)

    def attn_bwd(self, q, k, v, o, lse, dout, *, P, layout, causal, scale, segs):
        g = self.ring.ring_backward(q.numpy(), k.numpy(), v.numpy(), o.numpy(), lse.numpy(),
                                    dout.numpy(), layout, P, causal, scale,
                                    seg=self._seg(segs, q.shape[1]))
        return tuple(torch.from_numpy(x) for x in g)


def _segments(kind, N, B):
    if kind == "packed":
        cuts = sorted({0, N, 1, N // 3, N // 3 + 5, N - 2})
        return {"cu_seqlens": torch.tensor(cuts, dtype=torch.int32), "seq_lens": None}
    if kind == "padded":
        lens = [1, N, N // 2 + 3][:B]
        return {"cu_seqlens": None, "seq_lens": torch.tensor(lens, dtype=torch.int32)}
    return {"cu_seqlens": None, "seq_lens": None}


def _rank_main(rank, world, port, out_dir, layout, causal, B, hq, hkv, segkind):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    sys.path.insert(0, ROOT)
    import torch.distributed as dist

    from oracle import attention, layouts
    from sequence_attention_rm_b200 import ulysses_dist
    dist.init_process_group("gloo", rank=rank, world_size=world)
    N = 16 * world
    g = torch.Generator().manual_seed(4321)
    q, k, v, do = (torch.randn(B, N, h, 8, generator=g, dtype=torch.float64)
                   for h in (hq, hkv, hkv, hq))
    segs = _segments(segkind, N, B)
    ops = OracleOps()
    seg = ops._seg(segs, N)
    pos = layouts.rank_positions(layout, N, world, rank)
    shard = lambda x: x[:, torch.from_numpy(pos)].contiguous()
    mine = [shard(x) for x in (q, k, v, do)]
    kept = [x.clone() for x in mine]
    o, ctx = ulysses_dist.ulysses_forward(*mine[:3], layout=layout, causal=causal, ops=ops, **segs)
    grads = ulysses_dist.ulysses_backward(mine[3], ctx, ops=ops)
    o_ref, _ = attention.attention_forward(q.numpy(), k.numpy(), v.numpy(), causal=causal,
                                           seg=seg)
    g_ref = attention.attention_backward(q.numpy(), k.numpy(), v.numpy(), do.numpy(),
                                         causal=causal, seg=seg)
    err = {"o": float(np.abs(o.numpy() - o_ref[:, pos]).max())}
    for name, got, ref in zip(("dq", "dk", "dv"), grads, g_ref):
        err[name] = float(np.abs(got.numpy() - ref[:, pos]).max())
    # the round trip alone is the identity
    back = ulysses_dist.head_to_seq(ulysses_dist.seq_to_head(mine[0], ops=ops), ops=ops)
    err["round_trip"] = float((back - mine[0]).abs().max())
    err["inputs_changed"] = float(not all(torch.equal(a, b) for a, b in zip(mine, kept)))
    dist.barrier()
    dist.destroy_process_group()
    with open(os.path.join(out_dir, f"rank{rank}.json"), "w") as f:
        json.dump(err, f)


@pytest.mark.timeout(300)
@pytest.mark.parametrize("world,layout,causal,B,hq,hkv,segkind", [
    (2, "zigzag", True, 1, 4, 2, "none"), (4, "striped", True, 2, 4, 4, "none"),
    (2, "contiguous", False, 1, 2, 2, "packed"), (4, "contiguous", True, 1, 8, 4, "none"),
    (2, "zigzag", True, 3, 2, 2, "padded"), (1, "striped", True, 1, 2, 1, "none")])
def test_ulysses_over_gloo_ranks_equals_unsharded(tmp_path, world, layout, causal, B, hq, hkv,
                                                   segkind):
    mp.spawn(_rank_main, args=(world, _free_port(), str(tmp_path), layout, causal, B, hq, hkv,
                               segkind), nprocs=world, join=True)
    for r in range(world):
        err = json.load(open(tmp_path / f"rank{r}.json"))
        for name, e in err.items():
            assert e < 1e-10, f"rank {r} {name}: {e:.3e}"


def test_ulysses_rejects_indivisible_heads():
    sys.path.insert(0, ROOT)
    from sequence_attention_rm_b200.ulysses_dist import _check
    with pytest.raises(ValueError):
        _check(torch.empty(1, 8, 3, 4), 2)  # 3 heads over 2 ranks
    with pytest.raises(ValueError):
        _check(torch.empty(1, 6, 4, 4), 4)  # 6 local tokens over 4 ranks
    _check(torch.empty(1, 8, 4, 4), 4)
