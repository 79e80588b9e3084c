"""The multi-rank ring (``ring_dist``) on CPU: 1 to 4 gloo ranks, with the
shard-pair arithmetic supplied by the fp64 oracle instead of the CUDA
kernels, so that what is checked is the communication schedule (Mosaic, "How
Ring Attention Works": each device keeps its query chunk and passes KV
chunks around the ring; ringmaster, "Status": a ring backward).  Every rank
compares its own shard of O, LSE, dQ, dK and dV with the unsharded oracle."""

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


class OracleBlocks:
    """The shard-pair operations of ring_dist in fp64 numpy (CPU tensors)."""

    acc_dtype = torch.float64

    def __init__(self):
        from oracle import attention, layouts, merge
        self.att, self.lay, self.mrg = attention, layouts, merge

    def _pos(self, layout, N, P, r):
        return self.lay.rank_positions(layout, N, P, r)

    def _seg(self, segs, N):
        if segs["cu_seqlens"] is not None:
            return self.att.segments_from_boundaries(segs["cu_seqlens"].numpy(), N)
        if segs["seq_lens"] is not None:
            return self.att.segments_from_lengths(segs["seq_lens"].numpy(), N)
        return None

    def block_fwd(self, q, k, v, *, N, P, layout, causal, q_rank, kv_rank, scale, segs):
        o, l = self.att.attention_forward(q.numpy(), k.numpy(), v.numpy(), scale, causal,
                                          q_pos=self._pos(layout, N, P, q_rank),
                                          k_pos=self._pos(layout, N, P, kv_rank),
                                          seg=self._seg(segs, N))
        return torch.from_numpy(o), torch.from_numpy(l)

    def merge_into(self, o_acc, lse_acc, o_new, lse_new):
        o, l = self.mrg.lse_merge([o_acc.numpy(), o_new.numpy()], [lse_acc.numpy(), lse_new.numpy()])
        o_acc.copy_(torch.from_numpy(o))
        lse_acc.copy_(torch.from_numpy(l))

    def finish(self, o_acc, lse_acc, dtype):
        return o_acc.to(dtype)

    def delta(self, o, dout):
        return torch.from_numpy(self.att.delta_from_output(dout.numpy(), o.numpy()))

    def block_bwd(self, q, k, v, dout, lse, delta, dq, dk, dv, *, N, P, layout, causal, q_rank,
                  kv_rank, scale, segs):
        g = self.att.attention_backward_block(q.numpy(), k.numpy(), v.numpy(), dout.numpy(),
                                              lse.numpy(), delta.numpy(), scale, causal,
                                              q_pos=self._pos(layout, N, P, q_rank),
                                              k_pos=self._pos(layout, N, P, kv_rank),
                                              seg=self._seg(segs, N))
        for acc, x in zip((dq, dk, dv), g):
            acc += torch.from_numpy(x)

    def cast(self, acc, dtype):
        return acc.to(dtype)


def _segments(kind, N, B):
    """Seeded segment descriptions: packed boundaries (B = 1) or right-padding
    lengths (one entry empty but one token, one full)."""
    if kind == "packed":
        cuts = sorted({0, N, 1, N // 3, N // 3 + 5, N - 2})
        return {"cu_seqlens": torch.tensor(cuts, dtype=torch.int32), "seq_lens": None}
    if kind == "padded":
        lens = [1, N, N // 2 + 3][:B]
        return {"cu_seqlens": None, "seq_lens": torch.tensor(lens, dtype=torch.int32)}
    return {"cu_seqlens": None, "seq_lens": None}


def _rank_main(rank, world, port, out_dir, layout, causal, hq, hkv, segkind="none"):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    sys.path.insert(0, ROOT)
    import torch.distributed as dist

    from oracle import attention, layouts
    from sequence_attention_rm_b200 import ring_dist
    dist.init_process_group("gloo", rank=rank, world_size=world)
    N = 8 * world if layout != "zigzag" else 16 * world
    B = 1 if segkind == "packed" else 2
    g = torch.Generator().manual_seed(1234)
    q, k, v, do = (torch.randn(B, N, h, 8, generator=g, dtype=torch.float64)
                   for h in (hq, hkv, hkv, hq))
    segs = _segments(segkind, N, B)
    seg = OracleBlocks()._seg(segs, N)
    pos = layouts.rank_positions(layout, N, world, rank)
    shard = lambda x: x[:, torch.from_numpy(pos)].contiguous()
    blocks = OracleBlocks()
    mine = [shard(x) for x in (q, k, v, do)]
    kept = [x.clone() for x in mine]
    qr, kr, vr, dor = mine
    o, lse = ring_dist.ring_forward(qr, kr, vr, layout=layout, causal=causal, blocks=blocks,
                                    **segs)
    grads = ring_dist.ring_backward(qr, kr, vr, o, lse, dor, layout=layout, causal=causal,
                                    blocks=blocks, **segs)
    o_ref, l_ref = attention.attention_forward(q.numpy(), k.numpy(), v.numpy(), causal=causal,
                                               seg=seg)
    g_ref = attention.attention_backward(q.numpy(), k.numpy(), v.numpy(), do.numpy(),
                                         causal=causal, seg=seg)
    err = {
        "o": float(np.abs(o.numpy() - o_ref[:, pos]).max()),
        "lse": float(np.nanmax(np.where(np.isneginf(l_ref[:, :, pos]) &
                                        np.isneginf(lse.numpy()), 0.0,
                                        np.abs(lse.numpy() - l_ref[:, :, pos])))),
    }
    for name, got, ref in zip(("dq", "dk", "dv"), grads, g_ref):
        err[name] = float(np.abs(got.numpy() - ref[:, pos]).max())
    err["inputs_changed"] = float(not all(torch.equal(a, b) for a, b in zip(mine, kept)))
    dist.barrier()
    dist.destroy_process_group()
    with open(os.path.join(out_dir, f"rank{rank}.json"), "w") as f:
        json.dump(err, f)


@pytest.mark.timeout(300)
@pytest.mark.parametrize("world,layout,causal,hq,hkv,segkind", [
    (2, "zigzag", True, 4, 2, "none"), (3, "striped", True, 2, 1, "none"),
    (4, "contiguous", True, 2, 2, "none"), (2, "contiguous", False, 2, 1, "none"),
    (4, "zigzag", True, 2, 1, "none"), (3, "contiguous", True, 4, 2, "none"),
    (3, "zigzag", True, 2, 1, "packed"), (2, "striped", False, 2, 2, "padded"),
    (1, "zigzag", True, 2, 1, "none")])
def test_ring_over_gloo_ranks_equals_unsharded(tmp_path, world, layout, causal, hq, hkv,
                                                segkind):
    mp.spawn(_rank_main, args=(world, _free_port(), str(tmp_path), layout, causal, hq, hkv,
                               segkind), nprocs=world, join=True)
    for r in range(world):
        err = json.load(open(tmp_path / f"rank{r}.json"))
        for name, e in err.items():
            assert e < 1e-10, f"rank {r} {name}: {e:.3e}"


def test_empty_pairs_are_the_contiguous_future_shards():
    sys.path.insert(0, ROOT)
    from sequence_attention_rm_b200.ring_dist import pair_is_empty
    assert pair_is_empty("contiguous", 64, 4, 1, 2, True)
    assert not pair_is_empty("contiguous", 64, 4, 2, 1, True)
    assert not pair_is_empty("contiguous", 64, 4, 1, 2, False)
    for layout in ("zigzag", "striped"):
        assert not any(pair_is_empty(layout, 64, 4, r, s, True) for r in range(4) for s in range(4))


def _absent_rank_main(rank, world, port, out_dir, which):
    """Every rank but the last joins the exchange; the last never does (it
    sleeps past the process group's timeout, then exits)."""
    import datetime
    import time
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    sys.path.insert(0, ROOT)
    import torch.distributed as dist

    from sequence_attention_rm_b200 import ring_dist, ulysses_dist
    dist.init_process_group("gloo", rank=rank, world_size=world,
                            timeout=datetime.timedelta(seconds=3))
    if rank == world - 1:
        time.sleep(10)
        return
    x = torch.randn(1, 8, 2, 8, dtype=torch.float64)
    t0 = time.time()
    try:
        if which == "ring":
            ring_dist.ring_forward(x, x, x, layout="contiguous", causal=True, blocks=OracleBlocks())
        else:
            from tests.test_ulysses_dist_gloo import OracleOps
            ulysses_dist.ulysses_forward(x, x, x, layout="contiguous", causal=True, ops=OracleOps())
        outcome = "returned"
    except Exception as e:  # the expected path: the exchange times out
        outcome = f"raised: {type(e).__name__}: {str(e)[:200]}"
    with open(os.path.join(out_dir, f"rank{rank}.json"), "w") as f:
        json.dump({"outcome": outcome, "seconds": time.time() - t0}, f)


@pytest.mark.timeout(120)
@pytest.mark.parametrize("which", ["ring", "ulysses"])
def test_a_rank_that_never_joins_ends_the_others_with_an_error(tmp_path, which):
    """Failure made on the host: one rank never reaches the exchange; the
    others' transfers end with an error after the process group's timeout
    (3 s) instead of waiting for good."""
    mp.spawn(_absent_rank_main, args=(2, _free_port(), str(tmp_path), which), nprocs=2,
             join=True)
    res = json.load(open(tmp_path / "rank0.json"))
    assert res["outcome"].startswith("raised"), res
    assert res["seconds"] < 30, res
