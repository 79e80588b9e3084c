"""An in-process stand-in for torch.distributed's point-to-point and
all-to-all calls, for running several ranks as threads of one process on one
GPU (no method arithmetic here).

Every transfer is a host hand-off of a stream-ordered device copy: a send
queues a copy of its tensor, a receive copies the queued tensor into its
buffer.  As in the real backends, the n-th receive a rank posts from a peer
matches the n-th send that peer posted to it (per kind of call), whatever
order the requests are waited on.  No kernel ever waits for another rank's
kernel, so the ranks need not run at the same time."""

import queue
import threading
import types

import torch


class _Req:
    def __init__(self, fn=None):
        self.fn = fn

    def wait(self):
        if self.fn is not None:
            self.fn()


class ThreadRanks:
    def __init__(self, world):
        self.world = world
        self.local = threading.local()
        self.lock = threading.Lock()
        self.slots = {}
        self.posted = {}
        self.isend, self.irecv = "isend", "irecv"

    def P2POp(self, op, tensor, peer, group=None):
        return types.SimpleNamespace(op=op, tensor=tensor, peer=peer)

    def new_group(self, ranks, backend=None):
        """A group: its members' global ranks, in group-rank order."""
        return types.SimpleNamespace(ranks=list(ranks))

    def get_world_size(self, group=None):
        return self.world if group is None else len(group.ranks)

    def get_rank(self, group=None):
        me = self.local.rank
        return me if group is None else group.ranks.index(me)

    def get_global_rank(self, group, r):
        return r if group is None else group.ranks[r]

    def _slot(self, src, dst, kind, role):
        """The queue of the next message from src to dst of this kind (the
        sender's and the receiver's counters advance separately)."""
        with self.lock:
            key = (src, dst, kind, role)
            n = self.posted.get(key, 0)
            self.posted[key] = n + 1
            return self.slots.setdefault((src, dst, kind, n), queue.Queue(maxsize=1))

    def batch_isend_irecv(self, ops):
        me = self.local.rank
        reqs = []
        for op in ops:
            if op.op == self.isend:
                self._slot(me, op.peer, "p2p", "send").put(op.tensor.clone())
                reqs.append(_Req())
            else:
                slot, buf = self._slot(op.peer, me, "p2p", "recv"), op.tensor
                reqs.append(_Req(lambda slot=slot, buf=buf: buf.copy_(slot.get(timeout=120))))
        return reqs

    def all_to_all_single(self, output, input, group=None):
        me = self.local.rank
        members = list(range(self.world)) if group is None else group.ranks
        for dst, chunk in zip(members, input.chunk(len(members))):
            self._slot(me, dst, "a2a", "send").put(chunk.clone())
        for src, chunk in zip(members, output.chunk(len(members))):
            chunk.copy_(self._slot(src, me, "a2a", "recv").get(timeout=120))


def run_ranks(module, world, fn, fake=None):
    """Run fn(rank) for every rank in its own thread with module.dist (a
    module or a list of modules) replaced by a ThreadRanks; returns the
    results in rank order."""
    fake = ThreadRanks(world) if fake is None else fake
    modules = module if isinstance(module, (list, tuple)) else [module]
    results, errors = [None] * world, []

    def body(r):
        fake.local.rank = r
        try:
            results[r] = fn(r)
        except BaseException as e:  # reported by the caller's thread
            errors.append(e)

    real = [m.dist for m in modules]
    for m in modules:
        m.dist = fake
    try:
        threads = [threading.Thread(target=body, args=(r,)) for r in range(world)]
        for t in threads:
            t.start()
        for t in threads:
            t.join(timeout=300)
        torch.cuda.synchronize()
    finally:
        for m, d in zip(modules, real):
            m.dist = d
    if errors:
        raise errors[0]
    return results
