"""The ZeRO-2 step's cross-rank ordering, on CPU (gloo, 2 and 3 ranks).

zero.IpcEventBarrier orders the ranks' streams with interprocess CUDA events:
record this rank's event of the crossing's parity, a host barrier (only to know
the peers' records are issued), then wait on the peers' events of the same
parity.  Here the events are stand-ins that keep, in memory shared by the
ranks, how many records each event has had; a wait notes which record it
refers to (the last one issued).  Every wait of crossing r must refer to
exactly the peers' record of crossing r -- not an earlier one (the ordering
would be lost) and not a later one (the wait would stall a crossing) -- under
random delays between the calls.  zero2_step's order of operations and its RankLost
are checked with a stand-in shard.
"""
import os
import random
import socket
import time

import pytest
import torch.multiprocessing as mp

CROSSINGS = 12


def _free_port():
    s = socket.socket()
    s.bind(("127.0.0.1", 0))
    port = s.getsockname()[1]
    s.close()
    return port


class _Event:
    def __init__(self, counts, key):
        self.counts, self.key = counts, key

    def record(self, stream):
        self.counts[self.key] = self.counts.get(self.key, 0) + 1

    def ipc_handle(self):
        return self.key


class _Stream:
    def __init__(self, counts, log):
        self.counts, self.log = counts, log

    def wait_event(self, ev):
        self.log.append((ev.key, self.counts.get(ev.key, 0)))


def _rank_barrier(rank, world, port, counts, q):
    import torch.distributed as dist

    from mixed_precision_zero_b200.zero import IpcEventBarrier
    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        made = []

        def event():
            e = _Event(counts, (rank, len(made)))
            made.append(e)
            return e

        b = IpcEventBarrier(event=event, open_event=lambda h: _Event(counts, tuple(h)))
        rng = random.Random(rank * 7919)
        log = []
        stream = _Stream(counts, log)
        for r in range(CROSSINGS):
            time.sleep(rng.random() * 0.02)
            before = len(log)
            b(stream)
            q.put((rank, r, log[before:]))
        dist.barrier()
    finally:
        dist.destroy_process_group()


@pytest.mark.parametrize("world", [2, 3])
def test_ipc_event_barrier_waits_refer_to_the_same_crossing(world):
    ctx = mp.get_context("spawn")
    mgr = ctx.Manager()
    counts = mgr.dict()
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_rank_barrier, args=(r, world, port, counts, q)) for r in range(world)]
    for p in procs:
        p.start()
    got = [q.get(timeout=120) for _ in range(world * CROSSINGS)]
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    for rank, r, waits in got:
        # one wait per other rank and crossing, on that rank's event of the crossing's
        # parity, referring to its (r // 2 + 1)-th record of that event: the same crossing's
        assert waits == [((p, r % 2), r // 2 + 1) for p in range(world) if p != rank], (rank, r, waits)


class _Shard:
    def __init__(self, log):
        self.log = log

    def grad_stats(self, grads, params, stats):
        self.log.append("pass1")

    def apply(self, grads, params, lr, stats):
        self.log.append("pass2")
        return "result"


def _rank_zero2(rank, world, port, q):
    import torch
    import torch.distributed as dist

    from mixed_precision_zero_b200.zero import RankLost, zero2_step
    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        log = []
        stats = torch.tensor([1.0 + rank, 0.0], dtype=torch.float64)
        res = zero2_step(_Shard(log), [0, 0], None, 1e-3, stats, lambda: log.append("barrier"))
        out = {"log": log, "res": res, "stats": stats.tolist()}

        def broken():
            raise RuntimeError("peer gone")
        log2 = []
        try:
            zero2_step(_Shard(log2), [0, 0], None, 1e-3, stats, broken)
            out["lost"] = None
        except RankLost as exc:
            out["lost"] = (str(exc), log2)
        q.put((rank, out))
    finally:
        dist.destroy_process_group()


def test_zero2_step_order_and_rank_lost():
    world = 2
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_rank_zero2, args=(r, world, port, q)) for r in range(world)]
    for p in procs:
        p.start()
    got = dict(q.get(timeout=120) for _ in range(world))
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    for r in range(world):
        o = got[r]
        assert o["log"] == ["barrier", "pass1", "pass2", "barrier"]
        assert o["res"] == "result"
        assert o["stats"] == [3.0, 0.0]             # the statistics were all-reduced between the passes
        msg, log2 = o["lost"]
        assert "barrier before the step" in msg and log2 == []   # nothing of the step ran


def test_make_stream_barrier_single_rank_is_a_no_op():
    import torch.distributed as dist

    from mixed_precision_zero_b200.zero import NullBarrier, make_stream_barrier
    port = _free_port()
    dist.init_process_group("gloo", init_method=f"tcp://127.0.0.1:{port}", rank=0, world_size=1)
    try:
        b = make_stream_barrier()
        assert isinstance(b, NullBarrier) and b() is None
    finally:
        dist.destroy_process_group()


if __name__ == "__main__":
    pytest.main([__file__, "-q"])
