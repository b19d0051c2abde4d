"""Host logic of the peer pointers behind the fused ZeRO-2 reduce-scatter and
weight all-gather (mixed_precision_zero_b200.peer), on CPU: two gloo ranks
exchange real records through torch.distributed, with the CUDA IPC export /
open / close replaced by fakes that record their calls."""
import os
import socket

import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp

from mixed_precision_zero_b200 import peer


def _free_port():
    s = socket.socket()
    s.bind(("127.0.0.1", 0))
    port = s.getsockname()[1]
    s.close()
    return port


class FakeIpc:
    """Handles name (rank, allocation); opening one maps it at a fixed base."""

    def __init__(self, rank):
        self.rank, self.opened, self.closed = rank, [], []

    def exporter(self, alloc):
        def export(ptr):
            return bytes([self.rank, alloc]) + bytes(62), 256 * (alloc + 1)
        return export

    def opener(self, handle):
        self.opened.append(handle[:2])
        return 0x7000_0000_0000 + 0x1_0000_0000 * handle[0] + 0x1000_0000 * handle[1]

    def closer(self, base):
        self.closed.append(base)


def _exchange(ws):
    def ex(obj):
        out = [None] * ws
        dist.all_gather_object(out, obj)
        return out
    return ex


def _worker(rank, world, port, q):
    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        fake = FakeIpc(rank)
        n = 1000                      # elements per rank's slice
        grads = torch.zeros(world * n, dtype=torch.float16)
        weights = torch.zeros(world * n, dtype=torch.float16)
        gm = peer.PeerMap(grads, rank, world, _exchange(world), exporter=fake.exporter(0), opener=fake.opener,
                          closer=fake.closer)
        # a second buffer in the SAME allocation of every rank: no second open
        gm2 = peer.PeerMap(grads, rank, world, _exchange(world), exporter=fake.exporter(0), opener=fake.opener,
                           closer=fake.closer)
        wm = peer.PeerMap(weights, rank, world, _exchange(world), exporter=fake.exporter(1), opener=fake.opener,
                          closer=fake.closer)
        res = {"grad_ptrs": peer.zero2_grad_ptrs(gm, n), "w_dsts": peer.allgather_weight_dsts(wm, n),
               "gptrs": list(gm.ptrs), "local_g": grads.data_ptr(), "local_w": weights.data_ptr(),
               "opened": list(fake.opened)}
        gm.close()
        res["closed_after_first"] = list(fake.closed)
        gm2.close()
        wm.close()
        res["closed"] = list(fake.closed)
        try:
            peer.PeerMap(torch.zeros(10 + rank, dtype=torch.float16), rank, world, _exchange(world),
                         exporter=fake.exporter(2), opener=fake.opener, closer=fake.closer)
            res["size_check"] = "missed"
        except ValueError:
            res["size_check"] = "ok"
        try:
            gm.slice_ptrs(world, n * 2)
            res["bounds_check"] = "missed"
        except ValueError:
            res["bounds_check"] = "ok"
        q.put((rank, res))
    finally:
        dist.destroy_process_group()


def test_peer_map_pointers_and_mapping_lifetime():
    world, port = 2, _free_port()
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    procs = [ctx.Process(target=_worker, args=(r, world, port, q)) for r in range(world)]
    for p in procs:
        p.start()
    out = dict(q.get(timeout=120) for _ in range(world))
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    n, es = 1000, 2
    for rank, res in out.items():
        other = 1 - rank
        gbase = 0x7000_0000_0000 + 0x1_0000_0000 * other + 0x1000_0000 * 0
        wbase = 0x7000_0000_0000 + 0x1_0000_0000 * other + 0x1000_0000 * 1
        # rank r's own buffer is its local pointer; the peer's is its mapped base + the exporter's offset
        assert res["gptrs"][rank] == res["local_g"] and res["gptrs"][other] == gbase + 256
        # the reduce-scatter reads slice `rank` of every rank's gradient, in rank order
        expect = [0, 0]
        expect[rank] = res["local_g"] + rank * n * es
        expect[other] = gbase + 256 + rank * n * es
        assert res["grad_ptrs"] == expect
        # the all-gather writes slice `rank` of every OTHER rank's weights
        assert res["w_dsts"] == [wbase + 512 + rank * n * es]
        # one open per peer allocation (two maps of one allocation share it), closed with its last user
        assert res["opened"] == [bytes([other, 0]), bytes([other, 1])]
        assert res["closed_after_first"] == []
        assert sorted(res["closed"]) == sorted([gbase, wbase])
        assert res["size_check"] == "ok" and res["bounds_check"] == "ok"


def test_peer_map_refuses_ranks_on_two_hosts():
    recs = [("hostA", bytes(64), 0, 100), ("hostB", bytes([1]) + bytes(63), 0, 100)]
    with pytest.raises(RuntimeError, match="one node"):
        peer.PeerMap(torch.zeros(50, dtype=torch.float16), 0, 2, lambda obj: recs,
                     exporter=lambda p: (bytes(64), 0), opener=lambda h: 1, closer=lambda b: None)
