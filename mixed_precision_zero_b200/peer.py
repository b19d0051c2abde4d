"""Device pointers of one buffer on every rank of a node, through CUDA IPC.

Under ZeRO stage 2 the owner of each flat slice needs every rank's copy of that
slice of the gradient, summed (the reduce-scatter), and under ZeRO stages 1/2
every rank needs every owner's updated weight slice (the all-gather)
("GPT-NeoX: how it opened the door to democratised 100B-scale training"
(ainews.cool), "技术深度解析").  The step's kernels do both without a
collective once they hold peer pointers: pass 1 ingests the K = world-size
peer slices of the gradient (pre-divide, FP32 sum, norm), and pass 2 stores
the cast into every peer's weight buffer.  ``PeerMap`` builds those pointers:
each rank exports its buffer (``neox_ipc_export``), the handles are exchanged
(``torch.distributed.all_gather_object`` by default), and each rank maps the
others' (``neox_ipc_open``).  Only the exchange runs in Python; the mapping is
the library's.
"""
from __future__ import annotations

import socket
from typing import Callable, Sequence

from ._abi import neox_ipc_close, neox_ipc_export, neox_ipc_open

# Open mappings of this process, keyed by the exporter's handle bytes: a
# process may open an allocation once, and two buffers of one peer can share
# an allocation (a caching allocator's segment).
_OPEN: dict[bytes, list] = {}


def _acquire(handle: bytes, opener: Callable[[bytes], int]) -> int:
    ent = _OPEN.get(handle)
    if ent is None:
        ent = _OPEN[handle] = [opener(handle), 0]
    ent[1] += 1
    return ent[0]


def _release(handle: bytes, closer: Callable[[int], None]) -> None:
    ent = _OPEN[handle]
    ent[1] -= 1
    if ent[1] == 0:
        del _OPEN[handle]
        closer(ent[0])


class PeerMap:
    """The address of one same-sized device buffer of every rank, valid in
    this process: ``ptrs[r]`` is rank r's buffer (this rank's own pointer for
    itself).  All ranks must call the constructor together (it exchanges)."""

    def __init__(self, tensor, rank: int, world_size: int, exchange: Callable[[object], Sequence[object]], *,
                 exporter: Callable[[int], tuple] = neox_ipc_export, opener: Callable[[bytes], int] = neox_ipc_open,
                 closer: Callable[[int], None] = neox_ipc_close):
        self.rank, self.world_size = rank, world_size
        self.nbytes = tensor.numel() * tensor.element_size()
        self._closer = closer
        self._tensor = tensor  # the exported memory must outlive every peer's mapping
        local = tensor.data_ptr()
        handle, offset = exporter(local)
        recs = list(exchange((socket.gethostname(), handle, int(offset), int(self.nbytes))))
        if len(recs) != world_size:
            raise RuntimeError(f"exchange returned {len(recs)} records for {world_size} ranks")
        hosts = {r[0] for r in recs}
        if len(hosts) != 1:
            raise RuntimeError(f"CUDA IPC maps memory within one node; ranks are on {sorted(hosts)}")
        sizes = {r[3] for r in recs}
        if len(sizes) != 1:
            raise ValueError(f"every rank's buffer must have the same size, got {sorted(sizes)} bytes")
        self.ptrs: list[int] = []
        self._held: list[bytes] = []
        try:
            for r, (_, h, off, _) in enumerate(recs):
                if r == rank:
                    self.ptrs.append(local)
                else:
                    self.ptrs.append(_acquire(h, opener) + off)
                    self._held.append(h)
        except BaseException:
            self.close()
            raise

    @classmethod
    def from_group(cls, tensor, group=None) -> "PeerMap":
        """Exchange through torch.distributed (any backend; gloo works)."""
        import torch.distributed as dist
        rank, ws = dist.get_rank(group), dist.get_world_size(group)

        def exchange(obj):
            out = [None] * ws
            dist.all_gather_object(out, obj, group=group)
            return out
        return cls(tensor, rank, ws, exchange)

    def slice_ptrs(self, index: int, slice_bytes: int) -> list[int]:
        """Slice `index` (of `slice_bytes` bytes) of every rank's buffer, in rank order."""
        if slice_bytes < 0 or index < 0 or (index + 1) * slice_bytes > self.nbytes:
            raise ValueError(f"slice {index} of {slice_bytes} bytes lies outside the {self.nbytes}-byte buffer")
        return [p + index * slice_bytes for p in self.ptrs]

    def close(self) -> None:
        """Unmap the peers' buffers (call on every rank before any exporter frees its buffer)."""
        while self._held:
            _release(self._held.pop(), self._closer)


def zero2_grad_ptrs(grads: PeerMap, slice_numel: int, elem_size: int = 2) -> list[int]:
    """The K = world-size gradient pointers of this rank's shard for the fused
    reduce-scatter: every rank's copy of slice `rank`, in rank order."""
    return grads.slice_ptrs(grads.rank, slice_numel * elem_size)


def allgather_weight_dsts(weights: PeerMap, slice_numel: int, elem_size: int = 2) -> list[int]:
    """The destinations of this rank's updated weight slice in every other
    rank's full-weight buffer (this rank's own slice is the step's params)."""
    ptrs = weights.slice_ptrs(weights.rank, slice_numel * elem_size)
    return [p for r, p in enumerate(ptrs) if r != weights.rank]
