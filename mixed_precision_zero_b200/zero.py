"""One data-parallel step of a rank's shard, with the rank-loss check, and the
ZeRO-2 step over peer memory with its cross-rank ordering.

Every rank of a ZeRO / FSDP job steps its own shard, but the overflow flag,
the global gradient norm and so the loss scale and clip coefficient belong to
the whole model ("GPT-NeoX: how it opened the door to democratised 100B-scale
training" (ainews.cool), "技术深度解析"; the OPT summary, "方法适配").  A step
is therefore pass 1 (``grad_stats``), an all-reduce (SUM) of its 16 bytes
of statistics, then the shared decision and pass 2 (``apply``).

The OPT run lost hosts and restarted dozens of times (same summary).  Here a
rank that died or stopped answering shows up as a failed collective: the
process group's timeout bounds the wait, and ``zero_step`` raises
``RankLost``.  Pass 1 writes only the statistics, so at that point this
rank's shard -- state arrays, loss scale, counters -- is still exactly the
previous step's: save it (``state_dict`` plus the caller's tensors) and
restart from there.

Under ZeRO-2 through peer memory (``peer.PeerMap``) pass 1 reads every rank's
copy of this rank's gradient slice and pass 2 stores the cast into every
rank's full-weight buffer, so the ranks' streams must be ordered against each
other, which nothing in a single rank's stream does.  ``zero2_step`` puts a
stream-ordered barrier across the ranks on both sides of the step:

* before pass 1: every rank's gradients of this step are complete;
* after pass 2: every rank's step has finished, so a rank may overwrite its
  gradient buffer (next backward) and read its full-weight buffer (next
  forward).

A barrier orders the GPU work of the ranks; it never waits on the GPU from
the host and never spins in a kernel.
"""
from __future__ import annotations


class RankLost(RuntimeError):
    """A collective of the step failed: a rank is gone or timed out.  Raised
    before pass 2, the shard that raised it has not taken the step."""


def all_reduce_stats(stats, group=None) -> None:
    """SUM-all-reduce the 16-byte statistics in place.  Over gloo a CUDA
    tensor goes through host memory; NCCL reduces it on the device."""
    import torch.distributed as dist
    if stats.is_cuda and dist.get_backend(group) == "gloo":
        host = stats.cpu()
        dist.all_reduce(host, group=group)
        stats.copy_(host)
    else:
        dist.all_reduce(stats, group=group)


def zero_step(shard, grads, params, lr: float, stats, group=None):
    """Pass 1, the all-reduce, then the shared decision and pass 2; returns the
    step's result.  `stats`: a float64 tensor of 2 on the shard's device."""
    shard.grad_stats(grads, params, stats)
    try:
        all_reduce_stats(stats, group)
    except Exception as exc:  # the collective's own error (connection lost, timeout)
        raise RankLost(f"the statistics all-reduce failed: {exc}") from exc
    return shard.apply(grads, params, lr, stats)


# ---------------------------------------------------------------- stream barriers

class NullBarrier:
    """One rank: nothing to order."""

    def __call__(self, stream=None) -> None:
        return None


class NcclStreamBarrier:
    """A one-element NCCL all-reduce on the stream.  The collective finishes on
    a rank only once every rank's stream has reached it, and the stream waits
    for it without the host waiting; it can be captured in a CUDA graph."""

    def __init__(self, group=None, device=None):
        import torch
        self.group = group
        self.flag = torch.zeros(1, dtype=torch.int32, device=device or torch.cuda.current_device())

    def __call__(self, stream=None) -> None:
        import torch
        import torch.distributed as dist
        stream = stream or torch.cuda.current_stream(self.flag.device)
        with torch.cuda.stream(stream):
            dist.all_reduce(self.flag, group=self.group)


class IpcEventBarrier:
    """Interprocess CUDA events, for ranks whose process group carries no
    device collectives (gloo; also several processes on one GPU).

    Every rank owns two events that the others open through their IPC
    handles.  Crossing r of the barrier on a rank: record its event r mod 2
    on the stream; a host barrier over the group (it only tells each rank
    that the others have *issued* their records, and never waits for the
    GPU); then the stream waits on every other rank's event r mod 2.  A wait
    on an event refers to the last record issued before it, hence the host
    barrier.  With two events per rank no rank can record crossing r + 2
    before every rank has issued its waits of crossing r (that needs the host
    barrier of crossing r + 1), so no wait ever takes a later crossing's
    record for its own.

    `event`, `open_event`, `host_barrier` and `exchange` (the all-gather of
    the event handles) are injectable for tests of the protocol without a
    GPU."""

    def __init__(self, group=None, *, event=None, open_event=None, host_barrier=None, exchange=None):
        import torch.distributed as dist
        self.group = group
        self.rank = dist.get_rank(group)
        self.world = dist.get_world_size(group)
        if event is None:
            import torch

            def event():
                return torch.cuda.Event(interprocess=True)
        if open_event is None:
            import torch

            def open_event(handle):
                return torch.cuda.Event.from_ipc_handle(torch.cuda.current_device(), handle)
        self._host_barrier = host_barrier or (lambda: dist.barrier(group=group))
        if exchange is None:
            def exchange(obj):
                out = [None] * self.world
                dist.all_gather_object(out, obj, group=group)
                return out
        self.own = [event(), event()]
        handles = exchange([e.ipc_handle() for e in self.own])
        self.peers = [[None, None] if r == self.rank else [open_event(h) for h in handles[r]]
                      for r in range(self.world)]
        self.crossing = 0

    def __call__(self, stream=None) -> None:
        if stream is None:
            import torch
            stream = torch.cuda.current_stream()
        p = self.crossing & 1
        self.crossing += 1
        self.own[p].record(stream)
        self._host_barrier()
        for r in range(self.world):
            if r != self.rank:
                stream.wait_event(self.peers[r][p])


def make_stream_barrier(group=None):
    """The stream barrier for `group`: none for one rank, a one-element
    all-reduce over NCCL, interprocess events otherwise."""
    import torch.distributed as dist
    if dist.get_world_size(group) == 1:
        return NullBarrier()
    if dist.get_backend(group) == "nccl":
        return NcclStreamBarrier(group)
    return IpcEventBarrier(group)


def zero2_step(shard, grad_ptrs, params, lr: float, stats, barrier, group=None):
    """One ZeRO-2 step over peer memory: barrier (every rank's gradients are
    written), pass 1 over every rank's copy of this rank's slice, the
    statistics all-reduce, pass 2 with the weight copies into the peers'
    buffers, barrier (every rank's step is done).  `grad_ptrs`: the
    world-size peer pointers of ``peer.zero2_grad_ptrs``; `barrier`: from
    ``make_stream_barrier``.  Everything runs on the current stream; the
    gradient writes and weight reads of the caller's next iteration go on the
    same stream, after this call."""
    try:
        barrier()
    except Exception as exc:
        raise RankLost(f"the barrier before the step failed: {exc}") from exc
    res = zero_step(shard, grad_ptrs, params, lr, stats, group)
    barrier()
    return res
