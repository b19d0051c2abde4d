"""One data-parallel step of a rank's shard, with the rank-loss check.

Every rank of a ZeRO / FSDP job steps its own shard, but the overflow flag,
the global gradient norm and so the loss scale and clip coefficient belong to
the whole model ("GPT-NeoX: how it opened the door to democratised 100B-scale
training" (ainews.cool), "技术深度解析"; the OPT summary, "方法适配").  A step
is therefore pass 1 (``grad_stats``), an all-reduce (SUM) of its 16 bytes
of statistics, then the shared decision and pass 2 (``apply``).

The OPT run lost hosts and restarted dozens of times (same summary).  Here a
rank that died or stopped answering shows up as a failed all-reduce: the
process group's timeout bounds the wait, and ``zero_step`` raises
``RankLost``.  Pass 1 writes only the statistics, so at that point this
rank's shard -- state arrays, loss scale, counters -- is still exactly the
previous step's: save it (``state_dict`` plus the caller's tensors) and
restart from there.
"""
from __future__ import annotations


class RankLost(RuntimeError):
    """The statistics all-reduce failed: a rank is gone or timed out.  The
    shard that raised it has not taken the step."""


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
