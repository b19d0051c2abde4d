"""B200-native per-rank mixed-precision optimizer step over an owned flat shard.

The step (ingest + pre-divide + unscale, overflow flag, global norm, dynamic
loss scaler, global-norm clip, AdamW on FP32 master/m/v, cast to 16-bit
working weights) runs in the hand-written CUDA kernels of ``libneoxshard.so``
(C ABI: ``include/neox_shard.h``).  This package only marshals arguments:
PyTorch provides device memory and streams.

    from mixed_precision_zero_b200 import NeoxShard, Hparams
    shard = NeoxShard(master, exp_avg, exp_avg_sq, Hparams(clip_norm=1.0))
    res = shard.step([grad], params, lr=6e-4)   # res.overflow, res.grad_norm, ...
"""
from __future__ import annotations

import ctypes
from dataclasses import dataclass

from ._abi import (NEOX_BF16, NEOX_ERR_CUDA, NEOX_ERR_INVALID_ARGUMENT, NEOX_ERR_OUT_OF_MEMORY,  # noqa: F401
                   NEOX_ERR_UNSUPPORTED, NEOX_FP16, NEOX_OK, NeoxError, lib, neox_hparams,
                   neox_last_error, neox_model_state_bytes, neox_profile, neox_segment,
                   neox_shard_create, neox_shard_desc, neox_shard_destroy, neox_shard_get_profile,
                   neox_shard_get_state, neox_shard_reset_profile, neox_shard_scratch_bytes,
                   neox_shard_set_hparams, neox_shard_set_profiling, neox_shard_set_state,
                   neox_shard_step, neox_shard_step_async, neox_status_string, neox_step_result,
                   neox_tensor, neox_tensor_set, neox_multi_create, neox_multi_step, neox_multi_step_async,
                   neox_multi_rebind_grads, neox_multi_get_state, neox_multi_set_state,
                   neox_multi_set_hparams, neox_multi_destroy, neox_shard_grad_stats, neox_shard_apply,
                   neox_shard_set_weight_copies, neox_shard_get_hysteresis, neox_shard_set_hysteresis,
                   neox_multi_get_hysteresis, neox_multi_set_hysteresis, NEOX_ADAMW, NEOX_SGD,
                   NEOX_SHARD_ACCUMULATE, neox_multi_set_profiling, neox_multi_get_profile,
                   neox_multi_reset_profile)

__all__ = ["NeoxShard", "NeoxMultiShard", "Hparams", "NeoxError", "neox_shard_create", "neox_shard_step",
           "neox_shard_destroy", "neox_shard_set_hparams", "neox_shard_get_state",
           "neox_shard_set_state", "neox_status_string", "neox_last_error", "neox_model_state_bytes"]


@dataclass
class Hparams:
    beta1: float = 0.9
    beta2: float = 0.95
    eps: float = 1e-8
    clip_norm: float = 1.0
    predivide: float = 1.0
    init_scale: float = 65536.0
    scale_factor: float = 2.0
    min_scale: float = 1.0
    scale_window: int = 1000
    hysteresis: int = 1          # overflows before a back-off (0 or 1: at every overflow)
    optimizer: str = "adamw"     # "adamw" or "sgd"

    def c(self) -> neox_hparams:
        opts = {"adamw": NEOX_ADAMW, "sgd": NEOX_SGD}
        if self.optimizer not in opts:
            raise ValueError(f"optimizer must be 'adamw' or 'sgd', got {self.optimizer!r}")
        return neox_hparams(self.beta1, self.beta2, self.eps, self.clip_norm, self.predivide,
                            self.init_scale, self.scale_factor, self.min_scale, self.scale_window,
                            self.hysteresis, opts[self.optimizer])


def _ptr(g) -> int:
    return g if isinstance(g, int) else g.data_ptr()


def _dtype_code(t) -> int:
    import torch
    if t.dtype == torch.float16:
        return NEOX_FP16
    if t.dtype == torch.bfloat16:
        return NEOX_BF16
    raise TypeError(f"16-bit tensor must be float16 or bfloat16, got {t.dtype}")


class NeoxShard:
    """One owned flat shard on one GPU: caller-owned FP32 master / exp_avg /
    exp_avg_sq CUDA tensors of equal length, plus the library handle."""

    def __init__(self, master, exp_avg, exp_avg_sq, hp: Hparams | None = None, *,
                 wdtype=None, gdtype=None, segments=None, weight_decay: float = 0.0,
                 max_grads: int = 1, device: int | None = None, accumulate: bool = False):
        import torch
        hp = hp or Hparams()
        n = master.numel()
        for t in (master, exp_avg, exp_avg_sq):
            if t.dtype != torch.float32 or t.numel() != n or not t.is_contiguous():
                raise ValueError("master/exp_avg/exp_avg_sq must be contiguous float32 tensors of equal length")
        self.numel = n
        self.tensors = (master, exp_avg, exp_avg_sq)  # keep them alive with the handle
        self.wdtype = NEOX_FP16 if wdtype in (None, torch.float16) else NEOX_BF16
        self.gdtype = NEOX_FP16 if gdtype in (None, torch.float16) else NEOX_BF16
        if segments is not None:
            self._segs = (neox_segment * len(segments))(*[neox_segment(int(o), int(c), float(w))
                                                          for o, c, w in segments])
            segp, nsegs = ctypes.cast(self._segs, ctypes.POINTER(neox_segment)), len(segments)
        else:
            self._segs, segp, nsegs = None, None, 0
        desc = neox_shard_desc(n, self.wdtype, self.gdtype, segp, nsegs, float(weight_decay),
                               master.data_ptr() if n else None, exp_avg.data_ptr() if n else None,
                               exp_avg_sq.data_ptr() if n else None, int(max_grads),
                               NEOX_SHARD_ACCUMULATE if accumulate else 0)
        self.device = master.device.index if device is None else device
        if self.device is None:
            self.device = torch.cuda.current_device()
        self.handle = neox_shard_create(desc, hp.c(), self.device)

    def _check(self, grads, params):
        for g in grads:
            if isinstance(g, int):   # a raw device pointer (e.g. a peer's slice), the caller's to size
                continue
            if g.numel() != self.numel or _dtype_code(g) != self.gdtype or not g.is_contiguous():
                raise ValueError("each grad must be a contiguous 16-bit tensor of the shard's gradient type and length")
        if params.numel() != self.numel or _dtype_code(params) != self.wdtype or not params.is_contiguous():
            raise ValueError("params must be a contiguous 16-bit tensor of the shard's weight type and length")

    def step(self, grads, params, lr: float, stream=None) -> neox_step_result:
        import torch
        self._check(grads, params)
        if stream is None:
            stream = torch.cuda.current_stream(self.device)
        sp = stream.cuda_stream if hasattr(stream, "cuda_stream") else int(stream)
        return neox_shard_step(self.handle, [_ptr(g) for g in grads], params.data_ptr(), lr, sp)

    def step_async(self, grads, params, lr: float = 0.0, *, result=None, lr_device=None, stream=None) -> None:
        """Enqueue a step without waiting.  `result`: a device (or pinned) tensor
        of at least 32 bytes that receives the neox_step_result; `lr_device`: a
        float32 CUDA tensor holding the learning rate (read at run time)."""
        import torch
        self._check(grads, params)
        if stream is None:
            stream = torch.cuda.current_stream(self.device)
        sp = stream.cuda_stream if hasattr(stream, "cuda_stream") else int(stream)
        neox_shard_step_async(self.handle, [_ptr(g) for g in grads], params.data_ptr(), lr, sp,
                              None if result is None else result.data_ptr(),
                              None if lr_device is None else lr_device.data_ptr())

    def grad_stats(self, grads, params, stats, stream=None) -> None:
        """Pass 1 only: `stats` (float64 CUDA tensor of 2) receives this shard's
        {sum of squares, non-finite flag}; all-reduce it (SUM) across ranks,
        then call apply()."""
        import torch
        self._check(grads, params)
        if stats.dtype != torch.float64 or stats.numel() < 2 or not stats.is_cuda:
            raise ValueError("stats must be a float64 CUDA tensor of 2 elements")
        if stream is None:
            stream = torch.cuda.current_stream(self.device)
        sp = stream.cuda_stream if hasattr(stream, "cuda_stream") else int(stream)
        neox_shard_grad_stats(self.handle, [_ptr(g) for g in grads], params.data_ptr(), sp, stats.data_ptr())

    def apply(self, grads, params, lr: float, stats, stream=None) -> neox_step_result:
        """The step's decisions from the (all-reduced) statistics, then pass 2."""
        import torch
        self._check(grads, params)
        if stream is None:
            stream = torch.cuda.current_stream(self.device)
        sp = stream.cuda_stream if hasattr(stream, "cuda_stream") else int(stream)
        return neox_shard_apply(self.handle, [_ptr(g) for g in grads], params.data_ptr(), lr, stats.data_ptr(), sp)

    def set_weight_copies(self, dsts) -> None:
        """Extra 16-bit tensors (same length and type as params), or raw device
        pointers to such arrays, that pass 2 writes with the updated weights,
        e.g. peer-mapped slices of every rank's full-weight buffer
        (see peer.PeerMap).  An empty list removes them."""
        for d in dsts:
            if isinstance(d, int):   # a raw device pointer (e.g. a slice of a peer's weight buffer)
                continue
            if d.numel() != self.numel or _dtype_code(d) != self.wdtype or not d.is_contiguous():
                raise ValueError("each copy must be a contiguous 16-bit tensor like params")
        self._copies = list(dsts)  # keep them alive
        neox_shard_set_weight_copies(self.handle, [_ptr(d) for d in dsts])

    def set_hparams(self, hp: Hparams) -> None:
        neox_shard_set_hparams(self.handle, hp.c())

    def get_state(self):
        return neox_shard_get_state(self.handle)

    def set_state(self, scale: float, good: int, t: int) -> None:
        neox_shard_set_state(self.handle, scale, good, t)

    def get_hysteresis(self) -> int:
        return neox_shard_get_hysteresis(self.handle)

    def set_hysteresis(self, count: int) -> None:
        neox_shard_set_hysteresis(self.handle, count)

    def state_dict(self) -> dict:
        """The library-held step state for a checkpoint (master / m / v and the
        working weights are the caller's tensors and are saved with the model)."""
        scale, good, t = self.get_state()
        return {"loss_scale": scale, "good_steps": good, "applied_steps": t,
                "hysteresis_count": self.get_hysteresis()}

    def load_state_dict(self, d: dict) -> None:
        """Resume exactly where state_dict() was taken."""
        self.set_state(d["loss_scale"], d["good_steps"], d["applied_steps"])
        self.set_hysteresis(d["hysteresis_count"])

    def set_profiling(self, enable: bool) -> None:
        neox_shard_set_profiling(self.handle, enable)

    def profile(self) -> neox_profile:
        return neox_shard_get_profile(self.handle)

    def reset_profile(self) -> None:
        neox_shard_reset_profile(self.handle)

    def scratch_bytes(self) -> int:
        return neox_shard_scratch_bytes(self.handle)

    def close(self) -> None:
        if getattr(self, "handle", None):
            neox_shard_destroy(self.handle)
            self.handle = None

    def __del__(self):
        try:
            self.close()
        except Exception:
            pass


class NeoxMultiShard:
    """A shard made of separately allocated tensors (one per parameter), stepped
    as one: `tensors` is a list of dicts with keys master, exp_avg, exp_avg_sq
    (float32 CUDA tensors), params (16-bit), grads (list of K 16-bit tensors)
    and weight_decay.  All buffers are bound here and must stay alive."""

    def __init__(self, tensors, hp: Hparams | None = None, *, device: int | None = None):
        import torch
        hp = hp or Hparams()
        K = len(tensors[0]["grads"]) if tensors else 1
        self._keep = tensors
        self._grad_arrays = []
        descs = []
        wd_t = gd_t = None
        for t in tensors:
            n = t["master"].numel()
            for x in (t["master"], t["exp_avg"], t["exp_avg_sq"]):
                if x.dtype != torch.float32 or x.numel() != n or not x.is_contiguous():
                    raise ValueError("master/exp_avg/exp_avg_sq must be contiguous float32 tensors of equal length")
            if len(t["grads"]) != K:
                raise ValueError("every tensor needs the same number of gradient buffers")
            for g in [t["params"], *t["grads"]]:
                if g.numel() != n or not g.is_contiguous():
                    raise ValueError("params/grads must be contiguous and as long as master")
            wd_t = wd_t or t["params"].dtype
            gd_t = gd_t or t["grads"][0].dtype
            garr = (ctypes.c_void_p * K)(*[g.data_ptr() for g in t["grads"]])
            self._grad_arrays.append(garr)
            descs.append(neox_tensor(n, float(t.get("weight_decay", 0.0)), t["master"].data_ptr(),
                                     t["exp_avg"].data_ptr(), t["exp_avg_sq"].data_ptr(), t["params"].data_ptr(),
                                     ctypes.cast(garr, ctypes.POINTER(ctypes.c_void_p))))
        self._descs = (neox_tensor * max(1, len(descs)))(*descs)
        wcode = NEOX_BF16 if wd_t == torch.bfloat16 else NEOX_FP16
        gcode = NEOX_BF16 if gd_t == torch.bfloat16 else NEOX_FP16
        tset = neox_tensor_set(len(descs), K, wcode, gcode, ctypes.cast(self._descs, ctypes.POINTER(neox_tensor)))
        self.device = torch.cuda.current_device() if device is None else device
        self.handle = neox_multi_create(tset, hp.c(), self.device)

    @staticmethod
    def _sp(stream, device):
        import torch
        if stream is None:
            stream = torch.cuda.current_stream(device)
        return stream.cuda_stream if hasattr(stream, "cuda_stream") else int(stream)

    def step(self, lr: float, stream=None) -> neox_step_result:
        return neox_multi_step(self.handle, lr, self._sp(stream, self.device))

    def step_async(self, lr: float = 0.0, *, result=None, lr_device=None, stream=None) -> None:
        neox_multi_step_async(self.handle, lr, self._sp(stream, self.device),
                              None if result is None else result.data_ptr(),
                              None if lr_device is None else lr_device.data_ptr())

    def rebind_grads(self, grads_per_tensor) -> None:
        ptrs = [g.data_ptr() for gs in grads_per_tensor for g in gs]
        neox_multi_rebind_grads(self.handle, ptrs)

    def get_state(self):
        return neox_multi_get_state(self.handle)

    def set_state(self, scale: float, good: int, t: int) -> None:
        neox_multi_set_state(self.handle, scale, good, t)

    def get_hysteresis(self) -> int:
        return neox_multi_get_hysteresis(self.handle)

    def set_profiling(self, enable: bool) -> None:
        neox_multi_set_profiling(self.handle, enable)

    def profile(self) -> neox_profile:
        return neox_multi_get_profile(self.handle)

    def reset_profile(self) -> None:
        neox_multi_reset_profile(self.handle)

    def set_hysteresis(self, count: int) -> None:
        neox_multi_set_hysteresis(self.handle, count)

    def state_dict(self) -> dict:
        scale, good, t = self.get_state()
        return {"loss_scale": scale, "good_steps": good, "applied_steps": t,
                "hysteresis_count": self.get_hysteresis()}

    def load_state_dict(self, d: dict) -> None:
        self.set_state(d["loss_scale"], d["good_steps"], d["applied_steps"])
        self.set_hysteresis(d["hysteresis_count"])

    def set_hparams(self, hp: Hparams) -> None:
        neox_multi_set_hparams(self.handle, hp.c())

    def close(self) -> None:
        if getattr(self, "handle", None):
            neox_multi_destroy(self.handle)
            self.handle = None

    def __del__(self):
        try:
            self.close()
        except Exception:
            pass
