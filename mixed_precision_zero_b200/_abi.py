"""ctypes declarations of the C ABI in include/neox_shard.h (argument marshalling only).

The functions keep the C names.  Loading fails loudly when the CUDA library
has not been built: there is no fallback implementation of the step.
"""
from __future__ import annotations

import ctypes
import os

_PKG = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_PKG, "libneoxshard.so")

NEOX_OK = 0
NEOX_ERR_INVALID_ARGUMENT = 1
NEOX_ERR_CUDA = 2
NEOX_ERR_OUT_OF_MEMORY = 3
NEOX_ERR_UNSUPPORTED = 4

NEOX_FP16 = 0
NEOX_BF16 = 1

NEOX_ADAMW = 0
NEOX_SGD = 1

NEOX_SHARD_ACCUMULATE = 1


class neox_segment(ctypes.Structure):
    _fields_ = [("offset", ctypes.c_uint64), ("numel", ctypes.c_uint64), ("weight_decay", ctypes.c_float)]


class neox_hparams(ctypes.Structure):
    _fields_ = [("beta1", ctypes.c_float), ("beta2", ctypes.c_float), ("eps", ctypes.c_float),
                ("clip_norm", ctypes.c_float), ("predivide", ctypes.c_float),
                ("init_scale", ctypes.c_float), ("scale_factor", ctypes.c_float),
                ("min_scale", ctypes.c_float), ("scale_window", ctypes.c_int32),
                ("hysteresis", ctypes.c_int32), ("optimizer", ctypes.c_int32)]


class neox_shard_desc(ctypes.Structure):
    _fields_ = [("numel", ctypes.c_uint64), ("wdtype", ctypes.c_int), ("gdtype", ctypes.c_int),
                ("segs", ctypes.POINTER(neox_segment)), ("nsegs", ctypes.c_int32),
                ("default_weight_decay", ctypes.c_float),
                ("master", ctypes.c_void_p), ("exp_avg", ctypes.c_void_p), ("exp_avg_sq", ctypes.c_void_p),
                ("max_grads", ctypes.c_int32), ("flags", ctypes.c_int32)]


class neox_step_result(ctypes.Structure):
    _fields_ = [("overflow", ctypes.c_int32), ("grad_norm", ctypes.c_float), ("clip_coef", ctypes.c_float),
                ("loss_scale", ctypes.c_float), ("loss_scale_next", ctypes.c_float),
                ("good_steps", ctypes.c_int32), ("applied_steps", ctypes.c_int64)]

    def as_dict(self) -> dict:
        return {k: getattr(self, k) for k, _ in self._fields_}


class neox_ipc_handle(ctypes.Structure):
    _fields_ = [("bytes", ctypes.c_ubyte * 64)]


class neox_scaler_state(ctypes.Structure):
    _fields_ = [("scale", ctypes.c_float), ("good", ctypes.c_int32), ("t", ctypes.c_int64)]


class neox_tensor(ctypes.Structure):
    _fields_ = [("numel", ctypes.c_uint64), ("weight_decay", ctypes.c_float),
                ("master", ctypes.c_void_p), ("exp_avg", ctypes.c_void_p), ("exp_avg_sq", ctypes.c_void_p),
                ("params", ctypes.c_void_p), ("grads", ctypes.POINTER(ctypes.c_void_p))]


class neox_tensor_set(ctypes.Structure):
    _fields_ = [("ntensors", ctypes.c_int32), ("num_grads", ctypes.c_int32), ("wdtype", ctypes.c_int),
                ("gdtype", ctypes.c_int), ("tensors", ctypes.POINTER(neox_tensor))]


class neox_profile(ctypes.Structure):
    _fields_ = [("steps", ctypes.c_int64), ("launches", ctypes.c_int64),
                ("grad_pass_ms", ctypes.c_double), ("update_pass_ms", ctypes.c_double),
                ("last_grad_pass_ms", ctypes.c_double), ("last_update_pass_ms", ctypes.c_double)]


_lib = None
_H = ctypes.c_void_p


def lib() -> ctypes.CDLL:
    global _lib
    if _lib is None:
        if not os.path.exists(LIB_PATH):
            raise RuntimeError(
                f"CUDA library {LIB_PATH} is not built; run `python -m mixed_precision_zero_b200.build` "
                "(there is no CPU fallback for the shard step)")
        L = ctypes.CDLL(LIB_PATH)
        S = ctypes.c_int
        L.neox_shard_create.argtypes = [ctypes.POINTER(neox_shard_desc), ctypes.POINTER(neox_hparams), ctypes.c_int,
                                        ctypes.POINTER(_H)]
        L.neox_shard_create.restype = S
        L.neox_shard_step.argtypes = [_H, ctypes.POINTER(ctypes.c_void_p), ctypes.c_int32, ctypes.c_void_p,
                                      ctypes.c_float, ctypes.c_void_p, ctypes.POINTER(neox_step_result)]
        L.neox_shard_step.restype = S
        L.neox_shard_step_async.argtypes = [_H, ctypes.POINTER(ctypes.c_void_p), ctypes.c_int32, ctypes.c_void_p,
                                            ctypes.c_float, ctypes.c_void_p, ctypes.c_void_p, ctypes.c_void_p]
        L.neox_shard_step_async.restype = S
        L.neox_shard_grad_stats.argtypes = [_H, ctypes.POINTER(ctypes.c_void_p), ctypes.c_int32, ctypes.c_void_p,
                                            ctypes.c_void_p, ctypes.c_void_p]
        L.neox_shard_grad_stats.restype = S
        L.neox_shard_apply.argtypes = [_H, ctypes.POINTER(ctypes.c_void_p), ctypes.c_int32, ctypes.c_void_p,
                                       ctypes.c_float, ctypes.c_void_p, ctypes.c_void_p,
                                       ctypes.POINTER(neox_step_result)]
        L.neox_shard_apply.restype = S
        L.neox_shard_set_weight_copies.argtypes = [_H, ctypes.POINTER(ctypes.c_void_p), ctypes.c_int32]
        L.neox_shard_set_weight_copies.restype = S
        L.neox_shard_set_hparams.argtypes = [_H, ctypes.POINTER(neox_hparams)]
        L.neox_shard_set_hparams.restype = S
        L.neox_shard_get_state.argtypes = [_H, ctypes.POINTER(ctypes.c_float), ctypes.POINTER(ctypes.c_int32),
                                           ctypes.POINTER(ctypes.c_int64)]
        L.neox_shard_get_state.restype = S
        L.neox_shard_set_state.argtypes = [_H, ctypes.c_float, ctypes.c_int32, ctypes.c_int64]
        L.neox_shard_set_state.restype = S
        L.neox_shard_get_hysteresis.argtypes = [_H, ctypes.POINTER(ctypes.c_int32)]
        L.neox_shard_get_hysteresis.restype = S
        L.neox_shard_set_hysteresis.argtypes = [_H, ctypes.c_int32]
        L.neox_shard_set_hysteresis.restype = S
        L.neox_shard_destroy.argtypes = [_H]
        L.neox_shard_destroy.restype = None
        L.neox_status_string.argtypes = [S]
        L.neox_status_string.restype = ctypes.c_char_p
        L.neox_last_error.argtypes = [_H]
        L.neox_last_error.restype = ctypes.c_char_p
        L.neox_model_state_bytes.argtypes = [ctypes.c_uint64, ctypes.c_int, ctypes.c_int]
        L.neox_model_state_bytes.restype = ctypes.c_uint64
        L.neox_shard_scratch_bytes.argtypes = [_H]
        L.neox_shard_scratch_bytes.restype = ctypes.c_uint64
        L.neox_shard_set_profiling.argtypes = [_H, ctypes.c_int32]
        L.neox_shard_set_profiling.restype = S
        L.neox_shard_get_profile.argtypes = [_H, ctypes.POINTER(neox_profile)]
        L.neox_shard_get_profile.restype = S
        L.neox_shard_reset_profile.argtypes = [_H]
        L.neox_shard_reset_profile.restype = S
        L.neox_shard_step_noalloc.argtypes = [ctypes.POINTER(neox_shard_desc), ctypes.POINTER(neox_hparams),
                                              ctypes.POINTER(neox_scaler_state), ctypes.POINTER(ctypes.c_void_p),
                                              ctypes.c_int32, ctypes.c_void_p, ctypes.c_float, ctypes.c_void_p,
                                              ctypes.POINTER(neox_step_result)]
        L.neox_shard_step_noalloc.restype = S
        L.neox_multi_create.argtypes = [ctypes.POINTER(neox_tensor_set), ctypes.POINTER(neox_hparams), ctypes.c_int,
                                        ctypes.POINTER(_H)]
        L.neox_multi_create.restype = S
        L.neox_multi_step.argtypes = [_H, ctypes.c_float, ctypes.c_void_p, ctypes.POINTER(neox_step_result)]
        L.neox_multi_step.restype = S
        L.neox_multi_step_async.argtypes = [_H, ctypes.c_float, ctypes.c_void_p, ctypes.c_void_p, ctypes.c_void_p]
        L.neox_multi_step_async.restype = S
        L.neox_multi_rebind_grads.argtypes = [_H, ctypes.POINTER(ctypes.c_void_p)]
        L.neox_multi_rebind_grads.restype = S
        L.neox_multi_set_hparams.argtypes = [_H, ctypes.POINTER(neox_hparams)]
        L.neox_multi_set_hparams.restype = S
        L.neox_multi_get_state.argtypes = [_H, ctypes.POINTER(ctypes.c_float), ctypes.POINTER(ctypes.c_int32),
                                           ctypes.POINTER(ctypes.c_int64)]
        L.neox_multi_get_state.restype = S
        L.neox_multi_set_state.argtypes = [_H, ctypes.c_float, ctypes.c_int32, ctypes.c_int64]
        L.neox_multi_set_state.restype = S
        L.neox_multi_set_profiling.argtypes = [_H, ctypes.c_int32]
        L.neox_multi_set_profiling.restype = S
        L.neox_multi_get_profile.argtypes = [_H, ctypes.POINTER(neox_profile)]
        L.neox_multi_get_profile.restype = S
        L.neox_multi_reset_profile.argtypes = [_H]
        L.neox_multi_reset_profile.restype = S
        L.neox_multi_get_hysteresis.argtypes = [_H, ctypes.POINTER(ctypes.c_int32)]
        L.neox_multi_get_hysteresis.restype = S
        L.neox_multi_set_hysteresis.argtypes = [_H, ctypes.c_int32]
        L.neox_multi_set_hysteresis.restype = S
        L.neox_multi_destroy.argtypes = [_H]
        L.neox_multi_destroy.restype = None
        L.neox_multi_last_error.argtypes = [_H]
        L.neox_multi_last_error.restype = ctypes.c_char_p
        L.neox_noalloc_last_error.argtypes = []
        L.neox_noalloc_last_error.restype = ctypes.c_char_p
        L.neox_ipc_export.argtypes = [ctypes.c_void_p, ctypes.POINTER(neox_ipc_handle), ctypes.POINTER(ctypes.c_uint64)]
        L.neox_ipc_export.restype = S
        L.neox_ipc_open.argtypes = [ctypes.POINTER(neox_ipc_handle), ctypes.POINTER(ctypes.c_void_p)]
        L.neox_ipc_open.restype = S
        L.neox_ipc_close.argtypes = [ctypes.c_void_p]
        L.neox_ipc_close.restype = S
        L.neox_ipc_last_error.argtypes = []
        L.neox_ipc_last_error.restype = ctypes.c_char_p
        _lib = L
    return _lib


class NeoxError(RuntimeError):
    def __init__(self, status: int, message: str):
        super().__init__(f"{lib().neox_status_string(status).decode()} ({status}): {message}")
        self.status = status


# ---- same-named wrappers -------------------------------------------------------

def neox_shard_create(desc: neox_shard_desc, hp: neox_hparams, device: int) -> int:
    h = _H()
    st = lib().neox_shard_create(ctypes.byref(desc), ctypes.byref(hp), device, ctypes.byref(h))
    if st != NEOX_OK:
        raise NeoxError(st, lib().neox_last_error(None).decode())
    return h.value


def neox_shard_step(h: int, grad_ptrs, params_ptr: int, lr: float, stream: int) -> neox_step_result:
    arr = (ctypes.c_void_p * len(grad_ptrs))(*grad_ptrs)
    res = neox_step_result()
    st = lib().neox_shard_step(h, arr, len(grad_ptrs), params_ptr, lr, stream, ctypes.byref(res))
    if st != NEOX_OK:
        raise NeoxError(st, lib().neox_last_error(h).decode())
    return res


def neox_shard_step_async(h: int, grad_ptrs, params_ptr: int, lr: float, stream: int,
                          result_ptr: int | None = None, lr_device_ptr: int | None = None) -> None:
    arr = (ctypes.c_void_p * len(grad_ptrs))(*grad_ptrs)
    st = lib().neox_shard_step_async(h, arr, len(grad_ptrs), params_ptr, lr, lr_device_ptr, stream, result_ptr)
    if st != NEOX_OK:
        raise NeoxError(st, lib().neox_last_error(h).decode())


def neox_shard_grad_stats(h: int, grad_ptrs, params_ptr: int, stream: int, stats_ptr: int) -> None:
    arr = (ctypes.c_void_p * len(grad_ptrs))(*grad_ptrs)
    st = lib().neox_shard_grad_stats(h, arr, len(grad_ptrs), params_ptr, stream, stats_ptr)
    if st != NEOX_OK:
        raise NeoxError(st, lib().neox_last_error(h).decode())


def neox_shard_apply(h: int, grad_ptrs, params_ptr: int, lr: float, stats_ptr: int, stream: int) -> neox_step_result:
    arr = (ctypes.c_void_p * len(grad_ptrs))(*grad_ptrs)
    res = neox_step_result()
    st = lib().neox_shard_apply(h, arr, len(grad_ptrs), params_ptr, lr, stats_ptr, stream, ctypes.byref(res))
    if st != NEOX_OK:
        raise NeoxError(st, lib().neox_last_error(h).decode())
    return res


def neox_shard_set_hparams(h: int, hp: neox_hparams) -> None:
    st = lib().neox_shard_set_hparams(h, ctypes.byref(hp))
    if st != NEOX_OK:
        raise NeoxError(st, lib().neox_last_error(h).decode())


def neox_shard_get_state(h: int):
    s, g, t = ctypes.c_float(), ctypes.c_int32(), ctypes.c_int64()
    st = lib().neox_shard_get_state(h, ctypes.byref(s), ctypes.byref(g), ctypes.byref(t))
    if st != NEOX_OK:
        raise NeoxError(st, "get_state")
    return s.value, g.value, t.value


def neox_shard_set_state(h: int, scale: float, good: int, t: int) -> None:
    st = lib().neox_shard_set_state(h, scale, good, t)
    if st != NEOX_OK:
        raise NeoxError(st, lib().neox_last_error(h).decode())


def neox_shard_get_hysteresis(h: int) -> int:
    c = ctypes.c_int32()
    st = lib().neox_shard_get_hysteresis(h, ctypes.byref(c))
    if st != NEOX_OK:
        raise NeoxError(st, lib().neox_last_error(h).decode())
    return c.value


def neox_shard_set_hysteresis(h: int, count: int) -> None:
    st = lib().neox_shard_set_hysteresis(h, count)
    if st != NEOX_OK:
        raise NeoxError(st, lib().neox_last_error(h).decode())


def neox_shard_destroy(h: int) -> None:
    lib().neox_shard_destroy(h)


def neox_status_string(status: int) -> str:
    return lib().neox_status_string(status).decode()


def neox_last_error(h: int | None) -> str:
    return lib().neox_last_error(h).decode()


def neox_model_state_bytes(numel: int, wdtype: int = NEOX_FP16, gdtype: int = NEOX_FP16) -> int:
    return lib().neox_model_state_bytes(numel, wdtype, gdtype)


def neox_shard_scratch_bytes(h: int) -> int:
    return lib().neox_shard_scratch_bytes(h)


def neox_shard_set_profiling(h: int, enable: bool) -> None:
    lib().neox_shard_set_profiling(h, int(enable))


def neox_shard_get_profile(h: int) -> neox_profile:
    p = neox_profile()
    lib().neox_shard_get_profile(h, ctypes.byref(p))
    return p


def neox_shard_reset_profile(h: int) -> None:
    lib().neox_shard_reset_profile(h)


def neox_shard_step_noalloc(desc: neox_shard_desc, hp: neox_hparams, state: neox_scaler_state, grad_ptrs,
                            params_ptr: int, lr: float, stream: int) -> neox_step_result:
    """The step without a handle or any allocation; `state` is updated in place."""
    arr = (ctypes.c_void_p * len(grad_ptrs))(*grad_ptrs)
    res = neox_step_result()
    st = lib().neox_shard_step_noalloc(ctypes.byref(desc), ctypes.byref(hp), ctypes.byref(state), arr,
                                       len(grad_ptrs), params_ptr, lr, stream, ctypes.byref(res))
    if st != NEOX_OK:
        raise NeoxError(st, lib().neox_noalloc_last_error().decode())
    return res


# ---- multi-tensor shard -----------------------------------------------------------

def _merr(h):
    return lib().neox_multi_last_error(h).decode()


def neox_multi_create(tset: neox_tensor_set, hp: neox_hparams, device: int) -> int:
    h = _H()
    st = lib().neox_multi_create(ctypes.byref(tset), ctypes.byref(hp), device, ctypes.byref(h))
    if st != NEOX_OK:
        raise NeoxError(st, _merr(None))
    return h.value


def neox_multi_step(h: int, lr: float, stream: int) -> neox_step_result:
    res = neox_step_result()
    st = lib().neox_multi_step(h, lr, stream, ctypes.byref(res))
    if st != NEOX_OK:
        raise NeoxError(st, _merr(h))
    return res


def neox_multi_step_async(h: int, lr: float, stream: int, result_ptr=None, lr_device_ptr=None) -> None:
    st = lib().neox_multi_step_async(h, lr, lr_device_ptr, stream, result_ptr)
    if st != NEOX_OK:
        raise NeoxError(st, _merr(h))


def neox_multi_rebind_grads(h: int, grad_ptrs) -> None:
    arr = (ctypes.c_void_p * len(grad_ptrs))(*grad_ptrs)
    st = lib().neox_multi_rebind_grads(h, arr)
    if st != NEOX_OK:
        raise NeoxError(st, _merr(h))


def neox_multi_get_state(h: int):
    s, g, t = ctypes.c_float(), ctypes.c_int32(), ctypes.c_int64()
    st = lib().neox_multi_get_state(h, ctypes.byref(s), ctypes.byref(g), ctypes.byref(t))
    if st != NEOX_OK:
        raise NeoxError(st, _merr(h))
    return s.value, g.value, t.value


def neox_multi_set_state(h: int, scale: float, good: int, t: int) -> None:
    st = lib().neox_multi_set_state(h, scale, good, t)
    if st != NEOX_OK:
        raise NeoxError(st, _merr(h))


def neox_multi_get_hysteresis(h: int) -> int:
    c = ctypes.c_int32()
    st = lib().neox_multi_get_hysteresis(h, ctypes.byref(c))
    if st != NEOX_OK:
        raise NeoxError(st, _merr(h))
    return c.value


def neox_multi_set_hysteresis(h: int, count: int) -> None:
    st = lib().neox_multi_set_hysteresis(h, count)
    if st != NEOX_OK:
        raise NeoxError(st, _merr(h))


def neox_multi_set_hparams(h: int, hp: neox_hparams) -> None:
    st = lib().neox_multi_set_hparams(h, ctypes.byref(hp))
    if st != NEOX_OK:
        raise NeoxError(st, _merr(h))


def neox_multi_set_profiling(h: int, enable: bool) -> None:
    lib().neox_multi_set_profiling(h, int(enable))


def neox_multi_get_profile(h: int) -> neox_profile:
    p = neox_profile()
    lib().neox_multi_get_profile(h, ctypes.byref(p))
    return p


def neox_multi_reset_profile(h: int) -> None:
    lib().neox_multi_reset_profile(h)


def neox_multi_destroy(h: int) -> None:
    lib().neox_multi_destroy(h)


def neox_shard_set_weight_copies(h: int, dst_ptrs) -> None:
    arr = (ctypes.c_void_p * max(1, len(dst_ptrs)))(*dst_ptrs)
    st = lib().neox_shard_set_weight_copies(h, arr, len(dst_ptrs))
    if st != NEOX_OK:
        raise NeoxError(st, lib().neox_last_error(h).decode())


# ---- CUDA IPC (peer buffers for the fused reduce-scatter / all-gather) ---------------

def neox_ipc_export(dev_ptr: int):
    """(64 handle bytes, byte offset of dev_ptr in the exported allocation)."""
    h, off = neox_ipc_handle(), ctypes.c_uint64()
    st = lib().neox_ipc_export(dev_ptr, ctypes.byref(h), ctypes.byref(off))
    if st != NEOX_OK:
        raise NeoxError(st, lib().neox_ipc_last_error().decode())
    return bytes(h.bytes), off.value


def neox_ipc_open(handle: bytes) -> int:
    """Map a peer process's exported allocation; returns its base address."""
    if len(handle) != 64:
        raise ValueError("an IPC handle is 64 bytes")
    h = neox_ipc_handle()
    ctypes.memmove(h.bytes, handle, 64)
    base = ctypes.c_void_p()
    st = lib().neox_ipc_open(ctypes.byref(h), ctypes.byref(base))
    if st != NEOX_OK:
        raise NeoxError(st, lib().neox_ipc_last_error().decode())
    return base.value


def neox_ipc_close(base: int) -> None:
    st = lib().neox_ipc_close(base)
    if st != NEOX_OK:
        raise NeoxError(st, lib().neox_ipc_last_error().decode())
