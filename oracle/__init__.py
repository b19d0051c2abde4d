"""CPU oracle for the per-rank mixed-precision optimizer step (test infrastructure).

Only the test suite, ``__graft_entry__.smoke()`` and the CPU-baseline leg of
``bench.py`` may import this package.  The product path (the CUDA library and
its Python binding) never imports, loads or calls it, and shares no code with it.

The arithmetic lives in ``oracle.c`` (plain C, single-threaded, FP32 state with
every operation rounded on its own, plus a float64 brute force).  This module
only marshals numpy arrays into it through ctypes and keeps the per-shard state
(master, m, v, the 16-bit working copy and the loss-scaler counters) between calls.

Every function in ``oracle.c`` is pinned by ``tests/test_oracle_*.py`` against
values fixed by the pages and by mathematics (closed forms, invariants, library
special cases and exhaustive comparisons), never against the CUDA path.
"""
from __future__ import annotations

import contextlib
import ctypes
import os
import subprocess
import threading
from concurrent.futures import ThreadPoolExecutor
from dataclasses import dataclass, field

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "oracle.c")
_LIB_PATH = os.path.join(_HERE, "liboracle.so")
_CFLAGS = ["-O2", "-std=c99", "-ffp-contract=off", "-fno-fast-math", "-fPIC", "-shared"]

_lock = threading.Lock()
_lib = None


def build(force: bool = False) -> str:
    """Compile ``oracle.c`` into ``liboracle.so`` next to it (gcc, no contraction)."""
    if force or not os.path.exists(_LIB_PATH) or os.path.getmtime(_LIB_PATH) < os.path.getmtime(_SRC):
        tmp = _LIB_PATH + f".tmp{os.getpid()}"
        subprocess.check_call(["gcc", *_CFLAGS, "-o", tmp, _SRC, "-lm"])
        os.replace(tmp, _LIB_PATH)
    return _LIB_PATH


class Hparams(ctypes.Structure):
    _fields_ = [("beta1", ctypes.c_float), ("beta2", ctypes.c_float), ("eps", ctypes.c_float),
                ("clip_norm", ctypes.c_float), ("predivide", ctypes.c_float),
                ("scale_factor", ctypes.c_float), ("min_scale", ctypes.c_float),
                ("scale_window", ctypes.c_int32), ("hysteresis", ctypes.c_int32), ("optimizer", ctypes.c_int32)]


class Scaler(ctypes.Structure):
    _fields_ = [("scale", ctypes.c_float), ("good", ctypes.c_int32), ("t", ctypes.c_int64),
                ("hyst", ctypes.c_int32), ("pad_", ctypes.c_int32)]


class Segment(ctypes.Structure):
    _fields_ = [("offset", ctypes.c_uint64), ("numel", ctypes.c_uint64), ("weight_decay", ctypes.c_float)]


class StepInfo(ctypes.Structure):
    _fields_ = [("overflow", ctypes.c_int32), ("pad_", ctypes.c_int32),
                ("sumsq", ctypes.c_double), ("norm", ctypes.c_double),
                ("coef", ctypes.c_float), ("scale_used", ctypes.c_float),
                ("scale_next", ctypes.c_float), ("step_size", ctypes.c_float),
                ("bc2_sqrt", ctypes.c_float), ("pad2_", ctypes.c_int32),
                ("t", ctypes.c_int64)]

    def as_dict(self) -> dict:
        return {k: getattr(self, k) for k, _ in self._fields_ if not k.startswith("pad")}


_P = ctypes.c_void_p
_U64 = ctypes.c_uint64


def lib():
    global _lib
    with _lock:
        if _lib is None:
            build()
            _lib = _configure(ctypes.CDLL(_LIB_PATH))
    return _lib


@contextlib.contextmanager
def use_library(path: str):
    """Temporarily route every call of this module to another build of the
    oracle (the mutation tests load deliberately broken copies this way)."""
    global _lib
    with _lock:
        saved = _lib
        _lib = _configure(ctypes.CDLL(path))
    try:
        yield _lib
    finally:
        with _lock:
            _lib = saved


def _configure(L):
    """Declare the C signatures on a loaded oracle library."""
    for nm in ("orc_f16_encode_array", "orc_bf16_encode_array",
               "orc_f16_decode_array", "orc_bf16_decode_array"):
        getattr(L, nm).argtypes = [_P, _P, _U64]
        getattr(L, nm).restype = None
    L.orc_ingest_factors.argtypes = [ctypes.c_int32, ctypes.c_float, ctypes.c_float,
                                     ctypes.POINTER(ctypes.c_float), ctypes.POINTER(ctypes.c_float)]
    L.orc_grad_stats.argtypes = [_P, ctypes.c_int32, ctypes.c_int32, _U64, ctypes.c_float,
                                 ctypes.c_float, ctypes.POINTER(ctypes.c_int64),
                                 ctypes.POINTER(ctypes.c_double)]
    L.orc_unscaled_grads.argtypes = [_P, ctypes.c_int32, ctypes.c_int32, _U64, ctypes.c_float,
                                     ctypes.c_float, _P]
    L.orc_scaler_update.argtypes = [ctypes.POINTER(Hparams), ctypes.POINTER(Scaler), ctypes.c_int32]
    L.orc_clip_coef.argtypes = [ctypes.c_float, ctypes.c_double]
    L.orc_clip_coef.restype = ctypes.c_float
    L.orc_adam_apply.argtypes = [_U64, _P, _U64, _P, ctypes.c_int32, ctypes.c_int32,
                                 _P, ctypes.c_int32, _P, _P, _P, _P, ctypes.c_int32,
                                 ctypes.POINTER(Hparams), ctypes.c_float, ctypes.POINTER(StepInfo)]
    L.orc_sgd_apply.argtypes = [_U64, _P, _U64, _P, ctypes.c_int32, ctypes.c_int32, _P, ctypes.c_int32,
                                _P, _P, ctypes.c_int32, ctypes.POINTER(Hparams), ctypes.c_float,
                                ctypes.POINTER(StepInfo)]
    L.orc_step_decide.argtypes = [ctypes.POINTER(Hparams), ctypes.POINTER(Scaler), ctypes.c_float,
                                  ctypes.c_int64, ctypes.c_double, ctypes.POINTER(StepInfo)]
    L.orc_step.argtypes = [_U64, _P, ctypes.c_int32, ctypes.c_int32, _P, ctypes.c_int32,
                           _P, _P, _P, _P, ctypes.c_int32, ctypes.POINTER(Hparams),
                           ctypes.POINTER(Scaler), ctypes.c_float, ctypes.POINTER(StepInfo)]
    L.orc_step.restype = ctypes.c_int32
    L.orc64_step.argtypes = [_U64, _P, ctypes.c_int32, ctypes.c_int32, _P, ctypes.c_int32,
                             _P, _P, _P, ctypes.POINTER(Hparams), ctypes.POINTER(Scaler),
                             ctypes.c_float, ctypes.POINTER(ctypes.c_double)]
    L.orc64_step.restype = ctypes.c_int32
    return L


def _ptr(a: np.ndarray) -> int:
    assert a.flags["C_CONTIGUOUS"]
    return a.ctypes.data


def _grad_ptrs(grads):
    arr = (ctypes.c_void_p * len(grads))(*[_ptr(g) for g in grads])
    return arr


# ---- 16-bit codecs ---------------------------------------------------------

def f16_encode(x: np.ndarray) -> np.ndarray:
    x = np.ascontiguousarray(x, dtype=np.float32)
    out = np.empty(x.shape, np.uint16)
    lib().orc_f16_encode_array(_ptr(x), _ptr(out), x.size)
    return out


def bf16_encode(x: np.ndarray) -> np.ndarray:
    x = np.ascontiguousarray(x, dtype=np.float32)
    out = np.empty(x.shape, np.uint16)
    lib().orc_bf16_encode_array(_ptr(x), _ptr(out), x.size)
    return out


def f16_decode(h: np.ndarray) -> np.ndarray:
    h = np.ascontiguousarray(h, dtype=np.uint16)
    out = np.empty(h.shape, np.float32)
    lib().orc_f16_decode_array(_ptr(h), _ptr(out), h.size)
    return out


def bf16_decode(h: np.ndarray) -> np.ndarray:
    h = np.ascontiguousarray(h, dtype=np.uint16)
    out = np.empty(h.shape, np.float32)
    lib().orc_bf16_decode_array(_ptr(h), _ptr(out), h.size)
    return out


def encode16(x, bf16: bool):
    return bf16_encode(x) if bf16 else f16_encode(x)


def decode16(h, bf16: bool):
    return bf16_decode(h) if bf16 else f16_decode(h)


# ---- scalar pieces -----------------------------------------------------------

def ingest_factors(K: int, predivide: float, scale: float):
    a, b = ctypes.c_float(), ctypes.c_float()
    lib().orc_ingest_factors(K, predivide, scale, ctypes.byref(a), ctypes.byref(b))
    return a.value, b.value


def clip_coef(clip: float, norm: float) -> float:
    return lib().orc_clip_coef(clip, norm)


@dataclass
class OracleHparams:
    beta1: float = 0.9
    beta2: float = 0.95
    eps: float = 1e-8
    clip_norm: float = 1.0
    predivide: float = 1.0
    init_scale: float = 65536.0
    scale_factor: float = 2.0
    min_scale: float = 1.0
    scale_window: int = 1000
    hysteresis: int = 1
    optimizer: int = 0          # 0 AdamW, 1 SGD

    def c(self) -> Hparams:
        return Hparams(self.beta1, self.beta2, self.eps, self.clip_norm, self.predivide,
                       self.scale_factor, self.min_scale, self.scale_window, self.hysteresis, self.optimizer)

    @property
    def hyst0(self) -> int:
        return max(1, self.hysteresis)


def segments_array(segments, n: int, default_wd: float):
    """Segment table as a ctypes array; None means one segment [0, n)."""
    if segments is None:
        segments = [(0, n, default_wd)]
    arr = (Segment * len(segments))(*[Segment(int(o), int(c), float(w)) for o, c, w in segments])
    return arr


def scaler_update(hp: OracleHparams, scale: float, good: int, t: int, overflow: bool, hyst: int | None = None,
                  with_hyst: bool = False):
    """One scaler update; `hyst` is the hysteresis count (None: a full one,
    which is exact whenever hysteresis <= 1)."""
    sc = Scaler(scale, good, t, hp.hyst0 if hyst is None else hyst, 0)
    lib().orc_scaler_update(ctypes.byref(hp.c()), ctypes.byref(sc), int(overflow))
    if with_hyst:
        return sc.scale, sc.good, sc.t, sc.hyst
    return sc.scale, sc.good, sc.t


def grad_stats(grads, gbf16: bool, inv_pre: float, inv_us: float, threads: int = 1,
               chunk: int = 1 << 24):
    """Pass 1 over equal-length 16-bit buffers: (non-finite count, sum of squares).

    With threads > 1 the index range is cut into contiguous chunks, each summed
    by the single-threaded C routine, and the chunk sums are added in index
    order (so the double sum is re-associated at chunk boundaries only).
    """
    n = grads[0].size
    L = lib()

    def run(lo, hi):
        sub = [g[lo:hi] for g in grads]
        ptrs = _grad_ptrs(sub)
        bad, s = ctypes.c_int64(), ctypes.c_double()
        L.orc_grad_stats(ptrs, len(grads), int(gbf16), hi - lo, inv_pre, inv_us,
                         ctypes.byref(bad), ctypes.byref(s))
        return bad.value, s.value

    if threads <= 1 or n <= chunk:
        return run(0, n)
    bounds = [(lo, min(n, lo + chunk)) for lo in range(0, n, chunk)]
    with ThreadPoolExecutor(threads) as ex:
        parts = list(ex.map(lambda b: run(*b), bounds))
    return sum(p[0] for p in parts), float(sum(p[1] for p in parts))


def unscaled_grads(grads, gbf16: bool, inv_pre: float, inv_us: float) -> np.ndarray:
    grads = [np.ascontiguousarray(g, dtype=np.uint16) for g in grads]
    out = np.empty(grads[0].size, np.float32)
    lib().orc_unscaled_grads(_grad_ptrs(grads), len(grads), int(gbf16), out.size, inv_pre, inv_us,
                             _ptr(out))
    return out


def step_decide(hp: OracleHparams, scaler: Scaler, lr: float, nonfinite: int, sumsq: float) -> StepInfo:
    info = StepInfo()
    lib().orc_step_decide(ctypes.byref(hp.c()), ctypes.byref(scaler), lr, nonfinite, sumsq,
                          ctypes.byref(info))
    return info


def adam_apply(index, first: int, grads, gbf16: bool, segs, master, m, v, w, wbf16: bool,
               hp: OracleHparams, lr: float, info: StepInfo):
    """AdamW update of the elements whose gradients are `grads` (one array per
    buffer, aligned with the state arrays); `index` holds their global indices
    (uint64) or is None for first..first+n."""
    n = master.size
    idx_ptr = None if index is None else _ptr(np.ascontiguousarray(index, dtype=np.uint64))
    lib().orc_adam_apply(n, idx_ptr, first, _grad_ptrs(grads), len(grads), int(gbf16),
                         segs, len(segs), _ptr(master), _ptr(m), _ptr(v), _ptr(w), int(wbf16),
                         ctypes.byref(hp.c()), lr, ctypes.byref(info))


def sgd_apply(index, first: int, grads, gbf16: bool, segs, master, w, wbf16: bool, hp: OracleHparams, lr: float,
              info: StepInfo):
    """SGD update of the elements whose gradients are `grads` (see adam_apply)."""
    n = master.size
    idx_ptr = None if index is None else _ptr(np.ascontiguousarray(index, dtype=np.uint64))
    lib().orc_sgd_apply(n, idx_ptr, first, _grad_ptrs(grads), len(grads), int(gbf16), segs, len(segs), _ptr(master),
                        _ptr(w), int(wbf16), ctypes.byref(hp.c()), lr, ctypes.byref(info))


@dataclass
class OracleShard:
    """A whole shard held in host memory, stepped by the single-threaded oracle."""
    master: np.ndarray
    hp: OracleHparams = field(default_factory=OracleHparams)
    wbf16: bool = False
    gbf16: bool = False
    segments: list | None = None
    default_wd: float = 0.1

    def __post_init__(self):
        self.master = np.ascontiguousarray(self.master, dtype=np.float32).copy()
        n = self.master.size
        self.m = np.zeros(n, np.float32)
        self.v = np.zeros(n, np.float32)
        self.w = encode16(self.master, self.wbf16)
        self.segs = segments_array(self.segments, n, self.default_wd)
        self.scaler = Scaler(self.hp.init_scale, 0, 0, self.hp.hyst0, 0)

    @property
    def scale(self) -> float:
        return self.scaler.scale

    def step(self, grads, lr: float) -> StepInfo:
        grads = [np.ascontiguousarray(g, dtype=np.uint16) for g in grads]
        assert all(g.size == self.master.size for g in grads)
        info = StepInfo()
        lib().orc_step(self.master.size, _grad_ptrs(grads), len(grads), int(self.gbf16),
                       self.segs, len(self.segs), _ptr(self.master), _ptr(self.m), _ptr(self.v),
                       _ptr(self.w), int(self.wbf16), ctypes.byref(self.hp.c()),
                       ctypes.byref(self.scaler), lr, ctypes.byref(info))
        return info

    def step_threaded(self, grads, lr: float, threads: int, chunk: int = 1 << 22) -> StepInfo:
        """The same step with the index range cut into contiguous chunks, run
        on `threads` host threads: pass 1 chunk by chunk (the chunk sums added
        in index order), the decision, then the update chunk by chunk.  Every
        element's state is that of step(); only the double sum of squares is
        re-associated at the chunk boundaries.  (For timing the oracle on all
        host cores.)"""
        grads = [np.ascontiguousarray(g, dtype=np.uint16) for g in grads]
        n = self.master.size
        assert all(g.size == n for g in grads)
        inv_pre, inv_us = ingest_factors(len(grads), self.hp.predivide, self.scaler.scale)
        bad, ssum = grad_stats(grads, self.gbf16, inv_pre, inv_us, threads=threads, chunk=chunk)
        info = step_decide(self.hp, self.scaler, lr, bad, ssum)
        if info.overflow or n == 0:
            return info

        def run(lo):
            hi = min(n, lo + chunk)
            sub = [g[lo:hi] for g in grads]
            if self.hp.optimizer == 1:
                sgd_apply(None, lo, sub, self.gbf16, self.segs, self.master[lo:hi], self.w[lo:hi], self.wbf16,
                          self.hp, lr, info)
            else:
                adam_apply(None, lo, sub, self.gbf16, self.segs, self.master[lo:hi], self.m[lo:hi], self.v[lo:hi],
                           self.w[lo:hi], self.wbf16, self.hp, lr, info)

        with ThreadPoolExecutor(max(1, threads)) as ex:
            list(ex.map(run, range(0, n, chunk)))
        return info


@dataclass
class Oracle64Shard:
    """float64 brute force of the same step (tiny shards only)."""
    master: np.ndarray
    hp: OracleHparams = field(default_factory=OracleHparams)
    gbf16: bool = False
    segments: list | None = None
    default_wd: float = 0.1

    def __post_init__(self):
        self.master = np.ascontiguousarray(self.master, dtype=np.float64).copy()
        n = self.master.size
        self.m = np.zeros(n, np.float64)
        self.v = np.zeros(n, np.float64)
        self.segs = segments_array(self.segments, n, self.default_wd)
        self.scaler = Scaler(self.hp.init_scale, 0, 0, self.hp.hyst0, 0)

    def step(self, grads, lr: float):
        grads = [np.ascontiguousarray(g, dtype=np.uint16) for g in grads]
        norm = ctypes.c_double()
        ov = lib().orc64_step(self.master.size, _grad_ptrs(grads), len(grads), int(self.gbf16),
                              self.segs, len(self.segs), _ptr(self.master), _ptr(self.m),
                              _ptr(self.v), ctypes.byref(self.hp.c()), ctypes.byref(self.scaler),
                              lr, ctypes.byref(norm))
        return bool(ov), norm.value
