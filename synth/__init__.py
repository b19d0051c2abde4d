"""Seeded synthetic inputs for the shard step: gradients, master weights, injections.

This module holds none of the optimizer step's arithmetic.  It draws random
numbers with the counter-based Philox4x32-10 generator (Salmon, Moraes, Dror,
Shaw, "Parallel random numbers: as easy as 1, 2, 3", SC'11), turns them into
normal / Student-t samples, scales them and rounds them to the 16-bit storage
type.  The same bytes then feed both the CUDA path and the oracle: on the GPU
the CUDA generator in ``philox_gen.cu`` writes them into device memory and the
tests copy them to the host for the oracle; on a machine without a GPU the
numpy twin below draws the same Philox integers and the same distributions.

Stream layout (shared by both generators):
  key     = (seed, stream)  where stream = STREAM_* | tensor_id << 8
  counter = (block_lo, block_hi, step, 0) with block = element_index // 4 for
            normals (4 normals per Philox block, Box-Muller on lanes (0,1) and
            (2,3)), and block = element_index for Student-t (one block per
            element) and for rate injection.
"""
from __future__ import annotations

import numpy as np

# Philox4x32 constants (SC'11 paper, section 4: multipliers and the Weyl
# sequence used as the key schedule).
PHILOX_M0 = 0xD2511F53
PHILOX_M1 = 0xCD9E8D57
PHILOX_W0 = 0x9E3779B9
PHILOX_W1 = 0xBB67AE85
PHILOX_ROUNDS = 10

STREAM_GRAD = 1
STREAM_MASTER = 2
STREAM_INJECT_INDEX = 3
STREAM_INJECT_RATE = 4

_MASK32 = np.uint64(0xFFFFFFFF)


def philox4x32(c0, c1, c2, c3, k0, k1, rounds: int = PHILOX_ROUNDS):
    """Vectorised Philox4x32-R on numpy uint32 arrays; returns 4 uint32 arrays."""
    c0, c1, c2, c3 = (np.asarray(c, dtype=np.uint64) & _MASK32 for c in (c0, c1, c2, c3))
    k0 = np.asarray(k0, dtype=np.uint64) & _MASK32
    k1 = np.asarray(k1, dtype=np.uint64) & _MASK32
    for r in range(rounds):
        if r:
            k0 = (k0 + np.uint64(PHILOX_W0)) & _MASK32
            k1 = (k1 + np.uint64(PHILOX_W1)) & _MASK32
        p0 = np.uint64(PHILOX_M0) * c0
        p1 = np.uint64(PHILOX_M1) * c2
        hi0, lo0 = p0 >> np.uint64(32), p0 & _MASK32
        hi1, lo1 = p1 >> np.uint64(32), p1 & _MASK32
        c0, c1, c2, c3 = hi1 ^ c1 ^ k0, lo1, hi0 ^ c3 ^ k1, lo0
    return tuple(x.astype(np.uint32) for x in (c0, c1, c2, c3))


def uniform24(x):
    """uint32 -> float32 uniform in (0, 1): top 24 bits, centred in their cell."""
    return ((x >> np.uint32(8)).astype(np.float64) + 0.5) * (2.0 ** -24)


def _box_muller(u0, u1):
    r = np.sqrt(-2.0 * np.log(u0))
    th = 2.0 * np.pi * u1
    return r * np.cos(th), r * np.sin(th)


def normals(n: int, seed: int, stream: int, step: int, start: int = 0) -> np.ndarray:
    """Standard normals for elements start..start+n-1 (float64; CPU twin)."""
    idx = np.arange(start, start + n, dtype=np.uint64)
    blk = idx // np.uint64(4)
    lane = (idx % np.uint64(4)).astype(np.int64)
    x = philox4x32(blk & _MASK32, blk >> np.uint64(32), np.uint64(step), 0, seed, stream)
    u = [uniform24(v) for v in x]
    z01 = _box_muller(u[0], u[1])
    z23 = _box_muller(u[2], u[3])
    z = np.choose(lane, [z01[0], z01[1], z23[0], z23[1]])
    return z


def student_t3(n: int, seed: int, stream: int, step: int, start: int = 0) -> np.ndarray:
    """Student-t with 3 degrees of freedom: z0 / sqrt((z1^2 + z2^2 + z3^2) / 3)."""
    idx = np.arange(start, start + n, dtype=np.uint64)
    x = philox4x32(idx & _MASK32, idx >> np.uint64(32), np.uint64(step), 0, seed, stream)
    u = [uniform24(v) for v in x]
    z0, z1 = _box_muller(u[0], u[1])
    z2, z3 = _box_muller(u[2], u[3])
    return z0 / np.sqrt((z1 * z1 + z2 * z2 + z3 * z3) / 3.0)


def round16(x: np.ndarray, bf16: bool) -> np.ndarray:
    """Round float values to the 16-bit storage type (numpy / torch casts)."""
    x32 = np.asarray(x, dtype=np.float32)
    if not bf16:
        with np.errstate(over="ignore"):
            return x32.astype(np.float16).view(np.uint16)
    import torch
    return torch.from_numpy(np.ascontiguousarray(x32)).to(torch.bfloat16).view(torch.int16).numpy().view(np.uint16)


def grad_normal16(n, sigma, scale, seed, tensor_id, step, bf16=False, start=0):
    """RNE16(z * sigma * scale) computed as fl32(fl32(z * sigma) * scale)."""
    z = normals(n, seed, STREAM_GRAD | (tensor_id << 8), step, start).astype(np.float32)
    return round16((z * np.float32(sigma)) * np.float32(scale), bf16)


def grad_t3_16(n, scale, seed, tensor_id, step, bf16=False, start=0):
    t = student_t3(n, seed, STREAM_GRAD | (tensor_id << 8), step, start).astype(np.float32)
    return round16(t * np.float32(scale), bf16)


def master_normal(n, sigma, seed, tensor_id=0, start=0) -> np.ndarray:
    z = normals(n, seed, STREAM_MASTER | (tensor_id << 8), 0, start).astype(np.float32)
    return z * np.float32(sigma)


INJECT_VALUES = (np.float32(np.inf), np.float32(np.nan), np.float32(-np.inf))


def inject_index(n: int, seed: int, step: int, which: int = 0) -> int:
    """Seeded element index for a scripted injection on `step`."""
    x = philox4x32(which, 0, step, 0, seed, STREAM_INJECT_INDEX)
    v = (int(x[0]) << 32) | int(x[1])
    return v % n


def inject_value(count: int, bf16: bool) -> np.uint16:
    """+inf, NaN, -inf in turn across injections, as a 16-bit code."""
    return round16(np.array([INJECT_VALUES[count % 3]]), bf16)[0]


def rate_inject_mask(n: int, rate: float, seed: int, tensor_id: int, step: int, start: int = 0):
    """Elements hit by a per-element injection at `rate`, and the kind of value
    (0:+inf 1:NaN 2:-inf) for each; CPU twin of the GPU rate injector."""
    idx = np.arange(start, start + n, dtype=np.uint64)
    x = philox4x32(idx & _MASK32, idx >> np.uint64(32), np.uint64(step), 0, seed,
                   STREAM_INJECT_RATE | (tensor_id << 8))
    thresh = np.uint32(min(int(rate * 2.0 ** 32), 0xFFFFFFFF))
    hit = x[0] < thresh
    kind = (x[1] % np.uint32(3)).astype(np.int64)
    return hit, kind


# ---------------------------------------------------------------------------
# GPU generator (synth/philox_gen.cu), for inputs at full size.  Outputs are
# written into caller-provided torch CUDA tensors on torch's current stream.
# ---------------------------------------------------------------------------
import ctypes as _ct
import os as _os
import subprocess as _sp

_HERE = _os.path.dirname(_os.path.abspath(__file__))
_CU = _os.path.join(_HERE, "philox_gen.cu")
_SO = _os.path.join(_HERE, "libsynth.so")
_gpu_lib = None


def build_cuda(force: bool = False) -> str:
    if force or not _os.path.exists(_SO) or _os.path.getmtime(_SO) < _os.path.getmtime(_CU):
        tmp = _SO + f".tmp{_os.getpid()}"
        _sp.check_call(["/usr/local/cuda/bin/nvcc", "-gencode", "arch=compute_100a,code=sm_100a", "-O3",
                        "-lineinfo", "-Xcompiler", "-fPIC", "-shared", "-o", tmp, _CU])
        _os.replace(tmp, _SO)
    return _SO


def _lib():
    global _gpu_lib
    if _gpu_lib is None:
        if not _os.path.exists(_SO):
            build_cuda()
        L = _ct.CDLL(_SO)
        u64, u32, f, i, p = _ct.c_ulonglong, _ct.c_uint32, _ct.c_float, _ct.c_int, _ct.c_void_p
        L.synth_normal16.argtypes = [p, u64, u64, f, f, u32, u32, u32, i, p]
        L.synth_normal32.argtypes = [p, u64, u64, f, u32, u32, u32, p]
        L.synth_t3_16.argtypes = [p, u64, u64, f, u32, u32, u32, i, p]
        L.synth_rate_inject16.argtypes = [p, u64, u64, u32, u32, u32, u32, i, p, p]
        L.synth_philox_raw.argtypes = [p, u64, u32, u32, u32, p]
        _gpu_lib = L
    return _gpu_lib


def _stream():
    import torch
    return torch.cuda.current_stream().cuda_stream


def _check(rc: int, what: str):
    if rc != 0:
        raise RuntimeError(f"{what}: CUDA error {rc}")


def gpu_grad_normal16(out, sigma, scale, seed, tensor_id, step, bf16=False, start=0):
    """out (16-bit CUDA tensor) <- RNE16(fl32(z*sigma)*scale), z the Philox normals."""
    _check(_lib().synth_normal16(out.data_ptr(), out.numel(), start, sigma, scale, seed,
                                 STREAM_GRAD | (tensor_id << 8), step, int(bf16), _stream()), "synth_normal16")


def gpu_grad_t3_16(out, scale, seed, tensor_id, step, bf16=False, start=0):
    _check(_lib().synth_t3_16(out.data_ptr(), out.numel(), start, scale, seed,
                              STREAM_GRAD | (tensor_id << 8), step, int(bf16), _stream()), "synth_t3_16")


def gpu_master_normal(out, sigma, seed, tensor_id=0, start=0):
    _check(_lib().synth_normal32(out.data_ptr(), out.numel(), start, sigma, seed,
                                 STREAM_MASTER | (tensor_id << 8), 0, _stream()), "synth_normal32")


def gpu_rate_inject(out, rate, seed, tensor_id, step, bf16=False, start=0) -> int:
    """Overwrite each element with +inf / NaN / -inf with probability `rate`; returns the hit count."""
    import torch
    hits = torch.zeros(1, dtype=torch.int64, device=out.device)
    thresh = min(int(rate * 2.0 ** 32), 0xFFFFFFFF)
    _check(_lib().synth_rate_inject16(out.data_ptr(), out.numel(), start, thresh, seed,
                                      STREAM_INJECT_RATE | (tensor_id << 8), step, int(bf16),
                                      hits.data_ptr(), _stream()), "synth_rate_inject16")
    return int(hits.item())


def gpu_philox_raw(nblocks: int, step: int, seed: int, stream: int):
    """Raw Philox output of counters (b, step) for b < nblocks, as uint32 numpy [nblocks, 4]."""
    import torch
    out = torch.empty(nblocks * 4, dtype=torch.int32, device="cuda")
    _check(_lib().synth_philox_raw(out.data_ptr(), nblocks, step, seed, stream, _stream()), "synth_philox_raw")
    return out.cpu().numpy().view(np.uint32).reshape(nblocks, 4)
