#!/usr/bin/env python
"""Benchmark of the per-rank mixed-precision Adam shard step on B200.

    python bench.py [--gpus N --steps K --warmup W] [--workload opt_5b]
    python bench.py --impl reference ...      # the CPU oracle as the reference arm

One step = one neox_shard_step call over the whole owned shard: pass 1 (ingest,
overflow flag, global norm, loss scaler, clip coefficient) and pass 2 (AdamW on
FP32 master/m/v + cast to the 16-bit working copy).  The default workload is the
largest single-GPU one, the OPT-style 5e9-parameter BF16 shard; the others
(``--workload pythia_1p4b``, ``neox20b_slice``, ``accum8``, ``tiny``) run the
same way.  Inputs are resident in HBM (80 GB for the default shard, far above
the 126 MB L2, so no flush is needed between steps).  Under torchrun every rank steps its own shard of
the same size (weak scaling) with the split step: pass 1, a 16-byte NCCL
all-reduce of {sum of squares, non-finite flag}, then the shared decision and
pass 2, as data-parallel ranks with one global norm and loss scale do.

Prints one JSON line (rank 0).
"""
from __future__ import annotations

import argparse
import ctypes
import hashlib
import json
import os
import re
import statistics
import sys
import threading
import time

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

METRIC = "Adam shard-step Gparams/s and achieved HBM GB/s (% of B200 peak), 1 GPU"
# the same measurement with the plain-SGD update (a side line, not the headline)
METRIC_SGD = "SGD shard-step Gparams/s and achieved HBM GB/s (% of B200 peak), 1 GPU"
UNIT = "Gparams/s"
FALLBACK_HBM_GBS = 6650.0
KERNEL_SRCS = [os.path.join(ROOT, "mixed_precision_zero_b200", "csrc", f) for f in ("neox_shard.cu", "neox_common.cuh")]


def log(*a):
    print(*a, file=sys.stderr, flush=True)


def parse_args(argv=None):
    p = argparse.ArgumentParser()
    p.add_argument("--gpus", type=int, default=1)
    p.add_argument("--steps", type=int, default=100)
    p.add_argument("--warmup", type=int, default=5)
    p.add_argument("--impl", choices=["b200", "reference"], default="b200")
    p.add_argument("--workload", default=None,
                   help="default: opt_5b (the largest single-GPU shard); pythia_1p4b with --zero2")
    p.add_argument("--e2e-steps", type=int, default=5)
    p.add_argument("--split", action="store_true",
                   help="run the split step (statistics, all-reduce, apply) even on one rank")
    p.add_argument("--api", choices=["flat", "multi"], default="flat",
                   help="flat: neox_shard_step; multi: neox_multi_step with one tensor per segment")
    p.add_argument("--cpu-seconds", type=float, default=12.0, help="budget of the oracle CPU baseline")
    p.add_argument("--no-cpu-baseline", action="store_true")
    p.add_argument("--optimizer", choices=["adamw", "sgd"], default="adamw",
                   help="update rule of pass 2 (sgd: plain SGD, m and v untouched)")
    p.add_argument("--zero2", action="store_true",
                   help="ZeRO-2 over peer memory: every rank owns 1/N of the model, pass 1 reads every rank's "
                        "gradient slice, pass 2 stores the cast into every rank's weight buffer")
    a = p.parse_args(argv)
    if a.warmup < 3:
        p.error("--warmup must be >= 3")
    if a.workload is None:
        a.workload = "pythia_1p4b" if a.zero2 else "opt_5b"
    return a


# ------------------------------------------------------------------ workload bytes

def alg_bytes_per_param(K: int, acc: bool, sgd: bool = False):
    """Algorithmic HBM bytes per parameter of an applied step: (pass 1, pass 2).
    Pass 2 reads the gradient (K 16-bit buffers, or the FP32 sum) and the FP32
    state, and writes the state and the 16-bit weight: master/m/v for AdamW,
    master alone for SGD."""
    p1 = 2 * K + (4 if acc else 0)
    state = 4 if sgd else 12
    p2 = (4 if acc else 2 * K) + state + state + 2
    return p1, p2


def hbm_peak():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    try:
        with open(path) as f:
            return float(json.load(f)["hbm_gbs"]), "measured"
    except Exception:
        return FALLBACK_HBM_GBS, "fallback"


def kernel_source_hash() -> str:
    """Hash of the code of the flat-shard kernels (the ones bench.py times):
    the sources with comments, trailing blanks and empty lines removed, so
    that editing a comment does not disown the recorded counters."""
    h = hashlib.sha256()
    for path in KERNEL_SRCS:
        with open(path, encoding="utf-8") as f:
            text = f.read()
        text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
        lines = (re.sub(r"//.*$", "", ln).rstrip() for ln in text.splitlines())
        h.update("\n".join(ln for ln in lines if ln).encode())
    return h.hexdigest()[:16]


def recorded_traffic(workload: str, kernel: str = "adam_kernel"):
    """DRAM bytes per launch of the update kernel from the committed ncu summary,
    if it was taken on the current kernel source; else None."""
    path = os.path.join(ROOT, "profiles", f"{kernel}_{workload}.md")
    if not os.path.exists(path):
        return None
    text = open(path).read()
    m_src = re.search(r"kernel_source_sha256_16:\s*([0-9a-f]+)", text)
    m_tr = re.search(r"dram_bytes_per_launch_full_size:\s*([0-9.eE+]+)", text)
    if not (m_src and m_tr) or m_src.group(1) != kernel_source_hash():
        return None
    return float(m_tr.group(1))


# ------------------------------------------------------------------ clocks (NVML)

class ClockSampler:
    REASONS = {0x4: "sw_power_cap", 0x8: "hw_slowdown", 0x20: "sw_thermal_slowdown",
               0x40: "hw_thermal_slowdown", 0x80: "hw_power_brake_slowdown", 0x2: "applications_clocks_setting",
               0x1: "gpu_idle", 0x10: "sync_boost"}

    def __init__(self, device_index: int, interval=0.05):
        self.samples, self.reasons, self.max_mhz = [], set(), None
        self.interval = interval
        self._stop = threading.Event()
        self._thr = None
        try:
            import pynvml
            import torch
            pynvml.nvmlInit()
            uuid = str(torch.cuda.get_device_properties(device_index).uuid)
            self.h = None
            for i in range(pynvml.nvmlDeviceGetCount()):
                h = pynvml.nvmlDeviceGetHandleByIndex(i)
                u = pynvml.nvmlDeviceGetUUID(h)
                u = u.decode() if isinstance(u, bytes) else u
                if u.replace("GPU-", "") == uuid.replace("GPU-", ""):
                    self.h = h
            if self.h is not None:
                self.max_mhz = pynvml.nvmlDeviceGetMaxClockInfo(self.h, pynvml.NVML_CLOCK_SM)
            self.nv = pynvml
        except Exception as e:  # clocks are reported as unavailable, the run goes on
            log(f"clock sampling unavailable: {e}")
            self.h = None

    def _run(self):
        nv = self.nv
        while not self._stop.is_set():
            try:
                self.samples.append(nv.nvmlDeviceGetClockInfo(self.h, nv.NVML_CLOCK_SM))
                r = nv.nvmlDeviceGetCurrentClocksEventReasons(self.h)
                for bit, name in self.REASONS.items():
                    if r & bit and bit != 0x1:
                        self.reasons.add(name)
            except Exception:
                pass
            time.sleep(self.interval)

    def __enter__(self):
        if self.h is not None:
            self._thr = threading.Thread(target=self._run, daemon=True)
            self._thr.start()
        return self

    def __exit__(self, *exc):
        self._stop.set()
        if self._thr:
            self._thr.join()

    def summary(self):
        if not self.samples:
            return {"sm_mhz": None, "sm_max_mhz": self.max_mhz, "reasons": ["unavailable"], "samples": 0}
        return {"sm_mhz": statistics.median(self.samples), "sm_max_mhz": self.max_mhz,
                "reasons": sorted(self.reasons), "samples": len(self.samples)}


# ------------------------------------------------------------------ distributed plumbing

def dist_env():
    ws = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    return ws, rank, local


def max_over_ranks(x: float, device=None) -> float:
    import torch
    import torch.distributed as dist
    if not (dist.is_available() and dist.is_initialized()) or dist.get_world_size() == 1:
        return x
    t = torch.tensor([x], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def sum_over_ranks(x: float, device=None) -> float:
    import torch
    import torch.distributed as dist
    if not (dist.is_available() and dist.is_initialized()) or dist.get_world_size() == 1:
        return x
    t = torch.tensor([x], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.SUM)
    return float(t.item())


# ------------------------------------------------------------------ oracle on the host cores

def cpu_sample_range(wl, size):
    """A contiguous sample of the workload that crosses segment boundaries when
    it has any: centred on the first non-trivial segment boundary."""
    if wl.segments and len(wl.segments) > 1:
        b = wl.segments[1][0]
        lo = max(0, min(b - size // 2, wl.numel - size))
    else:
        lo = 0
    return lo, min(size, wl.numel - lo)


def sample_segments(wl, lo, n):
    if not wl.segments:
        return None, [("normal", 0, n)]
    segs, inits = [], []
    for off, cnt, wd, init in wl.segments:
        a, b = max(off, lo), min(off + cnt, lo + n)
        if a < b:
            segs.append((a - lo, b - a, wd))
            inits.append((init, a - lo, b - a))
    return segs, inits


def host_cores() -> int:
    return max(1, len(os.sched_getaffinity(0)))


def parallel_gen(fn, n, threads, chunk=1 << 22, **kw):
    """A numpy-twin input array of n elements drawn in contiguous chunks on
    `threads` host threads (the generators take the first element's index)."""
    from concurrent.futures import ThreadPoolExecutor

    import numpy as np
    starts = list(range(0, n, chunk))
    lo0 = kw.pop("start", 0)
    with ThreadPoolExecutor(threads) as ex:
        parts = list(ex.map(lambda a: fn(min(chunk, n - a), start=lo0 + a, **kw), starts))
    return np.concatenate(parts) if parts else np.zeros(0)


def sample_inputs_host(wl, n_sample, threads, rank_seed=0):
    """A contiguous sample of the workload drawn by the numpy twin of the
    generator: (lo, master, grads)."""
    import synth
    lo, n = cpu_sample_range(wl, n_sample)
    master = parallel_gen(synth.master_normal, n, threads, sigma=wl.master_sigma, seed=wl.seed + rank_seed,
                          tensor_id=0, start=lo)
    scale = wl.bench_scale or wl.init_scale
    grads = []
    for k in range(wl.K):
        if wl.grad_dist == "t3":
            grads.append(parallel_gen(synth.grad_t3_16, n, threads, scale=scale, seed=wl.seed + rank_seed,
                                      tensor_id=k, step=1, bf16=wl.bf16, start=lo))
        else:
            grads.append(parallel_gen(synth.grad_normal16, n, threads, sigma=wl.grad_sigma, scale=scale,
                                      seed=wl.seed + rank_seed, tensor_id=k, step=1, bf16=wl.bf16, start=lo))
    return lo, master, grads


def oracle_sample_size(wl) -> int:
    """Elements of the threaded oracle baseline: the whole workload when its
    host copy (FP32 master/m/v, 16-bit weights and K gradient buffers) takes
    less than half the host's available memory, else a 2^27-element slice."""
    need = wl.numel * (18 + 2 * wl.K)   # the input master, the oracle's master/m/v/w, the gradients
    try:
        import psutil
        avail = psutil.virtual_memory().available
    except Exception:
        avail = 0
    return wl.numel if need < avail // 2 else min(wl.numel, 1 << 27)


def sample_inputs_device(wl, n_sample, master_dev, grads_dev):
    """The same kind of sample copied from the workload resident on the GPU
    (its bytes come from the CUDA twin of the generator): (lo, master, grads)."""
    import numpy as np
    import torch
    lo, n = cpu_sample_range(wl, n_sample)
    master = master_dev[lo:lo + n].cpu().numpy()
    grads = [g[lo:lo + n].view(torch.int16).cpu().numpy().view(np.uint16) for g in grads_dev]
    return lo, master, grads


def run_oracle_sample(wl, inputs, steps, seconds, threads=1, optimizer="adamw"):
    """Time the oracle on up to `steps` calls (stopping once `seconds` have
    passed) over a contiguous sample of the workload, single-threaded or split
    over `threads` host threads by contiguous ranges.  The inputs are drawn
    before, untimed."""
    import numpy as np

    import oracle
    lo, master, grads = inputs
    n = master.size
    segs, inits = sample_segments(wl, lo, n)
    master = np.asarray(master, dtype=np.float32)   # the caller's sample: initialised in place
    for init, a, c in inits:
        if init == "zero":
            master[a:a + c] = 0
        elif init == "one":
            master[a:a + c] = 1
    hp = oracle.OracleHparams(wl.beta1, wl.beta2, wl.eps, wl.clip, wl.predivide, wl.bench_scale or wl.init_scale,
                              2.0, 1.0, wl.scale_window, optimizer=1 if optimizer == "sgd" else 0)
    sh = oracle.OracleShard(master, hp, wbf16=wl.bf16, gbf16=wl.bf16, segments=segs, default_wd=wl.weight_decay)
    chunk = max(1 << 16, -(-n // (4 * threads)))   # a few contiguous ranges per thread
    times = []
    t_all = time.perf_counter()
    for _ in range(steps):
        t0 = time.perf_counter()
        if threads > 1:
            sh.step_threaded(grads, wl.lr, threads, chunk=chunk)
        else:
            sh.step(grads, wl.lr)
        times.append(time.perf_counter() - t0)
        if seconds and time.perf_counter() - t_all > seconds:
            break
    return {"n": n, "lo": lo, "times": times, "threads": threads}


# ------------------------------------------------------------------ reference arm

def run_reference(args):
    from synth import workloads as W
    ws, rank, _ = dist_env()
    if rank != 0:
        return 0
    wl = W.ALL[args.workload]()
    total = args.steps + args.warmup
    cores = host_cores()
    per_step_budget = max(0.2, 120.0 / total)           # whole run within a few minutes
    # about 40 ns per element and thread for the AdamW step
    n_sample = int(min(1 << 27, wl.numel, max(1 << 16, per_step_budget * cores / 40e-9)))
    inputs = sample_inputs_host(wl, n_sample, cores)
    out = run_oracle_sample(wl, inputs, total, 0.0, threads=cores, optimizer=args.optimizer)
    times = out["times"][args.warmup:]
    sec = sum(times)
    value = out["n"] * len(times) / sec / 1e9
    line = {
        "impl": "reference", "metric": METRIC_SGD if args.optimizer == "sgd" else METRIC, "value": value, "unit": UNIT, "n_gpus": args.gpus,
        "steps": len(times), "warmup": args.warmup, "ms_per_step": 1e3 * sec / len(times),
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f32", "data": "synthetic",
        "config": {"workload": wl.name, "numel": wl.numel, "grad_buffers": wl.K, "optimizer": args.optimizer,
                   "sample": f"{out['n']} contiguous elements from index {out['lo']} per step"},
        "cpu_baseline": {"value": value, "unit": UNIT, "cores": cores, "kind": "oracle",
                         "sample": f"{out['n']} contiguous elements of {wl.name}, {len(times)} timed steps, "
                                   f"split over {cores} host threads by contiguous ranges"},
        "e2e": {"value": value, "unit": UNIT, "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
    }
    print(json.dumps(line), flush=True)
    return 0


# ------------------------------------------------------------------ B200 arm

def _at_offset(n, dtype, offset):
    """A CUDA tensor of n elements starting `offset` elements past an
    allocation boundary (the workload's misalignment)."""
    import torch
    base = torch.empty(n + offset, dtype=dtype, device="cuda")
    return base.narrow(0, offset, n)


def build_gpu_workload(wl, rank, optimizer="adamw"):
    import torch

    import synth
    from mixed_precision_zero_b200 import Hparams, NeoxShard
    n = wl.numel
    dt = torch.bfloat16 if wl.bf16 else torch.float16
    seed = wl.seed + 1000 * rank
    off = wl.elem_offset
    scale = wl.bench_scale or wl.init_scale
    master = _at_offset(n, torch.float32, off)
    synth.gpu_master_normal(master, wl.master_sigma, seed)
    for s_off, cnt, _, init in (wl.segments or []):
        if init == "zero":
            master[s_off:s_off + cnt].zero_()
        elif init == "one":
            master[s_off:s_off + cnt].fill_(1.0)
    m = _at_offset(n, torch.float32, off).zero_()
    v = _at_offset(n, torch.float32, off).zero_()
    params = _at_offset(n, dt, off)
    params.copy_(master.to(dt))
    grads = []
    for k in range(wl.K):
        g = _at_offset(n, dt, off)
        if wl.grad_dist == "t3":
            synth.gpu_grad_t3_16(g, scale, seed, k, 1, wl.bf16)
        else:
            synth.gpu_grad_normal16(g, wl.grad_sigma, scale, seed, k, 1, wl.bf16)
        grads.append(g)
    hp = Hparams(wl.beta1, wl.beta2, wl.eps, wl.clip, wl.predivide, scale, 2.0, 1.0, wl.scale_window,
                 optimizer=optimizer)
    shard = NeoxShard(master, m, v, hp, wdtype=dt, gdtype=dt, segments=wl.seg_table(),
                      weight_decay=wl.weight_decay, max_grads=wl.K)
    torch.cuda.synchronize()
    return shard, grads, params, (master, m, v)


def run_multi(args):
    """The multi-tensor step on the same workload: one tensor per segment, as
    views of the same device buffers, timed like the flat step."""
    import torch

    from mixed_precision_zero_b200 import Hparams, NeoxMultiShard
    from synth import workloads as W
    torch.cuda.set_device(0)
    wl = W.ALL[args.workload]()
    shard, grads, params, (master, m, v) = build_gpu_workload(wl, 0)
    shard.close()
    segs = wl.seg_table() or [(0, wl.numel, wl.weight_decay)]
    scale = wl.bench_scale or wl.init_scale
    hp = Hparams(wl.beta1, wl.beta2, wl.eps, wl.clip, wl.predivide, scale, 2.0, 1.0, wl.scale_window,
                 optimizer=args.optimizer)
    multi = NeoxMultiShard([{"master": master[o:o + c], "exp_avg": m[o:o + c], "exp_avg_sq": v[o:o + c],
                             "params": params[o:o + c], "grads": [g[o:o + c] for g in grads], "weight_decay": w}
                            for o, c, w in segs], hp)
    for _ in range(args.warmup):
        multi.step(wl.lr)
    t0 = multi.get_state()[2]
    multi.reset_profile()
    multi.set_profiling(True)
    launches0 = multi.profile().launches
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    torch.cuda.synchronize()
    with ClockSampler(0) as clocks:
        e0.record()
        for _ in range(args.steps):
            multi.step(wl.lr)
        e1.record()
        torch.cuda.synchronize()
    assert multi.get_state()[2] - t0 == args.steps
    ms = e0.elapsed_time(e1)
    prof = multi.profile()
    multi.set_profiling(False)
    p1b, p2b = alg_bytes_per_param(wl.K, False, args.optimizer == "sgd")
    peak, kind = hbm_peak()
    p2_ms = prof.update_pass_ms / prof.steps
    kernel2 = "mt_sgd_kernel" if args.optimizer == "sgd" else "mt_adam_chunked_kernel"
    line = {"metric": METRIC_SGD if args.optimizer == "sgd" else METRIC, "value": wl.numel * args.steps / (ms * 1e-3) / 1e9, "unit": UNIT, "n_gpus": 1,
            "steps": args.steps, "warmup": args.warmup, "ms_per_step": ms / args.steps, "higher_is_better": True,
            "scaling": "weak", "vs_baseline": None, "dtype": "f32", "data": "synthetic", "impl": "b200",
            "config": {"workload": wl.name, "api": "neox_multi_step", "tensors": len(segs),
                       "optimizer": args.optimizer},
            "hbm": {"step_gbs": (p1b + p2b) * wl.numel / (ms / args.steps * 1e-3) / 1e9,
                    "step_frac": (p1b + p2b) * wl.numel / (ms / args.steps * 1e-3) / 1e9 / peak, "peak_gbs": peak,
                    "peak_kind": kind},
            "roofline": {"bound": "hbm", "kernel": f"{kernel2} (pass 2)",
                         "achieved": p2b * wl.numel / (p2_ms * 1e-3) / 1e9, "peak": peak, "unit": "GB/s",
                         "frac": p2b * wl.numel / (p2_ms * 1e-3) / 1e9 / peak, "peak_kind": kind, "traffic": None,
                         "alg_bytes_per_launch": p2b * wl.numel, "avg_launch_ms": p2_ms,
                         "grad_pass_avg_ms": prof.grad_pass_ms / prof.steps},
            "gpu_launches": prof.launches - launches0,
            "clocks": clocks.summary()}
    multi.close()
    print(json.dumps(line), flush=True)
    return 0


def run_b200(args):
    import torch
    import torch.distributed as dist

    from mixed_precision_zero_b200.zero import zero_step
    from synth import workloads as W
    ws, rank, local = dist_env()
    if ws != args.gpus:
        log(f"note: --gpus {args.gpus} but WORLD_SIZE {ws}; using WORLD_SIZE")
    torch.cuda.set_device(local)
    dev = torch.device("cuda", local)
    if ws > 1 or (args.split and "RANK" in os.environ):
        from datetime import timedelta
        dist.init_process_group("nccl", timeout=timedelta(seconds=300), device_id=dev)
    wl = W.ALL[args.workload]()
    sgd = args.optimizer == "sgd"
    shard, grads, params, state = build_gpu_workload(wl, rank, args.optimizer)
    acc = wl.K >= 5
    p1b, p2b = alg_bytes_per_param(wl.K, acc, sgd)
    kernel2 = "sgd_kernel" if sgd else "adam_kernel"
    stream = torch.cuda.current_stream()

    # One step.  A single GPU runs the fused step; several ranks run the split
    # step, all-reducing the 16 bytes of pass-1 statistics (NCCL) so that every
    # rank takes the same overflow / scale / clip decision.
    stats = torch.zeros(2, dtype=torch.float64, device=dev)

    split = ws > 1 or args.split

    def one_step():
        if not split:
            return shard.step(grads, params, wl.lr)
        if dist.is_initialized():
            return zero_step(shard, grads, params, wl.lr, stats)
        shard.grad_stats(grads, params, stats)
        return shard.apply(grads, params, wl.lr, stats)

    for _ in range(args.warmup):
        res = one_step()
    t_before = shard.get_state()[2]
    shard.reset_profile()
    shard.set_profiling(True)
    launches0 = shard.profile().launches
    ev0, ev1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    if ws > 1:
        dist.barrier()
    torch.cuda.synchronize()
    with ClockSampler(local) as clocks:
        ev0.record(stream)
        for _ in range(args.steps):
            res = one_step()
        ev1.record(stream)
        torch.cuda.synchronize()
    if ws > 1:
        dist.barrier()
    ms_local = ev0.elapsed_time(ev1)
    prof = shard.profile()
    launches = prof.launches - launches0
    applied = shard.get_state()[2] - t_before
    assert applied == args.steps, f"{args.steps - applied} timed steps were skipped (overflow)"
    shard.set_profiling(False)

    ms = max_over_ranks(ms_local, dev)
    total_params = sum_over_ranks(float(wl.numel), dev)
    ms_step = ms / args.steps
    value = total_params * args.steps / (ms * 1e-3) / 1e9
    p1_ms = prof.grad_pass_ms / prof.steps if not split else None  # split steps time only the decision there
    p2_ms = prof.update_pass_ms / prof.steps
    peak, peak_kind = hbm_peak()
    achieved = p2b * wl.numel / (p2_ms * 1e-3) / 1e9
    step_gbs = (p1b + p2b) * wl.numel / (ms_local / args.steps * 1e-3) / 1e9
    traffic = recorded_traffic(args.workload, kernel2)

    # the same step through the asynchronous entry point, captured once in a
    # CUDA graph and replayed (no host synchronisation between steps)
    graph_line = None
    try:
        res_dev = torch.zeros(64, dtype=torch.uint8, device=dev)
        shard.step_async(grads, params, wl.lr, result=res_dev)   # sets up outside the capture
        torch.cuda.synchronize()
        g = torch.cuda.CUDAGraph()
        side = torch.cuda.Stream()
        side.wait_stream(torch.cuda.current_stream())
        with torch.cuda.stream(side), torch.cuda.graph(g, stream=side):
            shard.step_async(grads, params, wl.lr, result=res_dev)
        torch.cuda.synchronize()
        for _ in range(args.warmup):
            g.replay()
        t_g0 = shard.get_state()[2]
        l_g0 = shard.profile().launches
        g0, g1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        if ws > 1:
            dist.barrier()
        torch.cuda.synchronize()
        g0.record(stream)
        for _ in range(args.steps):
            g.replay()
        g1.record(stream)
        torch.cuda.synchronize()
        g_ms = max_over_ranks(g0.elapsed_time(g1), dev)
        assert shard.get_state()[2] - t_g0 == args.steps, "graph replays skipped steps"
        graph_line = {"value": total_params * args.steps / (g_ms * 1e-3) / 1e9, "unit": UNIT,
                      "ms_per_step": g_ms / args.steps, "api": "neox_shard_step_async in a CUDA graph",
                      "gpu_launches": 2 * args.steps}
        del g
    except Exception as exc:  # reported, not fatal: the headline is the synchronous call
        graph_line = {"error": f"{type(exc).__name__}: {exc}"}

    # End to end through the public API: every step copies its gradients from
    # pinned host memory and reads its result back.  One rank: the gradients
    # are double-buffered, so the copy for step s + 1 (on a copy stream)
    # overlaps step s (neox_shard_step_async, whose result the GPU writes into
    # pinned host memory).  Several ranks: the split step, one after the other.
    host_grads = []
    for g in grads:  # straight into pinned memory: one host copy per buffer, not two
        hg = torch.empty(g.shape, dtype=g.dtype, pin_memory=True)
        hg.copy_(g)
        host_grads.append(hg)
    torch.cuda.synchronize()
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    if ws > 1:
        dist.barrier()
    applied0 = shard.get_state()[2]
    if not split:
        from mixed_precision_zero_b200 import _abi
        bufs = [grads, [torch.empty_like(g) for g in grads]]
        res_host = [torch.zeros(64, dtype=torch.uint8).pin_memory() for _ in range(2)]
        copy_stream = torch.cuda.Stream(device=dev)
        copied = [torch.cuda.Event() for _ in range(2)]
        done = [torch.cuda.Event() for _ in range(2)]
        nres = ctypes.sizeof(_abi.neox_step_result)
        e2e_results = []
        e0.record(stream)
        for s in range(args.e2e_steps):
            j = s % 2
            with torch.cuda.stream(copy_stream):
                if s >= 2:
                    copy_stream.wait_event(done[j])  # step s - 2 has finished reading buffer j
                for b, hg in zip(bufs[j], host_grads):
                    b.copy_(hg, non_blocking=True)
                copied[j].record(copy_stream)
            stream.wait_event(copied[j])
            shard.step_async(bufs[j], params, wl.lr, result=res_host[j], stream=stream)
            done[j].record(stream)
            if s >= 1:  # the previous step's result, read on the host while this step runs
                done[1 - j].synchronize()
                e2e_results.append(_abi.neox_step_result.from_buffer_copy(res_host[1 - j].numpy().tobytes()[:nres]))
        done[(args.e2e_steps - 1) % 2].synchronize()
        e2e_results.append(_abi.neox_step_result.from_buffer_copy(
            res_host[(args.e2e_steps - 1) % 2].numpy().tobytes()[:nres]))
        e1.record(stream)
        torch.cuda.synchronize()
        assert [r.applied_steps for r in e2e_results] == list(range(applied0 + 1, applied0 + args.e2e_steps + 1))
        d2h = nres  # the result record the GPU writes into pinned host memory each step
    else:
        e0.record(stream)
        for _ in range(args.e2e_steps):
            for g, hg in zip(grads, host_grads):
                g.copy_(hg, non_blocking=True)
            res = one_step()
        e1.record(stream)
        torch.cuda.synchronize()
        d2h = 64  # the step's device scalar block, read into pinned memory by every call
    e2e_ms = max_over_ranks(e0.elapsed_time(e1), dev)
    e2e_value = total_params * args.e2e_steps / (e2e_ms * 1e-3) / 1e9
    h2d = sum(g.numel() * g.element_size() for g in grads)

    cpu = cpu1 = None
    if rank == 0 and ws == 1 and not args.no_cpu_baseline:
        # the oracle on every host core (contiguous ranges), then on one, on
        # slices of the resident workload (the bytes the GPU stepped on)
        cores = host_cores()
        master_dev = state[0]
        n_thr = oracle_sample_size(wl)
        out = run_oracle_sample(wl, sample_inputs_device(wl, n_thr, master_dev, grads), 50,
                                args.cpu_seconds, threads=cores, optimizer=args.optimizer)
        sec = sum(out["times"])
        what = (f"the whole {wl.name} shard ({out['n']} elements)" if out["n"] == wl.numel else
                f"{out['n']} contiguous elements of {wl.name} (from index {out['lo']})")
        cpu = {"value": out["n"] * len(out["times"]) / sec / 1e9, "unit": UNIT, "cores": cores, "kind": "oracle",
               "sample": f"{len(out['times'])} steps over {what}, split over {cores} host threads by "
                         "contiguous ranges"}
        out = run_oracle_sample(wl, sample_inputs_device(wl, 1 << 24, master_dev, grads), 50,
                                args.cpu_seconds / 3, threads=1, optimizer=args.optimizer)
        sec = sum(out["times"])
        cpu1 = {"value": out["n"] * len(out["times"]) / sec / 1e9, "unit": UNIT, "cores": 1, "kind": "oracle",
                "sample": f"{len(out['times'])} steps over {out['n']} contiguous elements of {wl.name} "
                          f"(from index {out['lo']}), single-threaded"}

    clk = clocks.summary()
    line = {
        "metric": METRIC_SGD if sgd else METRIC, "value": value, "unit": UNIT, "n_gpus": ws, "steps": args.steps, "warmup": args.warmup,
        "ms_per_step": ms_step, "higher_is_better": True, "scaling": "weak", "vs_baseline": None,
        "dtype": "f32", "data": "synthetic",
        "config": {"workload": wl.name, "numel_per_rank": wl.numel, "segments": len(wl.segments or [1]),
                   "grad_buffers": wl.K, "weights": "bf16" if wl.bf16 else "fp16",
                   "element_offset": wl.elem_offset, "loss_scale": wl.bench_scale or wl.init_scale,
                   "state": "fp32 master/m/v", "optimizer": args.optimizer,
                   "l2": f"inputs {((6 if sgd else 14) + 2 * wl.K) * wl.numel / 1e9:.1f} GB per rank >> 126 MB L2; "
                         "no flush",
                   "parallelism": (f"dp{ws}: one shard per GPU, 16-byte NCCL all-reduce of the pass-1 statistics "
                                   "per step" if split else "one shard on one GPU")},
        "hbm": {"step_gbs": step_gbs, "step_frac": step_gbs / peak, "bytes_per_param": p1b + p2b,
                "peak_gbs": peak, "peak_kind": peak_kind},
        "roofline": {"bound": "hbm", "kernel": f"{kernel2} (pass 2)", "achieved": achieved, "peak": peak,
                     "unit": "GB/s", "frac": achieved / peak, "peak_kind": peak_kind,
                     "traffic": traffic, "alg_bytes_per_launch": p2b * wl.numel,
                     "avg_launch_ms": p2_ms, "grad_pass_avg_ms": p1_ms},
        "e2e": {"value": e2e_value, "unit": UNIT, "h2d_bytes_per_step": h2d, "d2h_bytes_per_step": d2h,
                "steps": args.e2e_steps,
                # the gradients' host-to-device rate over the timed region: the bound of this line
                "h2d_gbs": h2d * args.e2e_steps / (e2e_ms * 1e-3) / 1e9},
        "gpu_launches": launches,
        "graph": graph_line,
        "clocks": clk,
        "impl": "b200",
    }
    if cpu:
        line["cpu_baseline"] = cpu
        line["cpu_baseline_single_thread"] = cpu1
    shard.close()
    if dist.is_initialized():
        dist.barrier()
        dist.destroy_process_group()
    if rank == 0:
        print(json.dumps(line), flush=True)
    return 0


# ------------------------------------------------------------------ ZeRO-2 over peer memory

def zero2_plan(wl, world: int, rank: int) -> dict:
    """This rank's part of a ZeRO-2 job over the whole workload: its slice
    [lo, lo + n) of the flat model (equal slices), the slice's segment table,
    and the bytes of one step that cross NVLink for this rank (pass 1 reads
    the other ranks' copies of its gradient slice, pass 2 writes its cast into
    the other ranks' weight buffers)."""
    N = wl.numel
    if N % world:
        raise ValueError(f"{N} parameters do not split into {world} equal slices")
    n = N // world
    lo = rank * n
    segs = None
    if wl.segments:
        segs = []
        for off, cnt, wd, _ in wl.segments:
            a, b = max(off, lo), min(off + cnt, lo + n)
            if a < b:
                segs.append((a - lo, b - a, wd))
    return {"N": N, "n": n, "lo": lo, "segments": segs,
            "nvlink_read_bytes": (world - 1) * 2 * n, "nvlink_write_bytes": (world - 1) * 2 * n}


def run_zero2(args):
    """The whole-model ZeRO-2 step: N ranks (one per GPU of the node), each the
    owner of 1/N of the flat model with its FP32 master/m/v, each holding the
    full gradient of its own micro-batches and a full 16-bit weight copy.  Per
    step (zero.zero2_step): a stream barrier, pass 1 over the N ranks' copies
    of the owned gradient slice through CUDA IPC (pre-divide N, FP32 sum kept
    for pass 2), the 16-byte statistics all-reduce, pass 2 storing the cast
    into every rank's weight buffer, a stream barrier.  Total work is fixed
    (one model), so the scaling is strong."""
    import torch
    import torch.distributed as dist

    import synth
    from mixed_precision_zero_b200 import Hparams, NeoxShard
    from mixed_precision_zero_b200.peer import PeerMap, allgather_weight_dsts, zero2_grad_ptrs
    from mixed_precision_zero_b200.zero import make_stream_barrier, zero2_step
    from synth import workloads as W
    ws, rank, local = dist_env()
    torch.cuda.set_device(local)
    dev = torch.device("cuda", local)
    own_group = False
    if not dist.is_initialized():
        from datetime import timedelta
        if "MASTER_ADDR" not in os.environ:  # one rank without torchrun
            import socket
            sk = socket.socket()
            sk.bind(("127.0.0.1", 0))
            os.environ["MASTER_ADDR"], os.environ["MASTER_PORT"] = "127.0.0.1", str(sk.getsockname()[1])
            sk.close()
            os.environ.setdefault("RANK", "0")
            os.environ.setdefault("WORLD_SIZE", "1")
        dist.init_process_group("nccl", timeout=timedelta(seconds=300), device_id=dev)
        own_group = True
    wl = W.ALL[args.workload]()
    plan = zero2_plan(wl, ws, rank)
    N, n, lo = plan["N"], plan["n"], plan["lo"]
    dt = torch.bfloat16 if wl.bf16 else torch.float16
    scale = wl.bench_scale or wl.init_scale
    master_full = torch.empty(N, dtype=torch.float32, device=dev)
    synth.gpu_master_normal(master_full, wl.master_sigma, wl.seed)       # the same model on every rank
    for s_off, cnt, _, init in (wl.segments or []):
        if init == "zero":
            master_full[s_off:s_off + cnt].zero_()
        elif init == "one":
            master_full[s_off:s_off + cnt].fill_(1.0)
    wfull = master_full.to(dt)
    master = master_full[lo:lo + n].clone()
    del master_full
    m, v = torch.zeros_like(master), torch.zeros_like(master)
    grads_full = torch.empty(N, dtype=dt, device=dev)
    synth.gpu_grad_normal16(grads_full, wl.grad_sigma, scale, wl.seed + 1000 * rank, 0, 1, wl.bf16)
    torch.cuda.synchronize()
    gmap = PeerMap.from_group(grads_full)
    wmap = PeerMap.from_group(wfull)
    hp = Hparams(wl.beta1, wl.beta2, wl.eps, wl.clip, float(ws), scale, 2.0, 1.0, wl.scale_window)
    shard = NeoxShard(master, m, v, hp, wdtype=dt, gdtype=dt, segments=plan["segments"],
                      weight_decay=wl.weight_decay, max_grads=ws, accumulate=True)
    params = wfull[lo:lo + n]
    shard.set_weight_copies(allgather_weight_dsts(wmap, n, wfull.element_size()))
    gptrs = zero2_grad_ptrs(gmap, n, grads_full.element_size())
    stats = torch.zeros(2, dtype=torch.float64, device=dev)
    barrier = make_stream_barrier()
    stream = torch.cuda.current_stream()

    def one_step():
        return zero2_step(shard, gptrs, params, wl.lr, stats, barrier)

    for _ in range(args.warmup):
        one_step()
    t0 = shard.get_state()[2]
    shard.reset_profile()
    shard.set_profiling(True)
    launches0 = shard.profile().launches
    ev0, ev1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    dist.barrier()
    torch.cuda.synchronize()
    with ClockSampler(local) as clocks:
        ev0.record(stream)
        for _ in range(args.steps):
            one_step()
        ev1.record(stream)
        torch.cuda.synchronize()
    dist.barrier()
    assert shard.get_state()[2] - t0 == args.steps, "timed ZeRO-2 steps were skipped (overflow)"
    prof = shard.profile()
    shard.set_profiling(False)
    ms = max_over_ranks(ev0.elapsed_time(ev1), dev)
    ms_step = ms / args.steps
    p2_ms = prof.update_pass_ms / prof.steps
    peak, peak_kind = hbm_peak()
    nv_bytes = plan["nvlink_read_bytes"] + plan["nvlink_write_bytes"]
    # pass 2 of a rank: reads the FP32 sum and master/m/v, writes master/m/v
    # and the 16-bit cast to itself and to the (N - 1) peers
    p2_bytes = (4 + 12 + 12 + 2 * ws) * n
    if ws == 1:  # no peers: pass 2 against the HBM copy bandwidth
        roofline = {"bound": "hbm", "kernel": "adam_kernel (pass 2, FP32 sum)", "avg_launch_ms": p2_ms,
                    "alg_bytes_per_launch": p2_bytes, "achieved": p2_bytes / (p2_ms * 1e-3) / 1e9, "peak": peak,
                    "unit": "GB/s", "frac": p2_bytes / (p2_ms * 1e-3) / 1e9 / peak, "peak_kind": peak_kind,
                    "traffic": None}
    else:  # the bytes each rank moves per direction over NVLink against the measured peer copy
        per_dir = plan["nvlink_read_bytes"] / (ms_step * 1e-3) / 1e9
        roofline = {"bound": "nvlink", "kernel": "whole step (pass 1 peer loads, pass 2 peer stores)",
                    "alg_bytes_per_step_per_direction": plan["nvlink_read_bytes"], "achieved": per_dir,
                    "peak": 770.0, "unit": "GB/s", "frac": per_dir / 770.0,
                    "peak_kind": "measured peer copy per direction on this pool", "traffic": None,
                    "pass2_avg_launch_ms": p2_ms}
    line = {
        "metric": METRIC + " (ZeRO-2 over peer memory)", "value": N * args.steps / (ms * 1e-3) / 1e9, "unit": UNIT,
        "n_gpus": ws, "steps": args.steps, "warmup": args.warmup, "ms_per_step": ms_step,
        "higher_is_better": True, "scaling": "strong", "vs_baseline": None, "dtype": "f32", "data": "synthetic",
        "impl": "b200",
        "config": {"workload": wl.name, "numel_model": N, "numel_per_rank": n, "grad_buffers_per_step": ws,
                   "weights": "bf16" if wl.bf16 else "fp16", "predivide": float(ws),
                   "parallelism": f"zero2 over {ws} ranks: gradient reduce-scatter fused with pass 1 (peer loads), "
                                  "weight all-gather fused with the cast (peer stores), 16-byte statistics "
                                  "all-reduce, stream barriers before and after the step",
                   "l2": "inputs far above the 126 MB L2; no flush"},
        "nvlink": {"bytes_per_rank_per_step": nv_bytes, "read_bytes": plan["nvlink_read_bytes"],
                   "write_bytes": plan["nvlink_write_bytes"],
                   "achieved_gbs_per_rank_whole_step": nv_bytes / (ms_step * 1e-3) / 1e9 if nv_bytes else None,
                   "reference_gbs_per_direction": 770.0},
        "roofline": roofline,
        "gpu_launches": prof.launches - launches0,
        "clocks": clocks.summary(),
    }
    shard.close()
    gmap.close()
    wmap.close()
    dist.barrier()
    if own_group:
        dist.destroy_process_group()
    if rank == 0:
        print(json.dumps(line), flush=True)
    return 0


def main(argv=None):
    args = parse_args(argv)
    if args.impl == "reference":
        return run_reference(args)
    if args.zero2:
        return run_zero2(args)
    if args.api == "multi":
        return run_multi(args)
    return run_b200(args)


if __name__ == "__main__":
    sys.exit(main())
