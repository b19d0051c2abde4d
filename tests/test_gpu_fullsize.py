"""GPU parity at the workloads' full sizes, in the launch configuration bench.py
times (the same kernel instances, grids and vector layouts).

Per call the oracle sees every gradient (copied to the host in chunks and
passed through its single-threaded pass-1 routine on several host threads),
so the overflow flag, the loss-scale trajectory and the norm are checked on
the whole shard.  The AdamW state is tracked by the oracle on a deterministic
sample of elements (every 4096th, the first and last 65,536, windows around
2^31 and 2^32 and around segment boundaries): apart from the global norm and
flag, each element's update depends only on its own inputs, so the sampled
comparison is exact in what it checks.

Two ways of running a call:

* exact -- the split step.  Pass 1 (``grad_stats``) writes the GPU's own
  {sum of squares, non-finite flag}, which must agree with the oracle's
  (flag exactly, norm within relative 1e-5).  The oracle's statistics are then
  written into the device buffer that ``apply`` decides from, so both sides
  form the clip coefficient from the same sum of squares (a double square
  root and division, correctly rounded on both).  From there every element's
  arithmetic is the same sequence of FP32 operations, so master, m, v and the
  16-bit copy must match the oracle bit for bit on every sampled element, at
  every call, over the configured trace length.  The oracle never takes a
  value from the CUDA path; the CUDA decision takes the oracle's input.
* fused -- ``neox_shard_step`` as bench.py times it: the GPU decides from its
  own norm, whose reduction order differs from the oracle's, so the clip
  coefficients can differ in their last bits and the state is compared with
  the stated tolerances (relative 1e-5, absolute floor 1e-7, 1 ulp for the
  16-bit copy).  The largest FP32 ulp distance of m and v over elements with
  |x| > 1e-30 is printed as a diagnostic.
"""
import os
import time

import numpy as np
import pytest
import torch

import oracle
import synth
from mixed_precision_zero_b200 import Hparams, NeoxShard
from synth import workloads as W
from tests.gpu_harness import Guarded, check_close, check_ulp16, ulp_distance_above

pytestmark = [pytest.mark.gpu, pytest.mark.slow]

THREADS = max(1, len(os.sched_getaffinity(0)))


def sample_indices(n, segments=None):
    parts = [np.arange(0, n, 4096, dtype=np.int64), np.arange(0, min(n, 65536)), np.arange(max(0, n - 65536), n)]
    for b in (1 << 31, 1 << 32):
        if b < n:
            parts.append(np.arange(max(0, b - 64), min(n, b + 64)))
    for off, cnt, *_ in (segments or []):
        parts.append(np.arange(max(0, off - 4), min(n, off + 4)))
    return np.unique(np.concatenate(parts))


class FullRun:
    def __init__(self, wl: W.Workload, seed_offset=0, optimizer="adamw"):
        self.wl = wl
        self.optimizer = optimizer
        n = wl.numel
        dt = torch.bfloat16 if wl.bf16 else torch.float16
        off = wl.elem_offset
        self.seed = wl.seed + seed_offset
        self.g = [Guarded(n, dt, off) for _ in range(wl.K)]
        self.w = Guarded(n, dt, off)
        self.master = Guarded(n, torch.float32, off)
        self.m = Guarded(n, torch.float32, off)
        self.v = Guarded(n, torch.float32, off)
        synth.gpu_master_normal(self.master.t, wl.master_sigma, self.seed)
        for so, sc, _, init in (wl.segments or []):
            if init == "zero":
                self.master.t[so:so + sc].zero_()
            elif init == "one":
                self.master.t[so:so + sc].fill_(1.0)
        self.m.t.zero_()
        self.v.t.zero_()
        self.w.t.copy_(self.master.t.to(dt))
        self.hp = Hparams(wl.beta1, wl.beta2, wl.eps, wl.clip, wl.predivide, wl.init_scale, 2.0, 1.0, wl.scale_window,
                          optimizer=optimizer)
        self.shard = NeoxShard(self.master.t, self.m.t, self.v.t, self.hp, wdtype=dt, gdtype=dt,
                               segments=wl.seg_table(), weight_decay=wl.weight_decay, max_grads=wl.K)
        self.ohp = oracle.OracleHparams(wl.beta1, wl.beta2, wl.eps, wl.clip, wl.predivide, wl.init_scale, 2.0, 1.0,
                                        wl.scale_window, optimizer=1 if optimizer == "sgd" else 0)
        self.scaler = oracle.Scaler(wl.init_scale, 0, 0)
        self.segs = oracle.segments_array(wl.seg_table(), n, wl.weight_decay)
        self.idx = sample_indices(n, wl.segments)
        self.idx_dev = torch.from_numpy(self.idx).cuda()
        self.s_master = self._gather32(self.master.t)
        self.s_m = np.zeros_like(self.s_master)
        self.s_v = np.zeros_like(self.s_master)
        self.s_w = oracle.encode16(self.s_master, wl.bf16)
        self.stats = torch.zeros(2, dtype=torch.float64, device="cuda")
        torch.cuda.synchronize()
        self.n_inject = 0

    def _gather32(self, t):
        return t[self.idx_dev].cpu().numpy().copy()

    def _gather16(self, t):
        return t.view(torch.int16)[self.idx_dev].cpu().numpy().view(np.uint16).copy()

    def gen(self, s):
        wl = self.wl
        for k, g in enumerate(self.g):
            if wl.grad_dist == "t3":
                synth.gpu_grad_t3_16(g.t, self.scaler.scale, self.seed, k, s, wl.bf16)
            else:
                synth.gpu_grad_normal16(g.t, wl.grad_sigma, self.scaler.scale, self.seed, k, s, wl.bf16)
        if s in wl.inject_steps:
            i = synth.inject_index(wl.numel, self.seed, s)
            code = np.uint16(synth.inject_value(self.n_inject, wl.bf16)).view(np.int16)
            self.g[0].t.view(torch.int16)[i] = int(code)
            self.n_inject += 1
        hits = 0
        if s in wl.inject_rate_steps:
            for k, g in enumerate(self.g):
                hits += synth.gpu_rate_inject(g.t, wl.inject_rate, self.seed, k, s, wl.bf16)
        return hits

    def oracle_pass1(self, chunk=1 << 26):
        """(non-finite count, sum of squares) over the whole shard on the host."""
        wl = self.wl
        inv_pre, inv_us = oracle.ingest_factors(wl.K, wl.predivide, self.scaler.scale)
        n = wl.numel
        bufs = [torch.empty(min(chunk, n), dtype=torch.int16, pin_memory=True) for _ in range(wl.K)]
        bad, ssum = 0, 0.0
        for lo in range(0, n, chunk):
            hi = min(n, lo + chunk)
            host = []
            for g, b in zip(self.g, bufs):
                b[: hi - lo].copy_(g.t.view(torch.int16)[lo:hi])
                host.append(b[: hi - lo].numpy().view(np.uint16))
            nb, s = oracle.grad_stats(host, wl.bf16, inv_pre, inv_us, threads=THREADS, chunk=1 << 22)
            bad += nb
            ssum += s
        return bad, ssum

    def _oracle_apply(self, sub, info):
        wl = self.wl
        if info.overflow:
            return
        if self.optimizer == "sgd":
            oracle.sgd_apply(self.idx.astype(np.uint64), 0, sub, wl.bf16, self.segs, self.s_master, self.s_w,
                             wl.bf16, self.ohp, wl.lr, info)
        else:
            oracle.adam_apply(self.idx.astype(np.uint64), 0, sub, wl.bf16, self.segs, self.s_master, self.s_m,
                              self.s_v, self.s_w, wl.bf16, self.ohp, wl.lr, info)

    def _check_decision(self, res, info):
        assert res.overflow == info.overflow, (res.overflow, info.overflow)
        assert res.loss_scale == info.scale_used and res.loss_scale_next == info.scale_next
        assert res.applied_steps == info.t and res.good_steps == self.scaler.good

    def step_fused(self, s):
        """neox_shard_step; the GPU decides from its own norm."""
        wl = self.wl
        torch.cuda.synchronize()
        nb, ssum = self.oracle_pass1()
        sub = [self._gather16(g.t) for g in self.g]
        res = self.shard.step([g.t for g in self.g], self.w.t, wl.lr)
        info = oracle.step_decide(self.ohp, self.scaler, wl.lr, nb, ssum)
        self._check_decision(res, info)
        if not info.overflow:
            assert abs(res.grad_norm - info.norm) <= 1e-5 * info.norm, (res.grad_norm, info.norm)
            assert abs(res.clip_coef - info.coef) <= 1e-5 * info.coef
        self._oracle_apply(sub, info)
        return res, info, nb

    def step_exact(self, s):
        """grad_stats, then apply deciding from the oracle's statistics."""
        wl = self.wl
        grads = [g.t for g in self.g]
        torch.cuda.synchronize()
        nb, ssum = self.oracle_pass1()
        sub = [self._gather16(g.t) for g in self.g]
        self.shard.grad_stats(grads, self.w.t, self.stats)
        gpu_sumsq, gpu_flag = (float(x) for x in self.stats.cpu().numpy())
        assert (gpu_flag != 0.0) == (nb > 0), (s, gpu_flag, nb)
        if nb == 0:
            assert abs(np.sqrt(gpu_sumsq) - np.sqrt(ssum)) <= 1e-5 * np.sqrt(ssum), (gpu_sumsq, ssum)
        self.stats.copy_(torch.tensor([ssum, 1.0 if nb else 0.0], dtype=torch.float64))
        res = self.shard.apply(grads, self.w.t, wl.lr, self.stats)
        info = oracle.step_decide(self.ohp, self.scaler, wl.lr, nb, ssum)
        self._check_decision(res, info)
        if not info.overflow:
            assert res.grad_norm == np.float32(info.norm) and res.clip_coef == np.float32(info.coef)
        self._oracle_apply(sub, info)
        return res, info, nb

    def check_state(self, exact):
        got = {"master": self._gather32(self.master.t), "exp_avg": self._gather32(self.m.t),
               "exp_avg_sq": self._gather32(self.v.t)}
        ref = {"master": self.s_master, "exp_avg": self.s_m, "exp_avg_sq": self.s_v}
        gw = self._gather16(self.w.t)
        if exact:
            for k in got:
                diff = np.count_nonzero(got[k].view(np.uint32) != ref[k].view(np.uint32))
                assert diff == 0, f"{k}: {diff} of {got[k].size} sampled elements not bit-exact"
            assert np.array_equal(gw, self.s_w), f"16-bit copy: {np.count_nonzero(gw != self.s_w)} differ"
            return {}
        for k in got:
            check_close(k, got[k], ref[k])
        check_ulp16(gw, self.s_w)
        return {"m_ulp": ulp_distance_above(got["exp_avg"], ref["exp_avg"]),
                "v_ulp": ulp_distance_above(got["exp_avg_sq"], ref["exp_avg_sq"])}

    def guards_intact(self):
        return all(x.guards_intact() for x in (*self.g, self.w, self.master, self.m, self.v))

    def close(self):
        self.shard.close()
        for x in (*self.g, self.w, self.master, self.m, self.v):
            del x.base, x.t
        torch.cuda.empty_cache()


@pytest.fixture(autouse=True)
def _free_memory():
    torch.cuda.set_device(0)
    yield
    torch.cuda.synchronize()
    torch.cuda.empty_cache()


def _run(wl, steps, exact, check_every=1, optimizer="adamw"):
    """`steps` calls; the state is compared after every `check_every`-th call
    and after the last."""
    t0 = time.time()
    r = FullRun(wl, optimizer=optimizer)
    flags, diag = [], {}
    for s in range(1, steps + 1):
        r.gen(s)
        res, info, nb = r.step_exact(s) if exact else r.step_fused(s)
        flags.append(res.overflow)
        if s % check_every == 0 or s == steps:
            d = r.check_state(exact)
            for k, v in d.items():
                diag[k] = max(diag.get(k, 0), v)
    assert r.guards_intact()
    print(f"{wl.name}: {steps} calls ({'split step, oracle statistics, bit-exact' if exact else 'fused step'}), "
          f"{len(r.idx)} sampled elements, {time.time() - t0:.1f}s, {THREADS} host threads"
          + (f"; max FP32 ulp distance m {diag['m_ulp']}, v {diag['v_ulp']} (|x| > 1e-30)" if diag else ""))
    return r, flags


def test_pythia_1p4b_shaped_full_size_exact():
    """The configured 10 calls of the 290-segment shard, bit-exact at every call."""
    wl = W.pythia_1p4b()
    r, flags = _run(wl, wl.steps, exact=True)
    assert flags == [0] * wl.steps
    r.close()


def test_pythia_1p4b_shaped_full_size_sgd_exact():
    """The plain-SGD update over the same 10 calls, bit-exact: master and the
    16-bit copy follow the oracle's SGD, and m and v stay zero."""
    wl = W.pythia_1p4b()
    r, flags = _run(wl, wl.steps, exact=True, optimizer="sgd")
    assert flags == [0] * wl.steps
    assert not r.m.t.any().item() and not r.v.t.any().item()
    r.close()


def test_pythia_1p4b_shaped_full_size_fused():
    wl = W.pythia_1p4b()
    r, flags = _run(wl, 3, exact=False)
    assert flags == [0, 0, 0]
    r.close()


def test_neox20b_slice_misaligned_full_size_exact():
    """2,570,000,001 elements (> 2^31, odd) at element offset 3 of every array:
    the configured 50 calls, bit-exact."""
    wl = W.neox20b_zero1_slice()
    r, flags = _run(wl, wl.steps, exact=True, check_every=10)
    assert flags == [0] * wl.steps
    r.close()


def test_neox20b_slice_misaligned_full_size_fused():
    wl = W.neox20b_zero1_slice()
    r, flags = _run(wl, 2, exact=False)
    assert flags == [0, 0]
    r.close()


def test_accum8_predivide_full_size_exact():
    """K = 8 Student-t(3) x 2^10 buffers, the configured 30 calls: the natural
    FP16 overflows drive the scale down until steps apply; the oracle's exact
    count of non-finite inputs decides every flag, and the rate injections on
    calls 20 and 25 skip those calls."""
    wl = W.accum8_predivide()
    r, flags = _run(wl, wl.steps, exact=True, check_every=5)
    assert flags[0] == 1 and 0 in flags
    assert flags[19] == 1 and flags[24] == 1
    r.close()


def test_opt_style_5e9_bf16_full_size_exact():
    """5e9 BF16 elements (> 2^32): the configured 100 calls with the scripted
    overflows on calls 3, 4 and 57, bit-exact."""
    wl = W.opt_style_5b()
    r, flags = _run(wl, wl.steps, exact=True, check_every=25)
    assert [i + 1 for i, f in enumerate(flags) if f] == [3, 4, 57]
    assert r.scaler.scale == 2.0 ** 13 and r.scaler.t == 97
    r.close()


def test_opt_style_5e9_bf16_full_size_fused():
    wl = W.opt_style_5b()
    r, flags = _run(wl, 5, exact=False)
    assert flags == [0, 0, 1, 1, 0]
    assert r.scaler.scale == 2.0 ** 14 and r.scaler.t == 3
    r.close()


def _trace_property(wl, steps):
    """Full trace of the fused step on the GPU; flags against 'some input not
    finite' (torch reduction on the device) and the scale against the scaler
    rule."""
    r = FullRun(wl)
    scale, good, t = wl.init_scale, 0, 0
    flags = []
    for s in range(1, steps + 1):
        r.scaler.scale = scale
        hits = r.gen(s)
        bad = any(not bool(torch.isfinite(g.t).all().item()) for g in r.g)
        res = r.shard.step([g.t for g in r.g], r.w.t, wl.lr)
        assert res.overflow == int(bad), (s, res.overflow, bad, hits)
        scale, good, t = oracle.scaler_update(r.ohp, scale, good, t, bad)
        if not bad:
            t += 1
        assert res.loss_scale_next == scale and res.applied_steps == t and res.good_steps == good
        flags.append(res.overflow)
    r.close()
    return flags, scale, t


def test_opt_style_100_call_trace():
    flags, scale, t = _trace_property(W.opt_style_5b(), 100)
    assert [i + 1 for i, f in enumerate(flags) if f] == [3, 4, 57]
    assert scale == 2.0 ** 13 and t == 97


def test_accum8_30_call_trace():
    flags, scale, t = _trace_property(W.accum8_predivide(), 30)
    assert flags[0] == 1 and 0 in flags
    assert flags[19] == 1 and flags[24] == 1  # rate injections on calls 20 and 25


def test_multi_tensor_full_size_equals_flat():
    """The 1.41e9-parameter Pythia-shaped shard as 290 separately addressed
    tensors (the multi-tensor entry point, as `bench.py --api multi` runs it)
    against the flat step on a copy of the same bytes, which the exact-mode
    tests tie to the oracle.  Clip off, so both sides apply coefficient 1:
    every byte of master, m, v and the 16-bit copy must agree after every
    call, through an overflow on call 2."""
    from mixed_precision_zero_b200 import NeoxMultiShard
    wl = W.pythia_1p4b()
    n = wl.numel
    hp = Hparams(wl.beta1, wl.beta2, wl.eps, 0.0, wl.predivide, wl.init_scale, 2.0, 1.0, wl.scale_window)
    master = torch.empty(n, dtype=torch.float32, device="cuda")
    synth.gpu_master_normal(master, wl.master_sigma, wl.seed)
    for so, sc, _, init in wl.segments:
        if init == "zero":
            master[so:so + sc].zero_()
        elif init == "one":
            master[so:so + sc].fill_(1.0)
    a = [master, torch.zeros_like(master), torch.zeros_like(master), master.to(torch.float16)]
    b = [x.clone() for x in a]
    g = torch.empty(n, dtype=torch.float16, device="cuda")
    segs = wl.seg_table()
    flat = NeoxShard(a[0], a[1], a[2], hp, segments=segs)
    multi = NeoxMultiShard([{"master": b[0][o:o + c], "exp_avg": b[1][o:o + c], "exp_avg_sq": b[2][o:o + c],
                             "params": b[3][o:o + c], "grads": [g[o:o + c]], "weight_decay": w}
                            for o, c, w in segs], hp)
    for s in range(1, 4):
        synth.gpu_grad_normal16(g, wl.grad_sigma, flat.get_state()[0], wl.seed, 0, s)
        if s == 2:
            g.view(torch.int16)[synth.inject_index(n, wl.seed, s)] = 0x7C00
        ra = flat.step([g], a[3], wl.lr)
        rb = multi.step(wl.lr)
        assert (ra.overflow, ra.loss_scale_next, ra.applied_steps) == (rb.overflow, rb.loss_scale_next, rb.applied_steps)
        assert ra.overflow == (1 if s == 2 else 0)
        if not ra.overflow:
            assert abs(ra.grad_norm - rb.grad_norm) <= 1e-6 * ra.grad_norm
        for x, y in zip(a, b):
            assert torch.equal(x.view(torch.uint8), y.view(torch.uint8))
    flat.close()
    multi.close()
    del a, b, g, master
