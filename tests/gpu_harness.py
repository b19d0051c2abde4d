"""Shared helpers of the GPU parity tests: buffers with guard regions at chosen
element offsets, a shard driven through the C ABI next to the oracle on the
same input bytes, and the comparison rules.

Tolerances (the step's stated parity bar):
  overflow flag, skipped-step state, loss-scale trajectory, counters: exact;
  master / m / v: relative 1e-5 with an absolute floor of 1e-7;
  16-bit working weights: within 1 ulp;  grad norm: relative 1e-5.
With clipping off the clip coefficient is exactly 1 on both sides and the
kernels evaluate every FP32 operation in the oracle's order, so there the
state must match bit for bit.
"""
from __future__ import annotations

import numpy as np
import torch

import oracle
import synth
from mixed_precision_zero_b200 import Hparams, NeoxShard

PAD_BYTES = 4096
PATTERN = 0xA5


def _torch_dtype(bf16: bool):
    return torch.bfloat16 if bf16 else torch.float16


class Guarded:
    """A device array of n elements starting `offset` elements past a 512-byte
    boundary, with PAD_BYTES of a fixed byte pattern on both sides."""

    def __init__(self, n: int, dtype, offset: int = 0):
        esz = torch.empty(0, dtype=dtype).element_size()
        pad = PAD_BYTES // esz
        self.base = torch.empty(pad * 2 + offset + n, dtype=dtype, device="cuda")
        self.base.view(torch.uint8).fill_(PATTERN)
        self.lo = pad + offset
        self.n = n
        self.t = self.base.narrow(0, self.lo, n)

    def guards_intact(self) -> bool:
        raw = self.base.view(torch.uint8)
        esz = self.base.element_size()
        head = raw[: self.lo * esz]
        tail = raw[(self.lo + self.n) * esz:]
        return bool((head == PATTERN).all().item()) and bool((tail == PATTERN).all().item())


def to_u16(t: torch.Tensor) -> np.ndarray:
    return t.contiguous().view(torch.int16).cpu().numpy().view(np.uint16)


def ordered16(h: np.ndarray) -> np.ndarray:
    h = h.astype(np.int64)
    return np.where(h & 0x8000, -(h & 0x7FFF), h)


def oracle_hparams(hp: Hparams):
    """The oracle's copy of the library's hyperparameters."""
    return oracle.OracleHparams(hp.beta1, hp.beta2, hp.eps, hp.clip_norm, hp.predivide, hp.init_scale,
                                hp.scale_factor, hp.min_scale, hp.scale_window, hysteresis=hp.hysteresis,
                                optimizer={"adamw": 0, "sgd": 1}[hp.optimizer])


class ShardCase:
    """A shard on the GPU (driven through the C ABI) and the oracle's copy."""

    def __init__(self, n, *, K=1, wbf16=False, gbf16=False, hp: Hparams | None = None, lr=6e-4,
                 segments=None, default_wd=0.1, max_grads=1, offsets=None, seed=0, master_sigma=0.02,
                 seg_init=None, accumulate=False):
        self.n, self.K, self.lr = n, K, lr
        self.wbf16, self.gbf16 = wbf16, gbf16
        self.hp = hp or Hparams()
        offsets = offsets or {}
        self.g = [Guarded(n, _torch_dtype(gbf16), offsets.get(f"g{k}", offsets.get("all", 0))) for k in range(K)]
        self.w = Guarded(n, _torch_dtype(wbf16), offsets.get("w", offsets.get("all", 0)))
        self.master = Guarded(n, torch.float32, offsets.get("master", offsets.get("all", 0)))
        self.m = Guarded(n, torch.float32, offsets.get("m", offsets.get("all", 0)))
        self.v = Guarded(n, torch.float32, offsets.get("v", offsets.get("all", 0)))
        if n:
            synth.gpu_master_normal(self.master.t, master_sigma, seed)
            if seg_init:
                for off, cnt, _, init in seg_init:
                    if init == "zero":
                        self.master.t[off:off + cnt].zero_()
                    elif init == "one":
                        self.master.t[off:off + cnt].fill_(1.0)
            self.m.t.zero_()
            self.v.t.zero_()
            self.w.t.copy_(self.master.t.to(_torch_dtype(wbf16)))
        torch.cuda.synchronize()
        self.segments = segments
        self.shard = NeoxShard(self.master.t, self.m.t, self.v.t, self.hp,
                               wdtype=_torch_dtype(wbf16), gdtype=_torch_dtype(gbf16),
                               segments=segments, weight_decay=default_wd, max_grads=max_grads,
                               accumulate=accumulate)
        ohp = oracle_hparams(self.hp)
        master_host = self.master.t.cpu().numpy()
        self.orc = oracle.OracleShard(master_host, ohp, wbf16=wbf16, gbf16=gbf16, segments=segments,
                                      default_wd=default_wd)
        if n:
            assert np.array_equal(to_u16(self.w.t), self.orc.w), "initial working copy differs from RNE16(master)"
        self.seed = seed

    # -- inputs -------------------------------------------------------------------
    def gen_normal(self, step, sigma):
        for k, g in enumerate(self.g):
            synth.gpu_grad_normal16(g.t, sigma, self.orc.scale, self.seed, k, step, self.gbf16)

    def gen_t3(self, step):
        for k, g in enumerate(self.g):
            synth.gpu_grad_t3_16(g.t, self.orc.scale, self.seed, k, step, self.gbf16)

    def inject(self, step, count=0, buffer=0):
        idx = synth.inject_index(self.n, self.seed, step)
        code = int(synth.inject_value(count, self.gbf16))
        self.g[buffer].t.view(torch.int16)[idx] = np.int16(np.uint16(code).view(np.int16))
        return idx

    # -- one call on both sides -----------------------------------------------------
    def step(self, lr=None):
        lr = self.lr if lr is None else lr
        torch.cuda.synchronize()
        host = [to_u16(g.t) for g in self.g]
        res = self.shard.step([g.t for g in self.g], self.w.t, lr)
        info = self.orc.step(host, lr)
        return res, info

    def check_result(self, res, info, norm_rtol=1e-5):
        assert res.overflow == info.overflow
        assert res.loss_scale == info.scale_used
        assert res.loss_scale_next == info.scale_next
        assert res.applied_steps == info.t
        assert res.good_steps == self.orc.scaler.good
        if info.overflow:
            assert np.isinf(res.grad_norm) and res.clip_coef == 0.0
        else:
            assert abs(res.grad_norm - info.norm) <= norm_rtol * abs(info.norm) + 1e-30, (res.grad_norm, info.norm)
            assert abs(res.clip_coef - info.coef) <= 1e-5 * info.coef

    def check_state(self, exact=False):
        gm, gmm, gv = (x.t.cpu().numpy() for x in (self.master, self.m, self.v))
        gw = to_u16(self.w.t)
        if exact:
            for name, a, b in (("master", gm, self.orc.master), ("m", gmm, self.orc.m), ("v", gv, self.orc.v)):
                assert a.tobytes() == b.tobytes(), f"{name} not bit-exact: {np.count_nonzero(a != b)} differ"
            assert np.array_equal(gw, self.orc.w)
            return
        for name, a, b in (("master", gm, self.orc.master), ("m", gmm, self.orc.m), ("v", gv, self.orc.v)):
            check_close(name, a, b)
        check_ulp16(gw, self.orc.w)
        # non-gating: how far m and v are in FP32 ulps where the absolute floor
        # would hide a difference (|x| > 1e-30)
        print(f"max FP32 ulp distance: m {ulp_distance_above(gmm, self.orc.m)}, "
              f"v {ulp_distance_above(gv, self.orc.v)}")

    def guards_intact(self):
        return all(x.guards_intact() for x in (*self.g, self.w, self.master, self.m, self.v))

    def close(self):
        self.shard.close()


def check_close(name, a, b, rtol=1e-5, atol=1e-7):
    a = np.asarray(a, np.float64)
    b = np.asarray(b, np.float64)
    bad = ~(np.abs(a - b) <= atol + rtol * np.abs(b))
    assert not bad.any(), (f"{name}: {bad.sum()} of {a.size} outside rtol {rtol} atol {atol}; "
                           f"first at {np.flatnonzero(bad)[:5]}: {a[bad][:5]} vs {b[bad][:5]}")


def check_ulp16(a, b):
    d = np.abs(ordered16(a) - ordered16(b))
    assert d.max(initial=0) <= 1, f"16-bit weights differ by up to {d.max()} ulp at {np.flatnonzero(d > 1)[:5]}"


def ulp_distance_above(a, b, floor=1e-30) -> int:
    """ulp_distance32 over the elements whose reference b exceeds `floor` in
    magnitude (a diagnostic of m and v, whose values sit far below the
    absolute floor of the tolerance)."""
    b = np.asarray(b, np.float32)
    sel = np.abs(b) > floor
    return ulp_distance32(np.asarray(a, np.float32)[sel], b[sel]) if sel.any() else 0


def ulp_distance32(a, b) -> int:
    """Largest distance in FP32 ulps between same-sign finite values (diagnostic)."""
    ai = np.asarray(a, np.float32).view(np.int32).astype(np.int64)
    bi = np.asarray(b, np.float32).view(np.int32).astype(np.int64)
    ai = np.where(ai < 0, -(ai & 0x7FFFFFFF), ai)
    bi = np.where(bi < 0, -(bi & 0x7FFFFFFF), bi)
    return int(np.abs(ai - bi).max(initial=0))
