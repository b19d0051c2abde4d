"""GPU parity of the multi-tensor (non-flat) step: a shard made of separately
allocated tensors, stepped in one pair of launches, against the oracle over
the concatenation of the tensors (one weight-decay segment per tensor)."""
import ctypes

import numpy as np
import pytest
import torch

import oracle
import synth
from mixed_precision_zero_b200 import Hparams, NeoxError, NeoxMultiShard, NeoxShard, _abi
from tests.gpu_harness import Guarded, check_close, check_ulp16, oracle_hparams, to_u16

pytestmark = pytest.mark.gpu

SIZES = [0, 1, 7, 8, 9, 4097, 65536 * 8 + 3, 131073, 300003, 2]
OFFSETS = [0, 1, 2, 3, 5, 7, 0, 3, 1, 6]
WDS = [0.1, 0.0, 0.1, 0.05, 0.0, 0.1, 0.1, 0.0, 0.1, 0.1]


class MultiCase:
    def __init__(self, K=1, hp=None, wbf16=False, gbf16=False, seed=3, lr=6e-4, same_offset=False):
        """same_offset: every array of tensor i starts at the same element
        offset, so every tensor streams 8-element vectors (pass 1 takes them
        as one sequence) after a peeled head; otherwise the arrays of most
        tensors have different residues and narrower vectors."""
        self.K, self.lr, self.seed, self.gbf16 = K, lr, seed, gbf16
        self.hp = hp or Hparams()
        wdt = torch.bfloat16 if wbf16 else torch.float16
        gdt = torch.bfloat16 if gbf16 else torch.float16
        self.parts = []
        for i, (n, off, wd) in enumerate(zip(SIZES, OFFSETS, WDS)):
            woff = off if same_offset else (off * 3) % 8
            goff = [off if same_offset else (off + k) % 8 for k in range(K)]
            p = {"n": n, "wd": wd, "master": Guarded(n, torch.float32, off), "m": Guarded(n, torch.float32, off),
                 "v": Guarded(n, torch.float32, off), "w": Guarded(n, wdt, woff),
                 "g": [Guarded(n, gdt, goff[k]) for k in range(K)]}
            if n:
                synth.gpu_master_normal(p["master"].t, 0.02, seed, tensor_id=i)
                p["m"].t.zero_()
                p["v"].t.zero_()
                p["w"].t.copy_(p["master"].t.to(wdt))
            self.parts.append(p)
        torch.cuda.synchronize()
        self.shard = NeoxMultiShard([{"master": p["master"].t, "exp_avg": p["m"].t, "exp_avg_sq": p["v"].t,
                                      "params": p["w"].t, "grads": [g.t for g in p["g"]], "weight_decay": p["wd"]}
                                     for p in self.parts], self.hp)
        segs, off = [], 0
        for p in self.parts:
            if p["n"]:
                segs.append((off, p["n"], p["wd"]))
            off += p["n"]
        self.total = off
        master = np.concatenate([p["master"].t.cpu().numpy() for p in self.parts])
        ohp = oracle_hparams(self.hp)
        self.orc = oracle.OracleShard(master, ohp, wbf16=wbf16, gbf16=gbf16, segments=segs)

    def gen(self, s, sigma):
        for i, p in enumerate(self.parts):
            for k, g in enumerate(p["g"]):
                if p["n"]:
                    synth.gpu_grad_normal16(g.t, sigma, self.orc.scale, self.seed, 16 * i + k, s, self.gbf16)

    def step(self):
        torch.cuda.synchronize()
        host = [np.concatenate([to_u16(p["g"][k].t) for p in self.parts]) for k in range(self.K)]
        res = self.shard.step(self.lr)
        info = self.orc.step(host, self.lr)
        return res, info

    def check(self, res, info, exact=False):
        assert res.overflow == info.overflow and res.loss_scale_next == info.scale_next
        assert res.applied_steps == info.t and res.loss_scale == info.scale_used
        if not info.overflow:
            assert abs(res.grad_norm - info.norm) <= 1e-5 * info.norm
        cat = lambda key: np.concatenate([p[key].t.cpu().numpy() for p in self.parts])
        gw = np.concatenate([to_u16(p["w"].t) for p in self.parts])
        if exact:
            for name, a, b in (("master", cat("master"), self.orc.master), ("m", cat("m"), self.orc.m),
                               ("v", cat("v"), self.orc.v)):
                assert a.tobytes() == b.tobytes(), name
            assert np.array_equal(gw, self.orc.w)
        else:
            check_close("master", cat("master"), self.orc.master)
            check_close("m", cat("m"), self.orc.m)
            check_close("v", cat("v"), self.orc.v)
            check_ulp16(gw, self.orc.w)
        for p in self.parts:
            for x in (p["master"], p["m"], p["v"], p["w"], *p["g"]):
                assert x.guards_intact()


@pytest.mark.parametrize("wbf16,gbf16", [(False, False), (True, True)])
def test_multi_bit_exact_clip_off(wbf16, gbf16):
    c = MultiCase(hp=Hparams(clip_norm=0.0, init_scale=2.0 ** 12), wbf16=wbf16, gbf16=gbf16, lr=1e-3)
    for s in range(1, 5):
        c.gen(s, 3e-3)
        res, info = c.step()
        c.check(res, info, exact=True)
    c.shard.close()


@pytest.mark.parametrize("K,pre", [(1, 1.0), (3, 2.0)])
def test_multi_with_clip_and_overflow(K, pre):
    c = MultiCase(K=K, hp=Hparams(clip_norm=1.0, predivide=pre, init_scale=2.0 ** 14, scale_window=2))
    for s in range(1, 7):
        c.gen(s, 2e-3)
        if s == 3:
            c.parts[7]["g"][K - 1].t.view(torch.int16)[100] = 0x7C00
        res, info = c.step()
        assert res.overflow == (1 if s == 3 else 0)
        c.check(res, info)
    c.shard.close()


@pytest.mark.parametrize("K,bf16", [(1, False), (3, True)])
def test_multi_sequence_path_bit_exact(K, bf16):
    """Every tensor on 8-element vectors after its head (pass 1 deals all of
    them to the threads as one sequence), K buffers each: bit-exact against
    the oracle with clipping off, through an overflow in the last buffer."""
    c = MultiCase(K=K, hp=Hparams(clip_norm=0.0, predivide=float(K), init_scale=2.0 ** 12, scale_window=2),
                  wbf16=bf16, gbf16=bf16, lr=1e-3, same_offset=True)
    for s in range(1, 6):
        c.gen(s, 3e-3)
        if s == 2:
            c.parts[8]["g"][K - 1].t.view(torch.int16)[12345] = 0x7F80 if bf16 else 0x7C00
        res, info = c.step()
        assert res.overflow == (1 if s == 2 else 0)
        c.check(res, info, exact=True)
    c.shard.close()


def test_multi_matches_flat_handle_on_views():
    """Tensors that are views of one flat buffer (a 2-layer, hidden-64 Pythia
    layout): with clipping off the multi-tensor step and the flat step with
    one segment per tensor give identical bytes."""
    from synth import workloads as W
    segs = W.pythia_like_segments(layers=2, hidden=64, vocab=1000)
    n = segs[-1][0] + segs[-1][1]
    hp = Hparams(clip_norm=0.0, init_scale=2.0 ** 10)
    master = torch.empty(n, dtype=torch.float32, device="cuda")
    synth.gpu_master_normal(master, 0.02, 8)
    a = [master, torch.zeros_like(master), torch.zeros_like(master), master.to(torch.float16)]
    b = [x.clone() for x in a]
    g = torch.empty(n, dtype=torch.float16, device="cuda")
    flat = NeoxShard(a[0], a[1], a[2], hp, segments=[(o, k, w) for o, k, w, _ in segs])
    multi = NeoxMultiShard([{"master": b[0][o:o + k], "exp_avg": b[1][o:o + k], "exp_avg_sq": b[2][o:o + k],
                             "params": b[3][o:o + k], "grads": [g[o:o + k]], "weight_decay": w}
                            for o, k, w, _ in segs], hp)
    for s in range(1, 5):
        synth.gpu_grad_normal16(g, 5e-2, 2.0 ** 10, 8, 0, s)
        ra = flat.step([g], a[3], 1e-3)
        rb = multi.step(1e-3)
        assert ra.overflow == rb.overflow and ra.applied_steps == rb.applied_steps
        assert abs(ra.grad_norm - rb.grad_norm) <= 1e-6 * ra.grad_norm
    for x, y in zip(a, b):
        assert torch.equal(x.view(torch.uint8), y.view(torch.uint8))
    flat.close()
    multi.close()


def test_multi_async_graph_and_rebind():
    c = MultiCase(hp=Hparams(clip_norm=1.0, init_scale=2.0 ** 16, scale_window=3))
    res_dev = torch.zeros(64, dtype=torch.uint8, device="cuda")
    lr_dev = torch.full((1,), c.lr, dtype=torch.float32, device="cuda")
    c.gen(1, 1e-3)
    torch.cuda.synchronize()
    host = [np.concatenate([to_u16(p["g"][0].t) for p in c.parts])]
    c.shard.step_async(result=res_dev, lr_device=lr_dev)
    info = c.orc.step(host, c.lr)
    torch.cuda.synchronize()
    graph = torch.cuda.CUDAGraph()
    side = torch.cuda.Stream()
    side.wait_stream(torch.cuda.current_stream())
    with torch.cuda.stream(side), torch.cuda.graph(graph, stream=side):
        c.shard.step_async(result=res_dev, lr_device=lr_dev)
    torch.cuda.synchronize()
    for s in range(2, 6):
        c.gen(s, 1e-3)
        torch.cuda.synchronize()
        host = [np.concatenate([to_u16(p["g"][0].t) for p in c.parts])]
        graph.replay()
        info = c.orc.step(host, c.lr)
        torch.cuda.synchronize()
        r = _abi.neox_step_result.from_buffer_copy(res_dev.cpu().numpy().tobytes()[:32])
        c.check(r, info)
    del graph
    # point every tensor at new gradient buffers with the same alignment
    new = [[Guarded(p["n"], torch.float16, (OFFSETS[i] + 0) % 8) for _ in range(1)] for i, p in enumerate(c.parts)]
    for i, p in enumerate(c.parts):
        if p["n"]:
            synth.gpu_grad_normal16(new[i][0].t, 1e-3, c.orc.scale, 99, i, 7)
        p["g"] = new[i]
    c.shard.rebind_grads([[g.t for g in p["g"]] for p in c.parts])
    res, info = c.step()
    c.check(res, info)
    c.shard.close()


def test_multi_rejects_bad_tensors():
    n = 1000
    m = torch.zeros(n, dtype=torch.float32, device="cuda")
    w = torch.zeros(n, dtype=torch.float16, device="cuda")
    good = {"master": m, "exp_avg": m.clone(), "exp_avg_sq": m.clone(), "params": w, "grads": [w.clone()]}
    with pytest.raises(ValueError):   # the binding refuses a K that differs between tensors
        NeoxMultiShard([good, {**good, "grads": [w.clone(), w.clone()]}])
    bad = {**good}
    bad["params"] = torch.zeros(n + 1, dtype=torch.float16, device="cuda")[1:]
    s = NeoxMultiShard([bad])   # odd element offset is fine (2-byte aligned)
    s.close()
    t = _abi.neox_tensor(n, 0.1, m.data_ptr(), m.data_ptr() + 2, m.data_ptr(), w.data_ptr(), None)
    ts = _abi.neox_tensor_set(1, 1, _abi.NEOX_FP16, _abi.NEOX_FP16, ctypes.pointer(t))
    with pytest.raises(NeoxError) as ei:
        _abi.neox_multi_create(ts, Hparams().c(), 0)
    assert ei.value.status == _abi.NEOX_ERR_INVALID_ARGUMENT


@pytest.mark.parametrize("optimizer", ["adamw", "sgd"])
def test_multi_large_tensors_match_flat(optimizer):
    """Tensors many grid strides long (the SGD form's four-stride batches, the
    rotated starts wrapping around the thread count) against the flat step on
    the same bytes, which is itself checked against the oracle: with clipping
    off the two give identical state."""
    torch.cuda.set_device(0)
    sizes = [3_000_017, 5, 2_000_003, 1_048_576, 777]
    wds = [0.1, 0.0, 0.1, 0.05, 0.0]
    segs, off = [], 0
    for n_, wd in zip(sizes, wds):
        segs.append((off, n_, wd))
        off += n_
    n = off
    hp = Hparams(clip_norm=0.0, init_scale=2.0 ** 10, optimizer=optimizer)
    master = torch.empty(n, dtype=torch.float32, device="cuda")
    synth.gpu_master_normal(master, 0.02, 12)
    a = [master, torch.zeros_like(master), torch.zeros_like(master), master.to(torch.float16)]
    b = [x.clone() for x in a]
    gs = [torch.empty(n, dtype=torch.float16, device="cuda") for _ in range(2)]
    flat = NeoxShard(a[0], a[1], a[2], hp, segments=segs, max_grads=2)
    multi = NeoxMultiShard([{"master": b[0][o:o + k], "exp_avg": b[1][o:o + k], "exp_avg_sq": b[2][o:o + k],
                             "params": b[3][o:o + k], "grads": [g[o:o + k] for g in gs], "weight_decay": w}
                            for o, k, w in segs], hp)
    for s in range(1, 5):
        for k, g in enumerate(gs):
            synth.gpu_grad_normal16(g, 2e-3, 2.0 ** 10, 12, k, s)
        ra = flat.step(gs, a[3], 1e-2)
        rb = multi.step(1e-2)
        assert ra.overflow == rb.overflow == 0 and ra.applied_steps == rb.applied_steps
        assert abs(ra.grad_norm - rb.grad_norm) <= 1e-6 * ra.grad_norm
    for x, y in zip(a, b):
        assert torch.equal(x.view(torch.uint8), y.view(torch.uint8))
    flat.close()
    multi.close()
