"""GPU parity of the two levers the OPT summary's "方法适配" section reports
using when the loss scale collapsed: a loss scaler with hysteresis (a back-off
only after several overflows since the last growth; reset on demand) and plain
SGD in place of AdamW.  Both are checked against the oracle through the C ABI,
flat and multi-tensor, synchronous and graph-replayed."""
import ctypes

import numpy as np
import pytest
import torch

import synth
from mixed_precision_zero_b200 import Hparams, NeoxError, NeoxShard, _abi
from tests.gpu_harness import ShardCase, check_close, check_ulp16, oracle_hparams, to_u16

pytestmark = pytest.mark.gpu

# Steps whose gradients carry an inf/NaN: a run of three, a pair, singles.
OVERFLOWS = {2, 3, 4, 7, 8, 12, 15}


def _run(c: ShardCase, steps, sigma=2e-3, overflows=OVERFLOWS, exact=False):
    for s in range(1, steps + 1):
        c.gen_normal(s, sigma)
        if s in overflows:
            c.inject(s, count=s)
        res, info = c.step()
        c.check_result(res, info)
        assert res.overflow == (1 if s in overflows else 0)
        assert c.shard.get_hysteresis() == c.orc.scaler.hyst
    c.check_state(exact=exact)
    assert c.guards_intact()


@pytest.mark.parametrize("hyst", [0, 1, 2, 3])
def test_hysteresis_trajectory(hyst):
    torch.cuda.set_device(0)
    c = ShardCase(300_007, hp=Hparams(clip_norm=0.0, init_scale=2.0 ** 14, scale_window=3, hysteresis=hyst),
                  lr=1e-3, seed=41)
    _run(c, 18, exact=True)
    c.close()


@pytest.mark.parametrize("wbf16,gbf16,K,max_grads,offsets", [
    (False, False, 1, 1, None),
    (True, True, 1, 1, {"all": 3}),
    (False, True, 3, 1, {"g0": 1, "g1": 5, "g2": 7, "w": 2, "master": 0, "m": 0, "v": 0}),
    (False, False, 6, 8, None),          # the FP32-sum buffer path
])
def test_sgd_bit_exact_clip_off(wbf16, gbf16, K, max_grads, offsets):
    torch.cuda.set_device(0)
    c = ShardCase(700_001, K=K, wbf16=wbf16, gbf16=gbf16, max_grads=max_grads, offsets=offsets, seed=42,
                  hp=Hparams(clip_norm=0.0, init_scale=2.0 ** 12, predivide=float(K), optimizer="sgd"), lr=5e-2,
                  segments=[(0, 4096, 0.0), (4096, 700_001 - 4096, 0.1)])
    _run(c, 6, overflows={3}, exact=True)
    # m and v are neither read nor written by SGD
    assert not c.m.t.any().item() and not c.v.t.any().item()
    c.close()


@pytest.mark.parametrize("wbf16,offset", [(False, 0), (True, 5)])
def test_sgd_unrolled_loop_bit_exact(wbf16, offset):
    """A shard long enough that every thread runs the SGD kernel's four-stride
    batches (more than 4 x resident threads x 8 elements), plus the one-stride
    remainder, the peeled head and the ragged tail."""
    torch.cuda.set_device(0)
    n = 6_000_007
    c = ShardCase(n, wbf16=wbf16, gbf16=wbf16, offsets={"all": offset}, seed=46, lr=2e-2,
                  hp=Hparams(clip_norm=0.0, init_scale=2.0 ** 12, optimizer="sgd"),
                  segments=[(0, 1_000_000, 0.1), (1_000_000, 3, 0.0), (1_000_003, n - 1_000_003, 0.1)])
    _run(c, 3, overflows={2}, exact=True)
    c.close()


def test_sgd_with_clip_overflow_and_hysteresis():
    torch.cuda.set_device(0)
    # Large gradients (norm about 500, so the clip is active) at a scale that
    # keeps them finite in FP16: the scale peaks at 2^8 on this overflow
    # pattern, and |g|*S stays below about 1e3.
    c = ShardCase(1_000_003, hp=Hparams(clip_norm=0.3, init_scale=2.0 ** 8, scale_window=2, hysteresis=2,
                                        optimizer="sgd"), lr=1e-2, seed=43)
    _run(c, 16, sigma=0.5)
    c.close()


def test_switch_adamw_to_sgd_and_reset_scaler():
    """AdamW for a while, then the OPT-style interventions: switch to SGD and
    reset the scaler (set_state refills the hysteresis count)."""
    torch.cuda.set_device(0)
    hp = Hparams(clip_norm=0.0, init_scale=2.0 ** 14, scale_window=4, hysteresis=3)
    c = ShardCase(250_001, hp=hp, lr=1e-3, seed=44)
    _run(c, 5, overflows={2, 3})
    m_before = c.m.t.clone()
    assert c.shard.get_hysteresis() == 1 == c.orc.scaler.hyst
    sgd = Hparams(clip_norm=0.0, init_scale=2.0 ** 14, scale_window=4, hysteresis=3, optimizer="sgd")
    c.shard.set_hparams(sgd)
    c.orc.hp = oracle_hparams(sgd)
    # reset: a healthy scale, counters cleared, hysteresis count full again
    c.shard.set_state(2.0 ** 12, 0, c.orc.scaler.t)
    c.orc.scaler.scale, c.orc.scaler.good, c.orc.scaler.hyst = 2.0 ** 12, 0, 3
    assert c.shard.get_hysteresis() == 3
    for s in range(6, 12):
        c.gen_normal(s, 2e-3)
        if s in (7, 8):
            c.inject(s)
        res, info = c.step(lr=1e-2)
        c.check_result(res, info)
        assert c.shard.get_hysteresis() == c.orc.scaler.hyst
    assert torch.equal(c.m.t, m_before)
    c.check_state(exact=True)
    # an exact checkpoint of the count
    c.shard.set_hysteresis(1)
    assert c.shard.get_hysteresis() == 1
    with pytest.raises(NeoxError):
        c.shard.set_hysteresis(-1)
    c.close()


def test_sgd_graph_replay_matches_oracle():
    """SGD through the asynchronous step captured in a CUDA graph, the learning
    rate read from device memory: bit-exact with the oracle (SGD has no bias
    correction, so the device-side step size plays no part)."""
    torch.cuda.set_device(0)
    n = 400_009
    hp = Hparams(clip_norm=0.0, init_scale=2.0 ** 12, scale_window=2, hysteresis=2, optimizer="sgd")
    c = ShardCase(n, hp=hp, lr=3e-2, seed=45)
    res_dev = torch.zeros(64, dtype=torch.uint8, device="cuda")
    lr_dev = torch.full((1,), c.lr, dtype=torch.float32, device="cuda")
    grads = [g.t for g in c.g]
    c.gen_normal(1, 1e-3)
    torch.cuda.synchronize()
    host = [to_u16(g.t) for g in c.g]
    c.shard.step_async(grads, c.w.t, result=res_dev, lr_device=lr_dev)
    c.orc.step(host, c.lr)
    torch.cuda.synchronize()
    graph = torch.cuda.CUDAGraph()
    side = torch.cuda.Stream()
    side.wait_stream(torch.cuda.current_stream())
    with torch.cuda.stream(side), torch.cuda.graph(graph, stream=side):
        c.shard.step_async(grads, c.w.t, result=res_dev, lr_device=lr_dev)
    torch.cuda.synchronize()
    for s in range(2, 9):
        c.gen_normal(s, 1e-3)
        if s in (3, 4, 6):
            c.inject(s)
        lr = 3e-2 * (1.0 - 0.1 * s)
        lr_dev.fill_(lr)
        torch.cuda.synchronize()
        host = [to_u16(g.t) for g in c.g]
        graph.replay()
        info = c.orc.step(host, float(np.float32(lr)))
        torch.cuda.synchronize()
        r = _abi.neox_step_result.from_buffer_copy(res_dev.cpu().numpy().tobytes()[:ctypes.sizeof(_abi.neox_step_result)])
        c.check_result(r, info)
    del graph
    assert c.shard.get_hysteresis() == c.orc.scaler.hyst
    c.check_state(exact=True)
    c.close()


def test_multi_sgd_with_hysteresis():
    from tests.test_gpu_multi import MultiCase
    torch.cuda.set_device(0)
    c = MultiCase(K=2, hp=Hparams(clip_norm=1.0, predivide=2.0, init_scale=2.0 ** 14, scale_window=2, hysteresis=2,
                                  optimizer="sgd"), lr=1e-2)
    for s in range(1, 9):
        c.gen(s, 2e-3)
        if s in (2, 3, 6):
            c.parts[5]["g"][1].t.view(torch.int16)[17] = 0x7C00
        res, info = c.step()
        assert res.overflow == (1 if s in (2, 3, 6) else 0)
        c.check(res, info)
        assert c.shard.get_hysteresis() == c.orc.scaler.hyst
    for p in c.parts:
        assert not p["m"].t.any().item() and not p["v"].t.any().item()
    c.shard.close()


def test_multi_hysteresis_bit_exact():
    from tests.test_gpu_multi import MultiCase
    torch.cuda.set_device(0)
    c = MultiCase(hp=Hparams(clip_norm=0.0, init_scale=2.0 ** 12, scale_window=3, hysteresis=3), lr=1e-3)
    for s in range(1, 11):
        c.gen(s, 3e-3)
        if s in (2, 3, 4, 5):
            c.parts[6]["g"][0].t.view(torch.int16)[s] = 0x7E00
        res, info = c.step()
        c.check(res, info, exact=True)
        assert c.shard.get_hysteresis() == c.orc.scaler.hyst
    c.shard.set_state(2.0 ** 10, 0, info.t)
    assert c.shard.get_hysteresis() == 3
    c.shard.close()


def test_checkpoint_resume_keeps_the_hysteresis_count():
    """N steps, state_dict() + the state arrays, destroy, re-create,
    load_state_dict(), M more steps == N + M uninterrupted steps, byte for
    byte.  The count is mid-way at the split (two overflows of three
    tolerated), so a resume that refilled it would back off one step later."""
    n = 200_003
    hp = Hparams(init_scale=2.0 ** 12, scale_window=4, hysteresis=3)
    overflows = {2, 3, 5}

    def run(split, exact_count=True):
        c = ShardCase(n, hp=hp, lr=6e-4, seed=47)
        for s in range(1, 9):
            if s == split:
                saved = [x.t.clone() for x in (c.master, c.m, c.v, c.w)]
                sd = c.shard.state_dict()
                assert sd["hysteresis_count"] == 1
                c.shard.close()
                for x, y in zip((c.master, c.m, c.v, c.w), saved):
                    x.t.copy_(y)
                c.shard = NeoxShard(c.master.t, c.m.t, c.v.t, hp, weight_decay=0.1)
                if exact_count:
                    c.shard.load_state_dict(sd)
                else:   # a scaler reset instead: the count is refilled
                    c.shard.set_state(sd["loss_scale"], sd["good_steps"], sd["applied_steps"])
            c.gen_normal(s, 1e-3)
            if s in overflows:
                c.inject(s)
            c.step()
        out = [x.t.clone() for x in (c.master, c.m, c.v, c.w)], c.shard.state_dict()
        c.close()
        return out

    (a, sa), (b, sb) = run(None), run(4)
    assert sa == sb
    for x, y in zip(a, b):
        assert torch.equal(x.view(torch.uint8), y.view(torch.uint8))
    _, sr = run(4, exact_count=False)
    assert sr["loss_scale"] == 2 * sa["loss_scale"]   # the refilled count tolerated step 5's overflow
