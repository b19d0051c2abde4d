"""GPU parity: the CUDA step (through the C ABI) against the oracle on the
same seeded input bytes, element by element, at sizes the oracle finishes in
seconds that still span many blocks, a peeled head and a ragged tail."""
import ctypes

import numpy as np
import pytest
import torch

import synth
from mixed_precision_zero_b200 import (Hparams, NeoxError, NeoxShard, _abi, neox_shard_get_profile)
from synth import workloads as W
from tests.gpu_harness import Guarded, ShardCase, to_u16

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def _cuda():
    assert torch.cuda.is_available(), "GPU tests need a CUDA device"
    torch.cuda.set_device(0)
    yield
    torch.cuda.synchronize()


def test_philox_gpu_matches_cpu_twin():
    """The GPU generator draws the same Philox integers as its numpy twin."""
    raw = synth.gpu_philox_raw(1 << 16, 7, 1234, synth.STREAM_GRAD | (3 << 8))
    b = np.arange(1 << 16, dtype=np.uint64)
    cpu = synth.philox4x32(b & np.uint64(0xFFFFFFFF), b >> np.uint64(32), 7, 0, 1234, synth.STREAM_GRAD | (3 << 8))
    assert np.array_equal(raw, np.stack(cpu, axis=1))


def test_tiny_workload_full_trace():
    """The 1,048,576-element FP16 workload: 10 calls, an inf at a seeded index
    on call 4, window 2; every result field and every state element checked
    after every call, and the scale trajectory is the hand-derived one."""
    wl = W.tiny()
    hp = Hparams(wl.beta1, wl.beta2, wl.eps, wl.clip, wl.predivide, wl.init_scale, 2.0, 1.0, wl.scale_window)
    c = ShardCase(wl.numel, hp=hp, lr=wl.lr, default_wd=wl.weight_decay, seed=wl.seed)
    scales = []
    for s in range(1, wl.steps + 1):
        c.gen_normal(s, wl.grad_sigma)
        if s in wl.inject_steps:
            c.inject(s)
        res, info = c.step()
        c.check_result(res, info)
        assert bool(res.overflow) == (s in wl.inject_steps)
        c.check_state()
        scales.append(res.loss_scale_next)
    assert scales == [2.0 ** e for e in (16, 17, 17, 16, 16, 17, 17, 18, 18, 19)]
    assert c.orc.scaler.t == 9 and c.guards_intact()
    c.close()


@pytest.mark.parametrize("wbf16,gbf16", [(False, False), (True, True), (True, False), (False, True)])
def test_bit_exact_with_clipping_off(wbf16, gbf16):
    """Clip off: the coefficient is exactly 1 on both sides, so master, m, v and
    the 16-bit copy match the oracle bit for bit."""
    n = 300_007
    c = ShardCase(n, wbf16=wbf16, gbf16=gbf16, hp=Hparams(clip_norm=0.0, init_scale=2.0 ** 12), lr=1e-3)
    for s in range(1, 6):
        c.gen_normal(s, 3e-3)
        res, info = c.step()
        c.check_result(res, info)
        c.check_state(exact=True)
    assert c.guards_intact()
    c.close()


@pytest.mark.parametrize("n", [1, 2, 7, 8, 9, 15, 17, 4095, 4097, 65_541, 1_000_003])
@pytest.mark.parametrize("off", [0, 3, 5])
def test_sizes_and_common_offsets(n, off):
    """Ragged sizes at a common element offset (the vector path with a peeled head)."""
    c = ShardCase(n, hp=Hparams(init_scale=2.0 ** 10, scale_window=2), offsets={"all": off}, lr=1e-3)
    for s in range(1, 4):
        c.gen_normal(s, 5e-2)
        res, info = c.step()
        c.check_result(res, info)
        c.check_state()
    assert c.guards_intact()
    c.close()


@pytest.mark.parametrize("offsets", [
    {"g0": 1, "w": 0, "master": 0, "m": 0, "v": 0},
    {"g0": 0, "w": 2, "master": 1, "m": 3, "v": 0},
    {"g0": 4, "w": 4, "master": 0, "m": 0, "v": 0},   # 16-bit at 8 B, FP32 at 16 B: 4-wide vectors
    {"g0": 6, "w": 2, "master": 2, "m": 2, "v": 2},   # common residue mod 2 only
])
def test_mixed_residues_fall_back_to_narrow_vectors(offsets):
    n = 123_457
    c = ShardCase(n, hp=Hparams(clip_norm=0.0, init_scale=2.0 ** 10), offsets=offsets, lr=1e-3)
    for s in range(1, 4):
        c.gen_normal(s, 5e-2)
        res, info = c.step()
        c.check_result(res, info)
        c.check_state(exact=True)
    assert c.guards_intact()
    c.close()


@pytest.mark.parametrize("K,max_grads,pre", [(2, 1, 2.0), (3, 1, 1.0), (5, 8, 4.0), (8, 8, 8.0), (8, 1, 8.0)])
def test_multi_buffer_predivide(K, max_grads, pre):
    """K Student-t(3) x 2^10 buffers with pre-divide: the natural FP16
    overflows drive the scaler down; the FP32-sum scratch path (max_grads >= 5)
    and the re-read path agree with the oracle."""
    n = (1 << 20) + 5
    hp = Hparams(clip_norm=0.3, predivide=pre, init_scale=2.0 ** 10)
    c = ShardCase(n, K=K, hp=hp, max_grads=max_grads, offsets={"all": 1}, lr=6e-4)
    flags = []
    for s in range(1, 9):
        c.gen_t3(s)
        res, info = c.step()
        c.check_result(res, info)
        c.check_state()
        flags.append(res.overflow)
    assert c.guards_intact()
    c.close()


@pytest.mark.parametrize("K,off,bf16", [(1, 0, False), (1, 3, True), (3, 5, False)])
def test_accumulate_flag_bit_exact(K, off, bf16):
    """NEOX_SHARD_ACCUMULATE at any K: pass 1 writes the FP32 sum (in split
    tiles), pass 2 reads it.  Clip off: bit-exact with the oracle, through an
    overflow, on a shard with whole tiles, a partial tile and a peeled head."""
    n = 3_000_013
    hp = Hparams(clip_norm=0.0, predivide=float(K), init_scale=2.0 ** 12, scale_window=2)
    c = ShardCase(n, K=K, hp=hp, wbf16=bf16, gbf16=bf16, offsets={"all": off}, accumulate=True, lr=1e-3)
    for s in range(1, 6):
        c.gen_normal(s, 2e-3)
        if s == 3:
            c.inject(s, buffer=K - 1)
        res, info = c.step()
        c.check_result(res, info)
        assert res.overflow == (1 if s == 3 else 0)
        c.check_state(exact=True)
    assert c.guards_intact()
    c.close()


def test_pythia_shaped_segments_small():
    """A 2-layer, hidden-64 model with the Pythia layout: 26 segments, wd 0 on
    biases and LayerNorms, LayerNorm weights initialised to one."""
    segs = W.pythia_like_segments(layers=2, hidden=64, vocab=1000)
    n = segs[-1][0] + segs[-1][1]
    c = ShardCase(n, hp=Hparams(init_scale=2.0 ** 12), segments=[(o, k, w) for o, k, w, _ in segs],
                  seg_init=segs, lr=6e-4)
    for s in range(1, 6):
        c.gen_normal(s, 1e-4 * 300)
        res, info = c.step()
        c.check_result(res, info)
        c.check_state()
    c.close()


def test_segment_boundaries_inside_vectors():
    """Segments with odd lengths so that boundaries fall inside 8-element vectors."""
    sizes = [1, 2, 3, 5, 7, 11, 13, 8191, 17, 100_003, 9]
    segs, off = [], 0
    for i, k in enumerate(sizes):
        segs.append((off, k, 0.1 * (i % 3)))
        off += k
    c = ShardCase(off, hp=Hparams(clip_norm=0.0, init_scale=1.0), segments=segs, offsets={"all": 3}, lr=1e-2)
    for s in range(1, 4):
        c.gen_normal(s, 1e-2)
        res, info = c.step()
        c.check_result(res, info)
        c.check_state(exact=True)
    c.close()


@pytest.mark.parametrize("bad_kind", [0, 1, 2])
def test_overflow_leaves_every_state_byte(bad_kind):
    n = 500_001
    c = ShardCase(n, hp=Hparams(init_scale=2.0 ** 15, scale_window=3), lr=6e-4)
    c.gen_normal(1, 1e-3)
    c.step()
    before = [x.t.clone() for x in (c.master, c.m, c.v, c.w)]
    c.gen_normal(2, 1e-3)
    c.inject(2, count=bad_kind)
    res, info = c.step()
    c.check_result(res, info)
    assert res.overflow == 1 and res.loss_scale_next == 2.0 ** 14 and res.applied_steps == 1
    for a, x in zip(before, (c.master, c.m, c.v, c.w)):
        assert torch.equal(a.view(torch.uint8), x.t.view(torch.uint8))
    c.close()


def test_scaler_floor_and_repeated_overflow():
    n = 10_000
    c = ShardCase(n, hp=Hparams(init_scale=16.0, min_scale=1.0, scale_window=2), lr=1e-3)
    for s in range(1, 9):
        c.gen_normal(s, 1e-3)
        if s <= 6:
            c.inject(s, count=s)
        res, info = c.step()
        c.check_result(res, info)
    assert c.orc.scale == 2.0 and c.orc.scaler.t == 2
    c.check_state()
    c.close()


def test_checkpoint_resume_is_bit_identical():
    """N calls, save (state arrays + scaler state), destroy, re-create, set the
    state, M more calls == N + M uninterrupted calls, byte for byte."""
    n = 200_003
    hp = Hparams(init_scale=2.0 ** 12, scale_window=2)

    def run(split):
        c = ShardCase(n, hp=hp, lr=6e-4, seed=5)
        for s in range(1, 9):
            if s == split:
                saved = [x.t.clone() for x in (c.master, c.m, c.v, c.w)]
                st = c.shard.get_state()
                c.shard.close()
                for x, y in zip((c.master, c.m, c.v, c.w), saved):
                    x.t.copy_(y)
                c.shard = NeoxShard(c.master.t, c.m.t, c.v.t, hp, weight_decay=0.1)
                c.shard.set_state(*st)
            c.gen_normal(s, 1e-3)
            if s == 6:
                c.inject(s)
            c.step()
        out = [x.t.clone() for x in (c.master, c.m, c.v, c.w)], c.shard.get_state()
        c.close()
        return out

    (a, sa), (b, sb) = run(None), run(4)
    assert sa == sb
    for x, y in zip(a, b):
        assert torch.equal(x.view(torch.uint8), y.view(torch.uint8))


def test_deterministic_across_runs():
    outs = []
    for _ in range(2):
        c = ShardCase(777_777, K=3, hp=Hparams(predivide=2.0, init_scale=2.0 ** 8), lr=6e-4, seed=9)
        for s in range(1, 4):
            c.gen_normal(s, 2e-3)
            res, _ = c.step()
        outs.append(([x.t.clone() for x in (c.master, c.m, c.v, c.w)], res.grad_norm))
        c.close()
    assert outs[0][1] == outs[1][1]
    for x, y in zip(outs[0][0], outs[1][0]):
        assert torch.equal(x.view(torch.uint8), y.view(torch.uint8))


def test_empty_shard():
    z = torch.empty(0, dtype=torch.float32, device="cuda")
    sh = NeoxShard(z, z, z, Hparams(scale_window=1, init_scale=4.0))
    w = torch.empty(0, dtype=torch.float16, device="cuda")
    res = sh.step([w], w, 1e-3)
    assert res.overflow == 0 and res.grad_norm == 0.0 and res.applied_steps == 1 and res.loss_scale_next == 8.0
    sh.close()


def test_invalid_arguments_launch_nothing():
    n = 4096
    c = ShardCase(n, lr=1e-3)
    c.shard.set_profiling(True)
    launches0 = c.shard.profile().launches
    before = [x.t.clone() for x in (c.master, c.m, c.v, c.w)]
    L = _abi.lib()
    res = _abi.neox_step_result()
    gptr = c.g[0].t.data_ptr()

    def call(grads, k, params, lr):
        arr = (ctypes.c_void_p * max(1, len(grads)))(*grads) if grads is not None else None
        return L.neox_shard_step(c.shard.handle, arr, k, params, lr, None, ctypes.byref(res))

    assert call([gptr], 0, c.w.t.data_ptr(), 1e-3) == _abi.NEOX_ERR_INVALID_ARGUMENT
    assert call([gptr], 65, c.w.t.data_ptr(), 1e-3) == _abi.NEOX_ERR_INVALID_ARGUMENT
    assert call(None, 1, c.w.t.data_ptr(), 1e-3) == _abi.NEOX_ERR_INVALID_ARGUMENT
    assert call([None], 1, c.w.t.data_ptr(), 1e-3) == _abi.NEOX_ERR_INVALID_ARGUMENT
    assert call([gptr + 1], 1, c.w.t.data_ptr(), 1e-3) == _abi.NEOX_ERR_INVALID_ARGUMENT
    assert call([gptr], 1, c.w.t.data_ptr() + 1, 1e-3) == _abi.NEOX_ERR_INVALID_ARGUMENT
    assert call([gptr], 1, None, 1e-3) == _abi.NEOX_ERR_INVALID_ARGUMENT
    assert call([gptr], 1, c.w.t.data_ptr(), float("nan")) == _abi.NEOX_ERR_INVALID_ARGUMENT
    assert call([gptr], 1, c.w.t.data_ptr(), -1.0) == _abi.NEOX_ERR_INVALID_ARGUMENT
    assert L.neox_shard_step(c.shard.handle, (ctypes.c_void_p * 1)(gptr), 1, c.w.t.data_ptr(), 1e-3, None,
                             None) == _abi.NEOX_ERR_INVALID_ARGUMENT
    assert c.shard.profile().launches == launches0
    for a, x in zip(before, (c.master, c.m, c.v, c.w)):
        assert torch.equal(a.view(torch.uint8), x.t.view(torch.uint8))
    assert c.shard.get_state() == (65536.0, 0, 0)
    # create-time validation
    z = c.master.t
    with pytest.raises(NeoxError):
        NeoxShard(z, c.m.t, c.v.t, Hparams(beta1=1.0))
    with pytest.raises(NeoxError):
        NeoxShard(z, c.m.t, c.v.t, Hparams(scale_window=0))
    with pytest.raises(NeoxError):
        NeoxShard(z, c.m.t, c.v.t, segments=[(0, 100, 0.1), (200, n - 200, 0.1)])
    with pytest.raises(NeoxError):
        NeoxShard(z, c.m.t, c.v.t, segments=[(0, n - 1, 0.1)])
    with pytest.raises(NeoxError):
        c.shard.set_state(0.0, 0, 0)
    c.close()


def test_profile_counts_and_timing():
    c = ShardCase(1 << 20, lr=1e-3)
    c.shard.set_profiling(True)
    for s in range(1, 4):
        c.gen_normal(s, 1e-3)
        c.step()
    p = c.shard.profile()
    assert p.steps == 3 and p.launches == 6 and p.grad_pass_ms > 0 and p.update_pass_ms > 0
    c.close()


def test_state_accounting_and_scratch():
    c = ShardCase(1000, lr=1e-3)
    assert _abi.neox_model_state_bytes(1000) == 16_000
    assert _abi.neox_model_state_bytes(175_000_000_000) == 2_800_000_000_000
    assert 0 < c.shard.scratch_bytes() < 1 << 20
    c.close()


def test_huge_finite_gradients_are_not_overflow():
    """FP16 gradients of about 1e4 carried at loss scale 2^-60 (floor 0): the
    unscaled values (about 1e22) are finite although their squares pass FP32's
    range.  No overflow, and the norm matches the oracle's double sum."""
    n = 4099
    c = ShardCase(n, hp=Hparams(clip_norm=1.0, init_scale=2.0 ** -60, min_scale=0.0, scale_window=1000),
                  offsets={"all": 1}, lr=1e-3)
    for s in range(1, 3):
        synth.gpu_grad_normal16(c.g[0].t, 1e4, 1.0, c.seed, 0, s)
        res, info = c.step()
        assert info.overflow == 0 and res.overflow == 0 and info.norm > 1e22
        c.check_result(res, info)
        c.check_state()
    c.close()


@pytest.mark.parametrize("max_grads", [64, 1])
def test_maximum_buffer_count(max_grads):
    """K = 64 gradient buffers (the largest the ABI takes), pre-divide 64,
    through the FP32-sum path and the re-read path."""
    n = 70_001
    hp = Hparams(clip_norm=1.0, predivide=64.0, init_scale=2.0 ** 8)
    c = ShardCase(n, K=64, hp=hp, max_grads=max_grads, offsets={"all": 2}, lr=6e-4)
    for s in range(1, 4):
        c.gen_normal(s, 1e-3)
        res, info = c.step()
        c.check_result(res, info)
        c.check_state()
    assert c.guards_intact()
    c.close()


@pytest.mark.parametrize("offsets", [[0, 0, 0], [3, 3, 3], [1, 2, 0]])
def test_weight_copies_receive_the_cast(offsets):
    """Pass 2 writes the updated 16-bit weights into every registered copy
    (the all-gather destinations of the other ranks, here local buffers at
    chosen element offsets), byte-identical to params, and leaves them alone
    on a skipped step."""
    n = 250_003
    c = ShardCase(n, hp=Hparams(init_scale=2.0 ** 12, scale_window=3), offsets={"all": offsets[0]}, lr=1e-3)
    copies = [Guarded(n, torch.float16, o) for o in offsets]
    for x in copies:
        x.t.fill_(0.0)
    c.shard.set_weight_copies([x.t for x in copies])
    for s in range(1, 5):
        c.gen_normal(s, 1e-3)
        if s == 3:
            c.inject(s)
            before = [x.t.clone() for x in copies]
        res, info = c.step()
        c.check_result(res, info)
        c.check_state()
        for j, x in enumerate(copies):
            if s == 3:
                assert torch.equal(x.t.view(torch.int16), before[j].view(torch.int16))
            else:
                assert torch.equal(x.t.view(torch.int16), c.w.t.view(torch.int16))
            assert x.guards_intact()
    c.shard.set_weight_copies([])
    c.close()


@pytest.mark.parametrize("K,max_grads,offset", [(1, 1, 0), (6, 8, 5), (2, 2, 3)])
def test_chunked_update_bit_exact(K, max_grads, offset):
    """A shard of more than one pass-2 chunk per block, so the AdamW pass takes
    its work from the chunk counter (through the FP32 sum for K = 6): the
    state equals the oracle byte for byte with clipping off, through an
    overflowed step, segment boundaries, the peeled head and the ragged tail."""
    torch.cuda.set_device(0)
    n = 8_000_011
    segs = [(0, 1_000_003, 0.1), (1_000_003, 4_097, 0.0), (1_004_100, n - 1_004_100, 0.1)]
    c = ShardCase(n, K=K, max_grads=max_grads, offsets={"all": offset}, segments=segs, seed=61, lr=1e-3,
                  hp=Hparams(clip_norm=0.0, predivide=float(K), init_scale=2.0 ** 12, scale_window=2))
    for s in range(1, 5):
        c.gen_normal(s, 2e-3)
        if s == 3:
            c.inject(s, buffer=K - 1)
        res, info = c.step()
        c.check_result(res, info)
        assert res.overflow == (1 if s == 3 else 0)
    c.check_state(exact=True)
    assert c.guards_intact()
    c.close()
