"""The allocation-free step against the handle-based step and the oracle.

neox_shard_step_noalloc serves callers that may not allocate device memory
(code inside an allocator's own hook, runtimes that own all device memory,
loops where cudaMalloc would synchronise the device).  It runs the same
kernels as neox_shard_step on the same vector layout, so on the same inputs
its results must equal the handle step's bit for bit, and (with clipping off,
where the clip coefficient is exactly 1 on both sides) the oracle's.  Its
first call on a device does the set-up: the address of the static scratch and
the loading of every kernel instance it can launch; after that no call, of
any dtype, buffer count or update rule, takes device memory.

This file sorts last so that a run stopping at its first failure has run
every other test already; it also passes alone in a fresh process.
"""
import ctypes

import numpy as np
import pytest
import torch

import oracle
import synth
from mixed_precision_zero_b200 import Hparams, NeoxError, NeoxShard, _abi
from tests.gpu_harness import oracle_hparams, to_u16

pytestmark = pytest.mark.gpu


def _segments(n):
    cuts = [0, 1000, 1003, 50_001, 50_002, 200_000, n]
    return [(a, b - a, 0.1 if i % 2 == 0 else 0.0) for i, (a, b) in enumerate(zip(cuts, cuts[1:]))]


def _aligned(n, dtype):
    """A CUDA tensor of n elements starting on a 1024-byte boundary, so that two
    shards built from such tensors get the same vector layout (head peel) and
    hence the same norm reduction order."""
    esz = torch.empty(0, dtype=dtype).element_size()
    base = torch.empty(n + 1024 // esz, dtype=dtype, device="cuda")
    off = (-base.data_ptr() % 1024) // esz
    return base.narrow(0, off, n)


def _shard_arrays(n, seed, wdtype=torch.float16):
    master = _aligned(n, torch.float32)
    synth.gpu_master_normal(master, 0.02, seed)
    m, v, w = _aligned(n, torch.float32).zero_(), _aligned(n, torch.float32).zero_(), _aligned(n, wdtype)
    w.copy_(master.to(wdtype))
    return [master, m, v, w]


def _clone(arrs):
    out = []
    for x in arrs:
        y = _aligned(x.numel(), x.dtype)
        y.copy_(x)
        out.append(y)
    return out


def _desc(n, arrs, segs=None, wdtype=_abi.NEOX_FP16, gdtype=_abi.NEOX_FP16, wd=0.0):
    seg_arr = None
    if segs:
        seg_arr = (_abi.neox_segment * len(segs))(*[_abi.neox_segment(o, c, w) for o, c, w in segs])
    d = _abi.neox_shard_desc(n, wdtype, gdtype,
                             ctypes.cast(seg_arr, ctypes.POINTER(_abi.neox_segment)) if segs else None,
                             len(segs) if segs else 0, wd, arrs[0].data_ptr(), arrs[1].data_ptr(),
                             arrs[2].data_ptr(), 1)
    d._keep = seg_arr
    return d


def _bytes_equal(a, b):
    for x, y in zip(a, b):
        assert torch.equal(x.view(torch.uint8), y.view(torch.uint8))


def test_noalloc_matches_handle_step_on_two_calls():
    """Clip on: the allocation-free step equals the handle step bit for bit,
    and the second call (after the first call's set-up) takes no device memory."""
    assert torch.cuda.is_available()
    torch.cuda.set_device(0)
    n, lr, seed = 300_007, 6e-4, 3
    hp = Hparams(clip_norm=1.0, init_scale=2.0 ** 16, scale_window=1000)
    segs = _segments(n)
    a = _shard_arrays(n, seed)                 # handle-based step
    b = _clone(a)                              # allocation-free step, same starting bytes
    grads = [_aligned(n, torch.float16) for _ in range(2)]
    for k, g in enumerate(grads):
        synth.gpu_grad_normal16(g, 1e-3, hp.init_scale, seed, 0, k + 1)

    shard = NeoxShard(a[0], a[1], a[2], hp, segments=segs)
    desc = _desc(n, b, segs)
    state = _abi.neox_scaler_state(hp.init_scale, 0, 0)
    stream = torch.cuda.current_stream().cuda_stream
    torch.cuda.synchronize()

    for call in range(2):
        free_before = torch.cuda.mem_get_info()[0]
        r_b = _abi.neox_shard_step_noalloc(desc, hp.c(), state, [grads[call].data_ptr()], b[3].data_ptr(), lr,
                                           stream)
        free_after = torch.cuda.mem_get_info()[0]
        if call == 1:  # after the set-up of the first call: no device memory taken
            assert free_after == free_before
        r_a = shard.step([grads[call]], a[3], lr)
        assert r_b.as_dict() == r_a.as_dict()
        assert r_b.overflow == 0 and r_b.applied_steps == call + 1
        assert (state.scale, state.good, state.t) == shard.get_state()
        _bytes_equal(a, b)
    shard.close()


def test_noalloc_first_bf16_and_sgd_calls_take_no_device_memory():
    """The set-up loads every kernel instance the step can launch, so a first
    BF16 call (K = 8, the re-read path) and a first SGD call, after any earlier
    call, leave the device's free memory unchanged."""
    torch.cuda.set_device(0)
    n, K = 100_003, 8
    bf = _shard_arrays(n, 11, torch.bfloat16)
    gb = [_aligned(n, torch.bfloat16) for _ in range(K)]
    for k, g in enumerate(gb):
        synth.gpu_grad_normal16(g, 1e-3, 2.0 ** 8, 11, k, 1, True)
    fp = _shard_arrays(n, 12)
    gf = _aligned(n, torch.float16)
    synth.gpu_grad_normal16(gf, 1e-3, 2.0 ** 8, 12, 0, 1)
    stream = torch.cuda.current_stream().cuda_stream
    # any earlier call does the set-up (in a fresh process, this one)
    st0 = _abi.neox_scaler_state(2.0 ** 8, 0, 0)
    _abi.neox_shard_step_noalloc(_desc(n, fp, wd=0.1), Hparams(init_scale=2.0 ** 8).c(), st0, [gf.data_ptr()],
                                 fp[3].data_ptr(), 1e-3, stream)
    torch.cuda.synchronize()

    free0 = torch.cuda.mem_get_info()[0]
    st1 = _abi.neox_scaler_state(2.0 ** 8, 0, 0)
    r1 = _abi.neox_shard_step_noalloc(_desc(n, bf, wdtype=_abi.NEOX_BF16, gdtype=_abi.NEOX_BF16, wd=0.1),
                                      Hparams(init_scale=2.0 ** 8, predivide=8.0).c(), st1,
                                      [g.data_ptr() for g in gb], bf[3].data_ptr(), 1e-3, stream)
    free1 = torch.cuda.mem_get_info()[0]
    st2 = _abi.neox_scaler_state(2.0 ** 8, 0, 0)
    r2 = _abi.neox_shard_step_noalloc(_desc(n, fp, wd=0.1), Hparams(init_scale=2.0 ** 8, optimizer="sgd").c(), st2,
                                      [gf.data_ptr()], fp[3].data_ptr(), 1e-3, stream)
    free2 = torch.cuda.mem_get_info()[0]
    assert free1 == free0 and free2 == free0
    assert r1.overflow == 0 and r1.applied_steps == 1 and r2.overflow == 0 and r2.applied_steps == 1


@pytest.mark.parametrize("bf16,K", [(False, 1), (True, 8)])
def test_noalloc_overflow_then_applied_bit_exact(bf16, K):
    """Clip off, a seeded inf on call 2: every call equals the handle step and
    the oracle bit for bit (flag, norm, scale, counters, the scaler state the
    caller holds, master, m, v and the 16-bit copy); on the overflowed call the
    shard's bytes are unchanged and the scale halves.  K = 8 BF16 buffers with
    predivide 8 take the path that re-reads the buffers in pass 2."""
    torch.cuda.set_device(0)
    n, lr, seed = 200_003, 1e-3, 21
    wt = torch.bfloat16 if bf16 else torch.float16
    code = _abi.NEOX_BF16 if bf16 else _abi.NEOX_FP16
    segs = _segments(n)
    hp = Hparams(clip_norm=0.0, init_scale=2.0 ** 10, scale_window=2, predivide=float(K))
    a = _shard_arrays(n, seed, wt)
    b = _clone(a)
    grads = [_aligned(n, wt) for _ in range(K)]
    shard = NeoxShard(a[0], a[1], a[2], hp, wdtype=wt, gdtype=wt, segments=segs, max_grads=1)
    orc = oracle.OracleShard(a[0].cpu().numpy(), oracle_hparams(hp), wbf16=bf16, gbf16=bf16, segments=segs)
    desc = _desc(n, b, segs, wdtype=code, gdtype=code)
    state = _abi.neox_scaler_state(hp.init_scale, 0, 0)
    stream = torch.cuda.current_stream().cuda_stream
    for s in range(1, 5):
        for k, g in enumerate(grads):
            synth.gpu_grad_normal16(g, 1e-3, orc.scale, seed, k, s, bf16)
        if s == 2:
            grads[K - 1].view(torch.int16)[77_777] = 0x7F80 if bf16 else 0x7C00
        torch.cuda.synchronize()
        host = [to_u16(g) for g in grads]
        before = [x.clone() for x in b]
        rb = _abi.neox_shard_step_noalloc(desc, hp.c(), state, [g.data_ptr() for g in grads], b[3].data_ptr(), lr,
                                          stream)
        ra = shard.step(grads, a[3], lr)
        info = orc.step(host, lr)
        assert rb.as_dict() == ra.as_dict()
        assert rb.overflow == info.overflow == (1 if s == 2 else 0)
        assert rb.loss_scale == info.scale_used and rb.loss_scale_next == info.scale_next
        assert (state.scale, state.good, state.t) == (info.scale_next, orc.scaler.good, info.t)
        assert (state.scale, state.good, state.t) == shard.get_state()
        if info.overflow:
            assert np.isinf(rb.grad_norm) and rb.clip_coef == 0.0
            _bytes_equal(before, b)
        else:
            assert rb.grad_norm == np.float32(info.norm) or abs(rb.grad_norm - info.norm) <= 1e-5 * info.norm
        _bytes_equal(a, b)
        assert b[0].cpu().numpy().tobytes() == orc.master.tobytes()
        assert b[1].cpu().numpy().tobytes() == orc.m.tobytes()
        assert b[2].cpu().numpy().tobytes() == orc.v.tobytes()
        assert np.array_equal(to_u16(b[3]), orc.w)
    assert state.scale == 2.0 ** 10 and state.t == 3   # 2^10 -> 2^9 (call 2) -> 2^10 (calls 3 and 4)
    shard.close()


def test_noalloc_rejects_segment_table_beyond_its_maximum():
    torch.cuda.set_device(0)
    nseg = 1025
    n = nseg * 4
    arrs = _shard_arrays(n, 1)
    segs = [(4 * i, 4, 0.1) for i in range(nseg)]
    g = torch.zeros(n, dtype=torch.float16, device="cuda")
    state = _abi.neox_scaler_state(1.0, 0, 0)
    before = arrs[0].clone()
    with pytest.raises(NeoxError) as ei:
        _abi.neox_shard_step_noalloc(_desc(n, arrs, segs), Hparams().c(), state, [g.data_ptr()], arrs[3].data_ptr(),
                                     1e-3, 0)
    assert ei.value.status == _abi.NEOX_ERR_INVALID_ARGUMENT and "1024" in str(ei.value)
    assert torch.equal(before, arrs[0]) and (state.scale, state.good, state.t) == (1.0, 0, 0)
