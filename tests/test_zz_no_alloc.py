"""The allocation-free step against the handle-based step.

neox_shard_step_noalloc serves callers that may not allocate device memory
(code inside an allocator's own hook, runtimes that own all device memory,
loops where cudaMalloc would synchronise the device).  It must give what
neox_shard_step gives on the same inputs.  This file sorts last so that a run
stopping at its first failure has run every other test already; it also
passes alone in a fresh process (the first call sets the device up).
"""
import ctypes

import numpy as np
import pytest
import torch

import synth
from mixed_precision_zero_b200 import Hparams, NeoxError, NeoxShard, _abi
from tests.gpu_harness import check_close, check_ulp16, to_u16

pytestmark = pytest.mark.gpu


def _segments(n):
    cuts = [0, 1000, 1003, 50_001, 50_002, 200_000, n]
    return [(a, b - a, 0.1 if i % 2 == 0 else 0.0) for i, (a, b) in enumerate(zip(cuts, cuts[1:]))]


def _shard_arrays(n, seed):
    master = torch.empty(n, dtype=torch.float32, device="cuda")
    synth.gpu_master_normal(master, 0.02, seed)
    return master, torch.zeros_like(master), torch.zeros_like(master), master.to(torch.float16)


def test_noalloc_matches_handle_step_on_two_calls():
    assert torch.cuda.is_available()
    torch.cuda.set_device(0)
    n, lr, seed = 300_007, 6e-4, 3
    hp = Hparams(clip_norm=1.0, init_scale=2.0 ** 16, scale_window=1000)
    segs = _segments(n)
    a = _shard_arrays(n, seed)                 # handle-based step
    b = [x.clone() for x in a]                 # allocation-free step, same starting bytes
    grads = [torch.empty(n, dtype=torch.float16, device="cuda") for _ in range(2)]
    for k, g in enumerate(grads):
        synth.gpu_grad_normal16(g, 1e-3, hp.init_scale, seed, 0, k + 1)

    shard = NeoxShard(a[0], a[1], a[2], hp, segments=segs)
    seg_arr = (_abi.neox_segment * len(segs))(*[_abi.neox_segment(o, c, w) for o, c, w in segs])
    desc = _abi.neox_shard_desc(n, _abi.NEOX_FP16, _abi.NEOX_FP16,
                                ctypes.cast(seg_arr, ctypes.POINTER(_abi.neox_segment)), len(segs), 0.0,
                                b[0].data_ptr(), b[1].data_ptr(), b[2].data_ptr(), 1)
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
        assert r_b.overflow == r_a.overflow == 0
        assert r_b.loss_scale == r_a.loss_scale and r_b.loss_scale_next == r_a.loss_scale_next
        assert r_b.applied_steps == r_a.applied_steps == call + 1 and r_b.good_steps == r_a.good_steps
        assert abs(r_b.grad_norm - r_a.grad_norm) <= 1e-5 * r_a.grad_norm
        assert abs(r_b.clip_coef - r_a.clip_coef) <= 1e-5 * r_a.clip_coef
        assert (state.scale, state.good, state.t) == shard.get_state()
        for name, x, y in (("master", b[0], a[0]), ("exp_avg", b[1], a[1]), ("exp_avg_sq", b[2], a[2])):
            check_close(name, x.cpu().numpy(), y.cpu().numpy())
        check_ulp16(to_u16(b[3]), to_u16(a[3]))
    shard.close()


def test_noalloc_rejects_segment_table_beyond_its_maximum():
    torch.cuda.set_device(0)
    nseg = 1025
    n = nseg * 4
    m, e1, e2, w = _shard_arrays(n, 1)
    seg_arr = (_abi.neox_segment * nseg)(*[_abi.neox_segment(4 * i, 4, 0.1) for i in range(nseg)])
    desc = _abi.neox_shard_desc(n, _abi.NEOX_FP16, _abi.NEOX_FP16,
                                ctypes.cast(seg_arr, ctypes.POINTER(_abi.neox_segment)), nseg, 0.0,
                                m.data_ptr(), e1.data_ptr(), e2.data_ptr(), 1)
    g = torch.zeros(n, dtype=torch.float16, device="cuda")
    state = _abi.neox_scaler_state(1.0, 0, 0)
    before = m.clone()
    with pytest.raises(NeoxError) as ei:
        _abi.neox_shard_step_noalloc(desc, Hparams().c(), state, [g.data_ptr()], w.data_ptr(), 1e-3, 0)
    assert ei.value.status == _abi.NEOX_ERR_INVALID_ARGUMENT and "1024" in str(ei.value)
    assert torch.equal(before, m) and (state.scale, state.good, state.t) == (1.0, 0, 0)
