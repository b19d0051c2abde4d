"""The asynchronous step (no host synchronisation, result written by the GPU)
against the synchronous step, directly and captured in a CUDA graph."""
import ctypes

import numpy as np
import pytest
import torch

import synth
from mixed_precision_zero_b200 import Hparams, NeoxShard, _abi
from tests.gpu_harness import check_close, check_ulp16, to_u16

pytestmark = pytest.mark.gpu


def _pair(n, seed, hp, segments=None):
    master = torch.empty(n, dtype=torch.float32, device="cuda")
    synth.gpu_master_normal(master, 0.02, seed)
    a = [master, torch.zeros_like(master), torch.zeros_like(master), master.to(torch.float16)]
    b = [x.clone() for x in a]
    sa = NeoxShard(a[0], a[1], a[2], hp, segments=segments, weight_decay=0.1)
    sb = NeoxShard(b[0], b[1], b[2], hp, segments=segments, weight_decay=0.1)
    return a, b, sa, sb


def _read_result(buf: torch.Tensor) -> _abi.neox_step_result:
    raw = buf.cpu().numpy().tobytes()
    return _abi.neox_step_result.from_buffer_copy(raw[:ctypes.sizeof(_abi.neox_step_result)])


def _same_result(ra, rb):
    assert ra.overflow == rb.overflow and ra.loss_scale == rb.loss_scale
    assert ra.loss_scale_next == rb.loss_scale_next and ra.applied_steps == rb.applied_steps
    assert ra.good_steps == rb.good_steps
    if not ra.overflow:
        assert abs(ra.grad_norm - rb.grad_norm) <= 1e-5 * ra.grad_norm
        assert abs(ra.clip_coef - rb.clip_coef) <= 1e-5 * ra.clip_coef


def _same_state(a, b):
    for name, x, y in (("master", b[0], a[0]), ("m", b[1], a[1]), ("v", b[2], a[2])):
        check_close(name, x.cpu().numpy(), y.cpu().numpy())
    check_ulp16(to_u16(b[3]), to_u16(a[3]))


def test_async_matches_sync_with_device_lr_and_overflow():
    torch.cuda.set_device(0)
    n = 500_009
    hp = Hparams(clip_norm=1.0, init_scale=2.0 ** 14, scale_window=3)
    a, b, sa, sb = _pair(n, 11, hp, segments=[(0, 1000, 0.0), (1000, n - 1000, 0.1)])
    g = torch.empty(n, dtype=torch.float16, device="cuda")
    lr_dev = torch.empty(1, dtype=torch.float32, device="cuda")
    res_dev = torch.zeros(64, dtype=torch.uint8, device="cuda")
    for s in range(1, 9):
        lr = 6e-4 * (1.0 - 0.05 * s)
        synth.gpu_grad_normal16(g, 1e-3, sa.get_state()[0], 11, 0, s)
        if s == 3:
            g.view(torch.int16)[12345] = 0x7C00
        lr_dev.fill_(lr)
        ra = sa.step([g], a[3], lr)
        sb.step_async([g], b[3], result=res_dev, lr_device=lr_dev)
        torch.cuda.synchronize()
        rb = _read_result(res_dev)
        _same_result(ra, rb)
        assert rb.overflow == (1 if s == 3 else 0)
    assert sb.get_state() == sa.get_state()   # the mirror is refreshed from the device
    _same_state(a, b)
    # a synchronous step after asynchronous ones picks the device state up
    synth.gpu_grad_normal16(g, 1e-3, sa.get_state()[0], 11, 0, 9)
    _same_result(sa.step([g], a[3], 5e-4), sb.step([g], b[3], 5e-4))
    _same_state(a, b)
    sa.close()
    sb.close()


def test_async_step_in_cuda_graph():
    """One asynchronous step captured in a CUDA graph and replayed, with the
    gradients and the learning rate refreshed between replays, tracks the
    synchronous step (including an overflowed replay)."""
    torch.cuda.set_device(0)
    n = 1 << 20
    hp = Hparams(clip_norm=1.0, init_scale=2.0 ** 16, scale_window=2)
    a, b, sa, sb = _pair(n, 12, hp)
    g = torch.empty(n, dtype=torch.float16, device="cuda")
    lr_dev = torch.full((1,), 6e-4, dtype=torch.float32, device="cuda")
    res_dev = torch.zeros(64, dtype=torch.uint8, device="cuda")
    # step 1 outside any capture on both sides (sets the handle up)
    synth.gpu_grad_normal16(g, 1e-3, hp.init_scale, 12, 0, 1)
    sa.step([g], a[3], 6e-4)
    sb.step_async([g], b[3], result=res_dev, lr_device=lr_dev)
    torch.cuda.synchronize()
    graph = torch.cuda.CUDAGraph()
    side = torch.cuda.Stream()
    side.wait_stream(torch.cuda.current_stream())
    with torch.cuda.stream(side):
        with torch.cuda.graph(graph, stream=side):
            sb.step_async([g], b[3], result=res_dev, lr_device=lr_dev)
    torch.cuda.synchronize()
    for s in range(2, 10):
        lr = 6e-4 * 0.9 ** s
        synth.gpu_grad_normal16(g, 1e-3, sa.get_state()[0], 12, 0, s)
        if s == 5:
            g.view(torch.int16)[777] = 0x7E00  # NaN
        lr_dev.fill_(lr)
        torch.cuda.synchronize()
        graph.replay()
        torch.cuda.synchronize()
        rb = _read_result(res_dev)
        ra = sa.step([g], a[3], lr)
        _same_result(ra, rb)
        # replays run outside the library: its state read must still see them
        assert sb.get_state() == (rb.loss_scale_next, rb.good_steps, rb.applied_steps)
    assert sb.get_state() == sa.get_state()
    _same_state(a, b)
    del graph
    sa.close()
    sb.close()
