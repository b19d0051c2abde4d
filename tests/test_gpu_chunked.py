"""The entry points on shards large enough that the AdamW pass takes its work
in chunks from the counter in the scalar block (more than 2 x 256 vectors per
block of its grid).  Each entry point resets or uses that counter its own way:
the split step (statistics pass, then the decision kernel), the asynchronous
step replayed from a CUDA graph and the weight copies (their own kernel
instance).  The fused flat step, itself bit-exact with the oracle at this
size, is the reference.  (The allocation-free step at this size is tested
with the other allocation-free tests, which run last.)"""
import ctypes

import pytest
import torch

import synth
from mixed_precision_zero_b200 import Hparams, NeoxShard, _abi
from tests.gpu_harness import check_close, check_ulp16, to_u16

pytestmark = pytest.mark.gpu

N = 8_000_011
SEGS = [(0, 1_000_003, 0.1), (1_000_003, 4_097, 0.0), (1_004_100, N - 1_004_100, 0.1)]


def _state(seed):
    master = torch.empty(N, dtype=torch.float32, device="cuda")
    synth.gpu_master_normal(master, 0.02, seed)
    return [master, torch.zeros_like(master), torch.zeros_like(master), master.to(torch.float16)]


def _grads(g, s, scale, seed):
    synth.gpu_grad_normal16(g, 2e-3, scale, seed, 0, s)
    if s == 3:
        g.view(torch.int16)[4_000_000] = 0x7C00


def _equal(a, b):
    for x, y in zip(a, b):
        assert torch.equal(x.view(torch.uint8), y.view(torch.uint8))


def test_split_step_equals_fused_when_chunked():
    torch.cuda.set_device(0)
    hp = Hparams(clip_norm=1.0, init_scale=2.0 ** 12, scale_window=2)
    a, b = _state(71), _state(71)
    fused = NeoxShard(a[0], a[1], a[2], hp, segments=SEGS)
    split = NeoxShard(b[0], b[1], b[2], hp, segments=SEGS)
    g = torch.empty(N, dtype=torch.float16, device="cuda")
    stats = torch.zeros(2, dtype=torch.float64, device="cuda")
    for s in range(1, 6):
        _grads(g, s, fused.get_state()[0], 71)
        ra = fused.step([g], a[3], 1e-3)
        split.grad_stats([g], b[3], stats)
        rb = split.apply([g], b[3], 1e-3, stats)
        assert ra.as_dict() == rb.as_dict()
    _equal(a, b)
    fused.close()
    split.close()


def test_graph_replayed_async_step_tracks_sync_when_chunked():
    torch.cuda.set_device(0)
    hp = Hparams(clip_norm=1.0, init_scale=2.0 ** 12, scale_window=2)
    a, b = _state(72), _state(72)
    sync = NeoxShard(a[0], a[1], a[2], hp, segments=SEGS)
    asy = NeoxShard(b[0], b[1], b[2], hp, segments=SEGS)
    g = torch.empty(N, dtype=torch.float16, device="cuda")
    res_dev = torch.zeros(64, dtype=torch.uint8, device="cuda")
    lr_dev = torch.full((1,), 1e-3, dtype=torch.float32, device="cuda")
    _grads(g, 1, 2.0 ** 12, 72)
    sync.step([g], a[3], 1e-3)
    asy.step_async([g], b[3], result=res_dev, lr_device=lr_dev)   # set-up outside the capture
    torch.cuda.synchronize()
    graph = torch.cuda.CUDAGraph()
    side = torch.cuda.Stream()
    side.wait_stream(torch.cuda.current_stream())
    with torch.cuda.stream(side), torch.cuda.graph(graph, stream=side):
        asy.step_async([g], b[3], result=res_dev, lr_device=lr_dev)
    torch.cuda.synchronize()
    for s in range(2, 7):
        _grads(g, s, sync.get_state()[0], 72)
        ra = sync.step([g], a[3], 1e-3)
        graph.replay()
        torch.cuda.synchronize()
        rb = _abi.neox_step_result.from_buffer_copy(res_dev.cpu().numpy().tobytes()[:ctypes.sizeof(_abi.neox_step_result)])
        assert (ra.overflow, ra.loss_scale_next, ra.applied_steps) == (rb.overflow, rb.loss_scale_next, rb.applied_steps)
    del graph
    for name, x, y in (("master", b[0], a[0]), ("m", b[1], a[1]), ("v", b[2], a[2])):
        check_close(name, x.cpu().numpy(), y.cpu().numpy())
    check_ulp16(to_u16(b[3]), to_u16(a[3]))
    sync.close()
    asy.close()


def test_weight_copies_when_chunked():
    torch.cuda.set_device(0)
    hp = Hparams(clip_norm=1.0, init_scale=2.0 ** 12, scale_window=2)
    a, b = _state(73), _state(73)
    plain = NeoxShard(a[0], a[1], a[2], hp, segments=SEGS)
    copied = NeoxShard(b[0], b[1], b[2], hp, segments=SEGS)
    dsts = [torch.zeros(N + 3, dtype=torch.float16, device="cuda")[3:], torch.zeros(N, dtype=torch.float16, device="cuda")]
    copied.set_weight_copies(dsts)
    g = torch.empty(N, dtype=torch.float16, device="cuda")
    for s in range(1, 5):
        _grads(g, s, plain.get_state()[0], 73)
        plain.step([g], a[3], 1e-3)
        copied.step([g], b[3], 1e-3)
        for d in dsts:
            assert torch.equal(d.view(torch.int16), b[3].view(torch.int16))
    _equal(a, b)
    plain.close()
    copied.close()
