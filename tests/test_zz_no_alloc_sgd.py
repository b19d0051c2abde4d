"""The allocation-free step with the SGD update, against the oracle; its
refusal of a hysteresis it cannot carry (its scaler state has no count); and
the step on a shard large enough that the AdamW pass takes chunks from the
counter in the static scratch.  Sorts after the first allocation-free test
file, which checks the first call's device set-up."""
import ctypes

import pytest
import torch

import oracle
import synth
from mixed_precision_zero_b200 import Hparams, NeoxError, NeoxShard, _abi
from tests.gpu_harness import oracle_hparams, to_u16
from tests.test_gpu_chunked import N, SEGS, _equal, _grads, _state

pytestmark = pytest.mark.gpu


def _desc(n, master, m, v):
    return _abi.neox_shard_desc(n, _abi.NEOX_FP16, _abi.NEOX_FP16, None, 0, 0.1, master.data_ptr(), m.data_ptr(),
                                v.data_ptr(), 1)


def test_noalloc_sgd_matches_oracle():
    torch.cuda.set_device(0)
    n, seed = 200_003, 5
    hp = Hparams(clip_norm=0.0, init_scale=2.0 ** 12, scale_window=2, optimizer="sgd")
    master = torch.empty(n, dtype=torch.float32, device="cuda")
    synth.gpu_master_normal(master, 0.02, seed)
    m, v = torch.zeros_like(master), torch.zeros_like(master)
    w = master.to(torch.float16)
    g = torch.empty(n, dtype=torch.float16, device="cuda")
    orc = oracle.OracleShard(master.cpu().numpy(), oracle_hparams(hp), default_wd=0.1)
    desc = _desc(n, master, m, v)
    state = _abi.neox_scaler_state(hp.init_scale, 0, 0)
    stream = torch.cuda.current_stream().cuda_stream
    for s in range(1, 6):
        synth.gpu_grad_normal16(g, 1e-3, orc.scale, seed, 0, s)
        if s == 2:
            g.view(torch.int16)[99] = 0x7C00
        torch.cuda.synchronize()
        host = [to_u16(g)]
        r = _abi.neox_shard_step_noalloc(desc, hp.c(), state, [g.data_ptr()], w.data_ptr(), 2e-2, stream)
        info = orc.step(host, 2e-2)
        assert r.overflow == info.overflow and r.loss_scale_next == info.scale_next and r.applied_steps == info.t
    assert master.cpu().numpy().tobytes() == orc.master.tobytes()
    assert (to_u16(w) == orc.w).all()
    assert not m.any().item() and not v.any().item()


def test_noalloc_rejects_hysteresis():
    torch.cuda.set_device(0)
    n = 1000
    master = torch.zeros(n, dtype=torch.float32, device="cuda")
    m, v = torch.zeros_like(master), torch.zeros_like(master)
    w = torch.zeros(n, dtype=torch.float16, device="cuda")
    g = torch.zeros(n, dtype=torch.float16, device="cuda")
    state = _abi.neox_scaler_state(1024.0, 0, 0)
    with pytest.raises(NeoxError) as ei:
        _abi.neox_shard_step_noalloc(_desc(n, master, m, v), Hparams(hysteresis=2).c(), state, [g.data_ptr()],
                                     w.data_ptr(), 1e-3, torch.cuda.current_stream().cuda_stream)
    assert ei.value.status == _abi.NEOX_ERR_INVALID_ARGUMENT and "hysteresis" in str(ei.value)
    assert (state.scale, state.good, state.t) == (1024.0, 0, 0)


def test_noalloc_step_equals_handle_when_chunked():
    torch.cuda.set_device(0)
    hp = Hparams(clip_norm=1.0, init_scale=2.0 ** 12, scale_window=2)
    a, b = _state(74), _state(74)
    shard = NeoxShard(a[0], a[1], a[2], hp, segments=SEGS)
    seg_arr = (_abi.neox_segment * len(SEGS))(*[_abi.neox_segment(o, c, w) for o, c, w in SEGS])
    desc = _abi.neox_shard_desc(N, _abi.NEOX_FP16, _abi.NEOX_FP16, ctypes.cast(seg_arr, ctypes.POINTER(_abi.neox_segment)),
                                len(SEGS), 0.0, b[0].data_ptr(), b[1].data_ptr(), b[2].data_ptr(), 1)
    state = _abi.neox_scaler_state(hp.init_scale, 0, 0)
    g = torch.empty(N, dtype=torch.float16, device="cuda")
    stream = torch.cuda.current_stream().cuda_stream
    for s in range(1, 5):
        _grads(g, s, shard.get_state()[0], 74)
        ra = shard.step([g], a[3], 1e-3)
        rb = _abi.neox_shard_step_noalloc(desc, hp.c(), state, [g.data_ptr()], b[3].data_ptr(), 1e-3, stream)
        assert (ra.overflow, ra.loss_scale_next, ra.applied_steps) == (rb.overflow, rb.loss_scale_next, rb.applied_steps)
    _equal(a, b)
    shard.close()
