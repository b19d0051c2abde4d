"""The split step (grad_stats -> all-reduce of 16 bytes -> apply), the form a
data-parallel rank runs so that all ranks share one global norm, overflow
flag and loss scale.

On one GPU: the split step without any reduction equals the fused step byte
for byte; and a shard cut into two "ranks" (two handles over the two halves,
run one after the other -- no kernel waits on another) whose statistics are
summed on the device equals the oracle over the whole shard."""
import numpy as np
import pytest
import torch

import oracle
import synth
from mixed_precision_zero_b200 import Hparams, NeoxShard
from tests.gpu_harness import Guarded, check_close, check_ulp16, to_u16

pytestmark = pytest.mark.gpu


def _state(n, seed, wdt):
    master = torch.empty(n, dtype=torch.float32, device="cuda")
    synth.gpu_master_normal(master, 0.02, seed)
    return [master, torch.zeros_like(master), torch.zeros_like(master), master.to(wdt)]


@pytest.mark.parametrize("K,bf16,max_grads,clip", [(1, False, 1, 1.0), (1, True, 1, 0.3), (8, False, 8, 0.3),
                                                   (3, False, 1, 0.0)])
def test_split_equals_fused(K, bf16, max_grads, clip):
    torch.cuda.set_device(0)
    n = 700_001
    dt = torch.bfloat16 if bf16 else torch.float16
    hp = Hparams(clip_norm=clip, predivide=float(K), init_scale=2.0 ** 10, scale_window=2)
    a = _state(n, 21, dt)
    b = [x.clone() for x in a]
    grads = [torch.empty(n, dtype=dt, device="cuda") for _ in range(K)]
    fused = NeoxShard(a[0], a[1], a[2], hp, wdtype=dt, gdtype=dt, max_grads=max_grads, weight_decay=0.1)
    split = NeoxShard(b[0], b[1], b[2], hp, wdtype=dt, gdtype=dt, max_grads=max_grads, weight_decay=0.1)
    stats = torch.zeros(2, dtype=torch.float64, device="cuda")
    for s in range(1, 7):
        for k, g in enumerate(grads):
            if K > 1:
                synth.gpu_grad_t3_16(g, fused.get_state()[0], 21, k, s, bf16)
            else:
                synth.gpu_grad_normal16(g, 1e-3, fused.get_state()[0], 21, k, s, bf16)
        if s == 4:
            grads[0].view(torch.int16)[77] = 0x7C00 if not bf16 else 0x7F80
        ra = fused.step(grads, a[3], 6e-4)
        split.grad_stats(grads, b[3], stats)
        rb = split.apply(grads, b[3], 6e-4, stats)
        assert ra.as_dict() == rb.as_dict()
    for x, y in zip(a, b):
        assert torch.equal(x.view(torch.uint8), y.view(torch.uint8))
    fused.close()
    split.close()


@pytest.mark.parametrize("clip", [0.0, 1.0])
def test_two_ranks_share_one_decision(clip):
    """Two halves of a shard stepped as two ranks with summed statistics
    track the oracle over the whole shard (bit-exact with clipping off);
    both ranks report the same norm, flag and scale trajectory."""
    torch.cuda.set_device(0)
    n, cut = 400_003, 150_001
    hp = Hparams(clip_norm=clip, init_scale=2.0 ** 14, scale_window=2)
    st = _state(n, 22, torch.float16)
    g = Guarded(n, torch.float16, 0)
    parts = [(0, cut), (cut, n - cut)]
    ranks = []
    for o, c in parts:
        views = [x[o:o + c] for x in st]
        ranks.append((NeoxShard(views[0], views[1], views[2], hp, weight_decay=0.1), views, g.t[o:o + c]))
    ohp = oracle.OracleHparams(clip_norm=clip, init_scale=2.0 ** 14, scale_window=2)
    orc = oracle.OracleShard(st[0].cpu().numpy(), ohp, default_wd=0.1)
    local = [torch.zeros(2, dtype=torch.float64, device="cuda") for _ in parts]
    for s in range(1, 7):
        synth.gpu_grad_normal16(g.t, 1e-3, orc.scale, 22, 0, s)
        if s == 3:
            g.t.view(torch.int16)[cut + 5] = 0x7E00  # NaN in the second rank's half
        torch.cuda.synchronize()
        host = to_u16(g.t)
        for (sh, views, gv), buf in zip(ranks, local):
            sh.grad_stats([gv], views[3], buf)
        total = local[0] + local[1]          # stands in for the all-reduce
        res = [sh.apply([gv], views[3], 6e-4, total) for sh, views, gv in ranks]
        info = orc.step([host], 6e-4)
        for r in res:
            assert r.overflow == info.overflow == (1 if s == 3 else 0)
            assert r.loss_scale_next == info.scale_next and r.applied_steps == info.t
            if not info.overflow:
                assert abs(r.grad_norm - info.norm) <= 1e-5 * info.norm
    exact = clip == 0.0
    gm, gmm, gv_ = (x.cpu().numpy() for x in st[:3])
    gw = to_u16(st[3])
    if exact:
        assert gm.tobytes() == orc.master.tobytes() and gmm.tobytes() == orc.m.tobytes()
        assert gv_.tobytes() == orc.v.tobytes() and np.array_equal(gw, orc.w)
    else:
        check_close("master", gm, orc.master)
        check_close("m", gmm, orc.m)
        check_close("v", gv_, orc.v)
        check_ulp16(gw, orc.w)
    for sh, _, _ in ranks:
        sh.close()


def test_split_rejects_missing_stats():
    torch.cuda.set_device(0)
    st = _state(1000, 1, torch.float16)
    sh = NeoxShard(st[0], st[1], st[2])
    g = torch.zeros(1000, dtype=torch.float16, device="cuda")
    from mixed_precision_zero_b200 import _abi, NeoxError
    with pytest.raises(NeoxError):
        _abi.neox_shard_grad_stats(sh.handle, [g.data_ptr()], st[3].data_ptr(), 0, None)
    with pytest.raises(NeoxError):
        _abi.neox_shard_apply(sh.handle, [g.data_ptr()], st[3].data_ptr(), 1e-3, 0, 0)
    sh.close()
