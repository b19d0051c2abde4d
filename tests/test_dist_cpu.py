"""Multi-process host logic on CPU (gloo, world size 2, 127.0.0.1).

1. bench.py's cross-rank reductions (max of the timed region, sum of params).
2. The ZeRO split of the step: each rank owns a contiguous slice of the flat
   shard, computes its pass-1 statistics, the ranks all-reduce the non-finite
   count and the sum of squares, and every rank then takes the same scaler /
   clip decision and updates its own slice.  The slices, put back together,
   must equal the single-process oracle over the whole shard, and every rank
   must see the same loss-scale trajectory.  (The oracle plays the per-rank
   compute here; the 16-byte exchange is what a multi-GPU step would add.)
"""
import os
import socket

import numpy as np
import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp


def _free_port():
    s = socket.socket()
    s.bind(("127.0.0.1", 0))
    port = s.getsockname()[1]
    s.close()
    return port


def _init(rank, world, port):
    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    dist.init_process_group("gloo", rank=rank, world_size=world)


def _bench_reductions(rank, world, port, q):
    _init(rank, world, port)
    import bench
    mx = bench.max_over_ranks(10.0 + rank)
    sm = bench.sum_over_ranks(1000.0 * (rank + 1))
    q.put((rank, mx, sm))
    dist.destroy_process_group()


def _zero_split(rank, world, port, q):
    _init(rank, world, port)
    import oracle
    import synth
    n, steps = 40_003, 8
    bounds = [0, 19_997, n]  # uneven, odd split
    lo, hi = bounds[rank], bounds[rank + 1]
    hp = oracle.OracleHparams(clip_norm=0.3, init_scale=2.0 ** 12, scale_window=3)
    master_all = synth.master_normal(n, 0.02, seed=1)
    segs = [(0, 7_001, 0.1), (7_001, 20_000, 0.0), (27_001, n - 27_001, 0.1)]
    seg_arr = oracle.segments_array(segs, n, 0.1)
    s_master = master_all[lo:hi].copy()
    s_m = np.zeros(hi - lo, np.float32)
    s_v = np.zeros(hi - lo, np.float32)
    s_w = oracle.encode16(s_master, False)
    scaler = oracle.Scaler(hp.init_scale, 0, 0)
    traj = []
    for s in range(1, steps + 1):
        g_all = synth.grad_normal16(n, 1e-3, scaler.scale, seed=1, tensor_id=0, step=s)
        if s == 4:
            g_all[synth.inject_index(n, 1, s)] = synth.inject_value(0, False)
        g = g_all[lo:hi].copy()
        inv_pre, inv_us = oracle.ingest_factors(1, hp.predivide, scaler.scale)
        nb, ss = oracle.grad_stats([g], False, inv_pre, inv_us)
        t = torch.tensor([float(nb), ss], dtype=torch.float64)
        dist.all_reduce(t)
        info = oracle.step_decide(hp, scaler, 6e-4, int(t[0].item()), float(t[1].item()))
        if not info.overflow:
            oracle.adam_apply(None, lo, [g], False, seg_arr, s_master, s_m, s_v, s_w, False, hp, 6e-4, info)
        traj.append((info.overflow, info.scale_next, info.t, info.norm))
    q.put((rank, lo, hi, s_master, s_m, s_v, s_w, traj))
    dist.destroy_process_group()


def _spawn(fn, world=2):
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=fn, args=(r, world, port, q)) for r in range(world)]
    for p in procs:
        p.start()
    out = [q.get(timeout=180) for _ in range(world)]
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    return sorted(out, key=lambda x: x[0])


def test_bench_cross_rank_reductions():
    out = _spawn(_bench_reductions)
    for rank, mx, sm in out:
        assert mx == 11.0 and sm == 3000.0


def test_zero_split_matches_single_shard_oracle(orc):
    import synth
    out = _spawn(_zero_split)
    n, steps = 40_003, 8
    hp = orc.OracleHparams(clip_norm=0.3, init_scale=2.0 ** 12, scale_window=3)
    segs = [(0, 7_001, 0.1), (7_001, 20_000, 0.0), (27_001, n - 27_001, 0.1)]
    whole = orc.OracleShard(synth.master_normal(n, 0.02, seed=1), hp, segments=segs)
    traj = []
    for s in range(1, steps + 1):
        g = synth.grad_normal16(n, 1e-3, whole.scale, seed=1, tensor_id=0, step=s)
        if s == 4:
            g[synth.inject_index(n, 1, s)] = synth.inject_value(0, False)
        info = whole.step([g], 6e-4)
        traj.append((info.overflow, info.scale_next, info.t, info.norm))
    for rank, lo, hi, m_, mm, vv, ww, tr in out:
        assert [x[:3] for x in tr] == [x[:3] for x in traj]
        for a, b in zip(tr, traj):
            assert a[3] == pytest.approx(b[3], rel=1e-12) or (np.isinf(a[3]) and np.isinf(b[3]))
        # the split re-associates the double sum only at the rank boundary
        np.testing.assert_allclose(m_, whole.master[lo:hi], rtol=1e-6, atol=1e-9)
        np.testing.assert_allclose(mm, whole.m[lo:hi], rtol=1e-5, atol=1e-12)
        np.testing.assert_allclose(vv, whole.v[lo:hi], rtol=1e-5, atol=1e-15)
        assert np.abs(ww.astype(np.int64) - whole.w[lo:hi].astype(np.int64)).max() <= 1
