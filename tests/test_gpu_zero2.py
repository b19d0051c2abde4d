"""ZeRO-2 through peer memory, as two or three processes sharing one GPU.

Each process is a data-parallel rank that owns one flat slice of the model
and holds the full gradient of its own micro-batches and a full copy of the
16-bit weights.  Through CUDA IPC (mixed_precision_zero_b200.peer) every rank
maps the other's buffers; then per step:
  - pass 1 reads every rank's copy of this rank's gradient slice and sums it
    (the reduce-scatter fused with the ingest, pre-divide before the sum);
  - the 16-byte statistics are all-reduced (gloo) and every rank takes the
    same decision;
  - pass 2 updates the slice and stores the cast into every rank's weight
    buffer (the all-gather fused with the cast).
The result must equal the oracle over the whole model with the K = 2 rank
gradients as its buffers: bit-exact with clipping off.

The ranks are ordered against each other only by zero.zero2_step's stream
barriers (interprocess CUDA events over this gloo group): there is no device
synchronisation and no host barrier between the steps, and each rank writes
its next gradients right after its step returns.  No kernel waits on
another: the barriers are stream waits on events whose records were issued
before the waits."""
import os
import socket
import traceback
from datetime import timedelta

import numpy as np
import pytest
import torch

import oracle
from tests.gpu_harness import check_close, check_ulp16

pytestmark = pytest.mark.gpu


def _free_port():
    s = socket.socket()
    s.bind(("127.0.0.1", 0))
    port = s.getsockname()[1]
    s.close()
    return port


def _rank_main(rank, world, port, q, cfg):
    import torch.distributed as dist
    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    dist.init_process_group("gloo", rank=rank, world_size=world, timeout=timedelta(seconds=120))
    try:
        import synth
        from mixed_precision_zero_b200 import Hparams, NeoxShard
        from mixed_precision_zero_b200.peer import PeerMap, allgather_weight_dsts, zero2_grad_ptrs
        from mixed_precision_zero_b200.zero import make_stream_barrier, zero2_step
        torch.cuda.set_device(0)
        n, steps, lr = cfg["n"], cfg["steps"], cfg["lr"]
        N = world * n
        hp = Hparams(**cfg["hp"])
        master_full = torch.empty(N, dtype=torch.float32, device="cuda")
        synth.gpu_master_normal(master_full, 0.02, 7)        # the same model on every rank
        master = master_full[rank * n:(rank + 1) * n].clone()
        m, v = torch.zeros_like(master), torch.zeros_like(master)
        wfull = master_full.to(torch.float16)                 # this rank's full working weights
        grads_full = torch.empty(N, dtype=torch.float16, device="cuda")
        gmap = PeerMap.from_group(grads_full)
        wmap = PeerMap.from_group(wfull)
        shard = NeoxShard(master, m, v, hp, weight_decay=0.1, max_grads=world, accumulate=cfg["accumulate"])
        params = wfull[rank * n:(rank + 1) * n]
        shard.set_weight_copies(allgather_weight_dsts(wmap, n))
        gptrs = zero2_grad_ptrs(gmap, n)
        stats = torch.zeros(2, dtype=torch.float64, device="cuda")
        barrier = make_stream_barrier()
        out = {"host_grads": [], "results": []}
        if rank == 0:
            out["master0"] = master_full.cpu().numpy()
        for s in range(1, steps + 1):
            # this rank's gradients of step s, written on its stream right after
            # its previous step returned (no host or device synchronisation)
            synth.gpu_grad_normal16(grads_full, 1e-3, shard.get_state()[0], 7, rank, s)
            if s == cfg["overflow_step"] and rank == 1:
                grads_full.view(torch.int16)[5] = 0x7C00       # in slice 0: rank 0's pass 1 must see it
            # barrier, pass 1 over both ranks' copies, all-reduce, pass 2 with the
            # weight copies, barrier
            res = zero2_step(shard, gptrs, params, lr, stats, barrier)
            # read back for the oracle (the step only reads the gradients)
            out["host_grads"].append(grads_full.view(torch.int16).cpu().numpy().view(np.uint16).copy())
            out["results"].append((res.overflow, res.loss_scale_next, res.applied_steps, res.grad_norm))
        out["master"] = master.cpu().numpy()
        out["m"] = m.cpu().numpy()
        out["v"] = v.cpu().numpy()
        out["wfull"] = wfull.view(torch.int16).cpu().numpy().view(np.uint16)
        shard.close()
        gmap.close()
        wmap.close()
        dist.barrier()                                         # nobody frees what a peer still maps
        q.put((rank, out))
    except BaseException:
        q.put((rank, {"error": traceback.format_exc()}))
    finally:
        dist.destroy_process_group()


@pytest.mark.parametrize("world,accumulate,clip", [(2, True, 0.0), (2, False, 1.0), (3, True, 0.0), (3, False, 0.0)])
def test_zero2_reduce_scatter_and_allgather_through_ipc(world, accumulate, clip):
    import torch.multiprocessing as mp
    cfg = {"n": 300_007, "steps": 5, "lr": 1e-3, "overflow_step": 3, "accumulate": accumulate,
           "hp": {"clip_norm": clip, "init_scale": 2.0 ** 12, "scale_window": 2, "predivide": 2.0}}
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_rank_main, args=(r, world, port, q, cfg)) for r in range(world)]
    for p in procs:
        p.start()
    got = {}
    try:
        for _ in range(world):
            r, out = q.get(timeout=600)
            got[r] = out
    finally:
        for p in procs:
            p.join(timeout=120)
            if p.is_alive():
                p.kill()
    for r in range(world):
        assert "error" not in got[r], got[r].get("error")
    n = cfg["n"]
    ohp = oracle.OracleHparams(clip_norm=clip, init_scale=2.0 ** 12, scale_window=2, predivide=2.0)
    orc = oracle.OracleShard(got[0]["master0"], ohp, default_wd=0.1)
    for s in range(cfg["steps"]):
        info = orc.step([got[r]["host_grads"][s] for r in range(world)], cfg["lr"])
        for r in range(world):
            ov, scale_next, t, norm = got[r]["results"][s]
            assert ov == info.overflow == (1 if s + 1 == cfg["overflow_step"] else 0)
            assert scale_next == info.scale_next and t == info.t
            if not info.overflow:
                assert abs(norm - info.norm) <= 1e-5 * info.norm
    master = np.concatenate([got[r]["master"] for r in range(world)])
    m = np.concatenate([got[r]["m"] for r in range(world)])
    v = np.concatenate([got[r]["v"] for r in range(world)])
    if clip == 0.0:
        assert master.tobytes() == orc.master.tobytes()
        assert m.tobytes() == orc.m.tobytes() and v.tobytes() == orc.v.tobytes()
        for r in range(world):   # every rank's full weights are the all-gathered cast
            assert np.array_equal(got[r]["wfull"], orc.w)
    else:
        check_close("master", master, orc.master)
        check_close("m", m, orc.m)
        check_close("v", v, orc.v)
        for r in range(world):
            check_ulp16(got[r]["wfull"], orc.w)
