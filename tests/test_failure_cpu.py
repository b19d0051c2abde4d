"""Rank loss and resume of the data-parallel step, on CPU (gloo, 2 ranks).

mixed_precision_zero_b200.zero.zero_step runs pass 1, the 16-byte statistics
all-reduce and pass 2.  Here each rank's shard is a stand-in with the same
interface whose passes are the oracle's (the GPU kernels are checked against
the oracle elsewhere); the collective, the failure path and the checkpoint
logic are the product's.

  run A: 8 steps, uninterrupted;
  run B: rank 1 leaves between steps (exits before step 5); rank 0's step 5
         raises RankLost within the process-group timeout, with its shard
         still exactly as checkpointed after step 4;
  run C: two fresh ranks load the step-4 checkpoints and run steps 5-8;
         the result equals run A byte for byte (hysteresis count included).
"""
import os
import socket
import time
from datetime import timedelta

import numpy as np
import torch
import torch.multiprocessing as mp

N, STEPS, LR = 30_011, 8, 6e-4
BOUNDS = [0, 14_999, N]
OVERFLOWS = {3, 4, 7}
TIMEOUT_S = 20


class OracleShard:
    """The rank's slice stepped by the oracle, with NeoxShard's split-step
    interface (grad_stats / apply / state_dict / load_state_dict)."""

    def __init__(self, rank):
        import oracle
        import synth
        self.o = oracle
        self.lo, self.hi = BOUNDS[rank], BOUNDS[rank + 1]
        self.hp = oracle.OracleHparams(clip_norm=1.0, init_scale=2.0 ** 10, scale_window=2, hysteresis=2)
        master = synth.master_normal(N, 0.02, seed=3)[self.lo:self.hi]
        self.master = master.copy()
        self.m = np.zeros_like(self.master)
        self.v = np.zeros_like(self.master)
        self.w = oracle.encode16(self.master, False)
        self.segs = oracle.segments_array(None, self.hi - self.lo, 0.1)
        self.scaler = oracle.Scaler(self.hp.init_scale, 0, 0, self.hp.hyst0, 0)

    @property
    def scale(self):
        return self.scaler.scale

    def grad_stats(self, grads, params, stats):
        inv_pre, inv_us = self.o.ingest_factors(1, self.hp.predivide, self.scaler.scale)
        bad, ss = self.o.grad_stats(grads, False, inv_pre, inv_us)
        stats[0], stats[1] = ss, 1.0 if bad else 0.0

    def apply(self, grads, params, lr, stats):
        info = self.o.step_decide(self.hp, self.scaler, lr, int(stats[1].item() > 0), float(stats[0].item()))
        if not info.overflow:
            self.o.adam_apply(None, 0, grads, False, self.segs, self.master, self.m, self.v, self.w, False, self.hp,
                              lr, info)
        return info

    def state_dict(self):
        return {"loss_scale": self.scaler.scale, "good_steps": self.scaler.good, "applied_steps": self.scaler.t,
                "hysteresis_count": self.scaler.hyst}

    def load_state_dict(self, d):
        self.scaler.scale, self.scaler.good = d["loss_scale"], d["good_steps"]
        self.scaler.t, self.scaler.hyst = d["applied_steps"], d["hysteresis_count"]

    def arrays(self):
        return {"master": self.master, "m": self.m, "v": self.v, "w": self.w}


def _grads(shard, step):
    import synth
    g = synth.grad_normal16(N, 1e-3, shard.scale, seed=3, tensor_id=0, step=step)
    if step in OVERFLOWS:
        g[synth.inject_index(N, 3, step)] = synth.inject_value(step, False)
    return [g[shard.lo:shard.hi].copy()]


def _save(ckdir, rank, step, shard):
    np.savez(os.path.join(ckdir, f"rank{rank}_step{step}.npz"), **shard.arrays(),
             **{k: np.asarray(v) for k, v in shard.state_dict().items()})


def _load(ckdir, rank, step, shard):
    z = np.load(os.path.join(ckdir, f"rank{rank}_step{step}.npz"))
    for k in ("master", "m", "v", "w"):
        getattr(shard, k)[:] = z[k]
    shard.load_state_dict({"loss_scale": float(z["loss_scale"]), "good_steps": int(z["good_steps"]),
                           "applied_steps": int(z["applied_steps"]), "hysteresis_count": int(z["hysteresis_count"])})


def _rank(rank, world, port, q, cfg):
    import torch.distributed as dist

    from mixed_precision_zero_b200.zero import RankLost, zero_step
    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    dist.init_process_group("gloo", rank=rank, world_size=world, timeout=timedelta(seconds=TIMEOUT_S))
    shard = OracleShard(rank)
    first = 1
    if cfg.get("resume_from"):
        _load(cfg["ckdir"], rank, cfg["resume_from"], shard)
        first = cfg["resume_from"] + 1
    stats = torch.zeros(2, dtype=torch.float64)
    traj = []
    for s in range(first, STEPS + 1):
        if cfg.get("die_rank") == rank and s == cfg.get("die_at"):
            os._exit(0)                       # leaves between steps, nothing in flight
        grads = _grads(shard, s)
        t0 = time.monotonic()
        try:
            info = zero_step(shard, grads, None, LR, stats)
        except RankLost:
            q.put((rank, {"lost_at": s, "elapsed": time.monotonic() - t0, "state": shard.state_dict(),
                          "arrays": {k: v.copy() for k, v in shard.arrays().items()}}))
            return                            # no further collective on a broken group
        traj.append((info.overflow, info.scale_next, info.t))
        _save(cfg["ckdir"], rank, s, shard)
    q.put((rank, {"state": shard.state_dict(), "arrays": shard.arrays(), "traj": traj}))
    dist.destroy_process_group()


def _run(cfg, expect):
    s = socket.socket()
    s.bind(("127.0.0.1", 0))
    port = s.getsockname()[1]
    s.close()
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    procs = [ctx.Process(target=_rank, args=(r, 2, port, q, cfg)) for r in range(2)]
    for p in procs:
        p.start()
    out = dict(q.get(timeout=TIMEOUT_S + 120) for _ in range(expect))
    for p in procs:
        p.join(timeout=TIMEOUT_S + 60)
        if p.is_alive():
            p.kill()
    return out


def test_rank_loss_is_detected_and_resume_is_exact(tmp_path):
    ck_a, ck_b = str(tmp_path / "a"), str(tmp_path / "b")
    os.makedirs(ck_a)
    os.makedirs(ck_b)
    a = _run({"ckdir": ck_a}, expect=2)
    assert a[0]["traj"] == a[1]["traj"]                   # one shared scaler trajectory
    assert [x[0] for x in a[0]["traj"]] == [1 if s in OVERFLOWS else 0 for s in range(1, STEPS + 1)]

    b = _run({"ckdir": ck_b, "die_rank": 1, "die_at": 5}, expect=1)
    lost = b[0]
    assert lost["lost_at"] == 5 and lost["elapsed"] < TIMEOUT_S + 5
    z = np.load(os.path.join(ck_b, "rank0_step4.npz"))   # untouched since its step-4 checkpoint
    for k, v in lost["arrays"].items():
        assert v.tobytes() == z[k].tobytes(), k
    assert lost["state"]["applied_steps"] == int(z["applied_steps"])
    assert lost["state"]["hysteresis_count"] == int(z["hysteresis_count"])

    c = _run({"ckdir": ck_b, "resume_from": 4}, expect=2)
    for r in range(2):
        assert c[r]["state"] == a[r]["state"]
        for k in ("master", "m", "v", "w"):
            assert c[r]["arrays"][k].tobytes() == a[r]["arrays"][k].tobytes(), (r, k)
        assert c[r]["traj"] == a[r]["traj"][4:]
