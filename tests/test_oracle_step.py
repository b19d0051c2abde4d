"""Pins of the oracle's optimizer step against closed forms, invariants, page
facts and library special cases (never against the CUDA path).

Each test names what it pins; together they are chosen so that a dropped term,
a wrong sign, a swapped operand or a wrong index in ``oracle.c`` fails one.
"""
import os
from fractions import Fraction

import numpy as np
import pytest
import torch

import synth

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")

F32 = np.float32


def f16(x):
    """Library RNE cast to binary16 codes (torch), independent of the oracle's encoder."""
    return torch.from_numpy(np.asarray(x, np.float32)).to(torch.float16).view(torch.int16).numpy().view(np.uint16)


def bf16(x):
    return torch.from_numpy(np.asarray(x, np.float32)).to(torch.bfloat16).view(torch.int16).numpy().view(np.uint16)


def dec_f16(h):
    return torch.from_numpy(np.asarray(h, np.uint16).view(np.int16)).view(torch.float16).to(torch.float64).numpy()


def make_shard(orc, n, seed=0, **hp):
    rng = np.random.default_rng(seed)
    master = (rng.standard_normal(n) * 0.02).astype(np.float32)
    kw = {k: hp.pop(k) for k in ("wbf16", "gbf16", "segments", "default_wd") if k in hp}
    return orc.OracleShard(master, orc.OracleHparams(**hp), **kw)


# ---------------------------------------------------------------- closed forms

def test_zero_grad_only_decays(orc):
    """g = 0 from m = v = 0: the Adam term vanishes, p <- p(1 - lr*wd), m = v = 0."""
    n, lr, wd = 4096, F32(6e-4), F32(0.1)
    sh = make_shard(orc, n, default_wd=float(wd))
    p0 = sh.master.copy()
    info = sh.step([np.zeros(n, np.uint16)], float(lr))
    assert info.overflow == 0 and info.norm == 0.0 and info.coef == 1.0
    keep = F32(1) - lr * wd
    np.testing.assert_array_equal(sh.master, p0 * keep)
    assert not sh.m.any() and not sh.v.any()
    np.testing.assert_array_equal(sh.w, f16(sh.master))


@pytest.mark.parametrize("wd", [0.0, 0.1])
def test_first_step_eps0_is_sign_update(orc, wd):
    """First step with eps = 0: m/bc1 = g and sqrt(v/bc2) = |g|, so the Adam
    step is lr*sign(g) exactly in the reals; FP32 rounding leaves a few ulps."""
    n, lr = 8192, 6e-4
    rng = np.random.default_rng(1)
    sh = make_shard(orc, n, eps=0.0, clip_norm=0.0, init_scale=1.0, default_wd=wd)
    g = f16(rng.choice([-1, 1], n) * rng.uniform(1e-3, 4.0, n))
    p0 = sh.master.astype(np.float64)
    sh.step([g], lr)
    sign = np.sign(dec_f16(g))
    expect = p0 * (1 - F32(lr) * F32(wd)) - F32(lr) * sign
    # FP32 storage of p costs up to 1 ulp of p on top of a few ulps of lr
    np.testing.assert_allclose(sh.master, expect, rtol=2.0 ** -22, atol=lr * 4e-7)


def test_constant_grad_bias_corrected_update(orc):
    """wd = 0, the same g on every step: m_t = (1-b1^t) g and v_t = (1-b2^t) g^2,
    so each bias-corrected step is lr*g/(|g|+eps) and after T steps
    p_T = p_0 - T*lr*g/(|g|+eps)."""
    n, lr, T, eps = 2048, 1e-3, 25, 1e-8
    rng = np.random.default_rng(2)
    sh = make_shard(orc, n, eps=eps, clip_norm=0.0, init_scale=1.0, default_wd=0.0)
    gv = rng.choice([-1, 1], n) * rng.uniform(1e-4, 2.0, n)
    g = f16(gv)
    gd = dec_f16(g)
    p0 = sh.master.astype(np.float64)
    for _ in range(T):
        sh.step([g], lr)
    expect = p0 - T * lr * gd / (np.abs(gd) + eps)
    # each of the T steps rounds p to FP32 (half an ulp of |p| <= 0.1) and the
    # Adam term to a few ulps of lr
    np.testing.assert_allclose(sh.master, expect, rtol=0, atol=T * (lr * 1e-6 + 2.0 ** -28))
    # m itself: (1-b1^T) g, v: (1-b2^T) g^2
    np.testing.assert_allclose(sh.m, (1 - 0.9 ** T) * gd, rtol=2e-6)
    np.testing.assert_allclose(sh.v, (1 - 0.95 ** T) * gd * gd, rtol=4e-6)


def test_norm_closed_form_power_of_two(orc):
    """All N = 4^k elements equal 2^j: norm = 2^(j+k) exactly."""
    for k, j in [(5, -3), (8, 0), (10, -12), (6, 4)]:
        n = 4 ** k
        g = f16(np.full(n, 2.0 ** j))
        nb, s = orc.grad_stats([g], False, 1.0, 1.0)
        assert nb == 0 and np.sqrt(s) == 2.0 ** (j + k)


def test_norm_matches_library_norm(orc):
    rng = np.random.default_rng(3)
    g = f16(rng.standard_normal(100_003) * 3.0)
    S = 2.0 ** 5
    inv_pre, inv_us = orc.ingest_factors(1, 1.0, S)
    nb, s = orc.grad_stats([g], False, inv_pre, inv_us)
    ref = torch.linalg.vector_norm(torch.from_numpy(dec_f16(g) / S)).item()
    assert nb == 0
    assert abs(np.sqrt(s) - ref) <= 1e-12 * ref


@pytest.mark.parametrize("K,pre,S", [(8, 8.0, 2.0 ** 10), (8, 1.0, 1.0), (4, 2.0, 2.0 ** 3), (2, 4.0, 0.5)])
def test_predivide_gives_exact_mean(orc, K, pre, S):
    """With power-of-two K, predivide and scale, and inputs whose sums are exact,
    the unscaled gradient is exactly mean_k(g_k) / S."""
    rng = np.random.default_rng(K)
    n = 5000
    ints = rng.integers(-1024, 1025, size=(K, n))
    grads = [f16(ints[k].astype(np.float32)) for k in range(K)]
    inv_pre, inv_us = orc.ingest_factors(K, pre, S)
    got = orc.unscaled_grads(grads, False, inv_pre, inv_us)
    Sf = Fraction(S)
    for j in range(0, n, 97):
        exact = Fraction(int(ints[:, j].sum()), K) / Sf
        assert Fraction(float(got[j])) == exact


def test_clip_coefficient_invariants(orc):
    """Post-clip norm <= clip; c == 1 when the norm is within the clip; clip <= 0 is off."""
    rng = np.random.default_rng(4)
    for clip in (1.0, 0.3):
        for norm in rng.uniform(0.0, 50.0, 2000):
            c = orc.clip_coef(clip, norm)
            assert 0.0 < c <= 1.0
            assert c * norm <= clip * (1 + 2 ** -23)
            if norm + 1e-6 <= clip:
                assert c == 1.0
            else:
                assert c * (norm + 1e-6) == pytest.approx(clip, rel=2 ** -23)
        # the 1e-6 margin: a norm equal to the clip is still scaled (just) down
        assert orc.clip_coef(clip, clip - 2e-6) == 1.0 and orc.clip_coef(clip, clip) < 1.0
    assert orc.clip_coef(0.0, 1e9) == 1.0 and orc.clip_coef(-1.0, 1e9) == 1.0
    # exact case: norm + 1e-6 = 4 * clip (in double) gives c = 0.25 exactly
    assert orc.clip_coef(0.5, 2.0 - 1e-6) == 0.25


def test_step_applies_clip_to_moments(orc):
    """First step: m = (1-b1) * c * g; recovering c*g from m gives a post-clip
    norm <= clip (0.3) while the raw norm is far above it."""
    n = 50_000
    rng = np.random.default_rng(5)
    sh = make_shard(orc, n, clip_norm=0.3, init_scale=2.0 ** 10)
    g = f16(rng.standard_normal(n) * 1e-2 * 2 ** 10)
    info = sh.step([g], 6e-4)
    assert info.norm > 1.0 and info.coef < 1.0
    clipped = sh.m.astype(np.float64) / (1 - F32(0.9))
    assert np.linalg.norm(clipped) <= 0.3 * (1 + 1e-6)
    assert np.linalg.norm(clipped) == pytest.approx(0.3, rel=1e-5)


# ---------------------------------------------------------------- overflow / skip

@pytest.mark.parametrize("bad", [np.inf, np.nan, -np.inf])
def test_overflow_skips_and_backs_off(orc, bad):
    n = 3000
    rng = np.random.default_rng(6)
    sh = make_shard(orc, n, init_scale=2.0 ** 16, scale_window=3)
    g = f16(rng.standard_normal(n) * 1e-3 * 2 ** 16)
    sh.step([g], 6e-4)
    sh.step([g], 6e-4)
    assert sh.scaler.good == 2 and sh.scaler.t == 2
    before = [a.copy() for a in (sh.master, sh.m, sh.v, sh.w)]
    g2 = g.copy()
    g2[1234] = f16([bad])[0]
    info = sh.step([g2], 6e-4)
    assert info.overflow == 1 and np.isinf(info.norm)
    for a, b in zip(before, (sh.master, sh.m, sh.v, sh.w)):
        assert a.tobytes() == b.tobytes()
    assert sh.scaler.t == 2 and sh.scaler.good == 0
    assert sh.scale == 2.0 ** 15 and info.scale_next == 2.0 ** 15 and info.scale_used == 2.0 ** 16


def test_nonfinite_count_exact(orc):
    """Pass 1 counts every non-finite unscaled element: +inf, -inf and NaN
    codes planted at known positions across K buffers, nothing else."""
    n, K = 10_000, 3
    rng = np.random.default_rng(11)
    grads = [f16(rng.standard_normal(n)) for _ in range(K)]
    planted = {(0, 5): np.inf, (1, 5): -np.inf, (2, 77): np.nan, (0, 9000): -np.inf, (2, 9999): np.inf}
    for (k, j), val in planted.items():
        grads[k][j] = f16([val])[0]
    inv_pre, inv_us = orc.ingest_factors(K, 1.0, 1.0)
    nb, _ = orc.grad_stats(grads, False, inv_pre, inv_us)
    assert nb == 4  # element 5 holds two of the five plants


def test_unscale_overflow_counts(orc):
    """Finite inputs whose unscaled value overflows FP32 (scale far below one,
    floor 0) are an overflow too."""
    n = 64
    sh = make_shard(orc, n, init_scale=2.0 ** -120, min_scale=0.0)
    g = f16(np.full(n, 60000.0))
    info = sh.step([g], 1e-3)
    assert info.overflow == 1 and sh.scale == 2.0 ** -121


def test_skipped_step_does_not_advance_t(orc):
    """Inserting an overflowed call between applied calls (grads carried at the
    current scale, power-of-two scales) leaves the final state bit-identical:
    the skip changes nothing but the scale, and t only counts applied steps."""
    n = 4096
    rng = np.random.default_rng(7)
    master = (rng.standard_normal(n) * 0.02).astype(np.float32)
    true = [rng.standard_normal(n) * 1e-3 for _ in range(5)]
    runs = []
    for skip_at in (None, 2):
        sh = orc.OracleShard(master, orc.OracleHparams(init_scale=2.0 ** 12, scale_window=100))
        seq = list(range(5))
        if skip_at is not None:
            seq.insert(skip_at, -1)
        for s in seq:
            if s < 0:
                g = f16(true[0] * sh.scale)
                g[17] = f16([np.inf])[0]
            else:
                g = f16(true[s] * sh.scale)
            sh.step([g], 6e-4)
        runs.append(sh)
    a, b = runs
    assert a.scaler.t == b.scaler.t == 5
    for x, y in ((a.master, b.master), (a.m, b.m), (a.v, b.v), (a.w, b.w)):
        assert x.tobytes() == y.tobytes()
    assert b.scale == a.scale / 2


def test_empty_shard(orc):
    """A rank owning zero elements: the norm is zero, the step is applied."""
    sh = orc.OracleShard(np.zeros(0, np.float32), orc.OracleHparams(scale_window=1))
    info = sh.step([np.zeros(0, np.uint16)], 1e-3)
    assert info.overflow == 0 and info.norm == 0.0 and info.t == 1 and sh.scale == 2.0 ** 17


# ---------------------------------------------------------------- scaler

def _golden_trajectories():
    recs = {}
    with open(os.path.join(GOLDEN, "scaler_trajectories.txt")) as f:
        for line in f:
            line = line.strip()
            if not line or line.startswith("#"):
                continue
            name, init, fac, win, ov, traj, t = [x.strip() for x in line.split("|")]
            seq = []
            for tok in traj.split():
                v, _, rep = tok.partition("x")
                seq += [float(v)] * (int(rep) if rep else 1)
            recs[name] = (float(init), float(fac), int(win), [int(x) for x in ov.split()], seq, int(t))
    return recs


@pytest.mark.parametrize("name", ["tiny", "opt_style"])
def test_scaler_trajectory_golden(orc, name):
    init, fac, win, ov_steps, traj, t_final = _golden_trajectories()[name]
    hp = orc.OracleHparams(init_scale=init, scale_factor=fac, scale_window=win)
    scale, good, t = init, 0, 0
    got = []
    for s in range(1, len(traj) + 1):
        ov = s in ov_steps
        scale, good, t = orc.scaler_update(hp, scale, good, t, ov)
        if not ov:
            t += 1
        got.append(scale)
    assert got == traj and t == t_final


def test_tiny_trajectory_through_full_steps(orc):
    """The tiny-shard workload end to end through orc_step: 1,048,576 FP16
    grads N(0,1e-3)*S, an inf at a seeded index on call 4, window 2."""
    init, fac, win, ov_steps, traj, t_final = _golden_trajectories()["tiny"]
    n = 1 << 20
    master = synth.master_normal(n, 0.02, seed=0)
    sh = orc.OracleShard(master, orc.OracleHparams(init_scale=init, scale_window=win))
    got = []
    for s in range(1, 11):
        g = synth.grad_normal16(n, 1e-3, sh.scale, seed=0, tensor_id=0, step=s)
        if s in ov_steps:
            g[synth.inject_index(n, 0, s)] = synth.inject_value(0, False)
        info = sh.step([g], 6e-4)
        assert bool(info.overflow) == (s in ov_steps)
        got.append(sh.scale)
    assert got == traj and sh.scaler.t == t_final


def test_scaler_matches_torch_gradscaler(orc):
    """Backoff / growth / counter reset agree with torch's GradScaler update
    (growth 2, backoff 0.5, growth_interval = window) on random flag sequences."""
    rng = np.random.default_rng(8)
    for win in (1, 2, 5):
        flags = rng.random(300) < 0.2
        hp = orc.OracleHparams(init_scale=2.0 ** 16, scale_window=win, min_scale=0.0)
        scale_t = torch.tensor([2.0 ** 16], dtype=torch.float32)
        tracker = torch.tensor([0], dtype=torch.int32)
        s, good, t = 2.0 ** 16, 0, 0
        for fl in flags:
            torch._amp_update_scale_(scale_t, tracker, torch.tensor([float(fl)]), 2.0, 0.5, win)
            s, good, t = orc.scaler_update(hp, s, good, t, bool(fl))
            assert s == scale_t.item() and good == tracker.item()


def test_scaler_floor(orc):
    hp = orc.OracleHparams(init_scale=8.0, min_scale=1.0)
    s, g, t = 8.0, 0, 0
    seen = []
    for _ in range(6):
        s, g, t = orc.scaler_update(hp, s, g, t, True)
        seen.append(s)
    assert seen == [4.0, 2.0, 1.0, 1.0, 1.0, 1.0]
    hp0 = orc.OracleHparams(init_scale=8.0, min_scale=0.0)
    s = 8.0
    for _ in range(200):
        s, g, t = orc.scaler_update(hp0, s, g, t, True)
    assert s == 0.0


# ---------------------------------------------------------------- library special case

def test_matches_torch_adamw_float64(orc):
    """K = 1, predivide 1, scale 1: the step is clip_grad_norm_ followed by
    AdamW.  torch in float64 (foreach=False) on two parameter groups (wd 0.1
    and 0) bounds the FP32 oracle within the step's tolerance."""
    rng = np.random.default_rng(9)
    n1, n2 = 3000, 700
    lr, b1, b2, eps, wd = (float(F32(x)) for x in (6e-4, 0.9, 0.95, 1e-8, 0.1))
    master = (rng.standard_normal(n1 + n2) * 0.02).astype(np.float32)
    sh = orc.OracleShard(master, orc.OracleHparams(beta1=b1, beta2=b2, eps=eps, clip_norm=1.0,
                                                   init_scale=1.0, scale_window=10 ** 6),
                         segments=[(0, n1, wd), (n1, n2, 0.0)])
    p1 = torch.nn.Parameter(torch.from_numpy(master[:n1].astype(np.float64)))
    p2 = torch.nn.Parameter(torch.from_numpy(master[n1:].astype(np.float64)))
    opt = torch.optim.AdamW([{"params": [p1], "weight_decay": wd}, {"params": [p2], "weight_decay": 0.0}],
                            lr=lr, betas=(b1, b2), eps=eps, foreach=False)
    for step in range(30):
        sigma = 0.05 if step % 3 else 1e-3     # alternate clipped / unclipped steps
        g = f16(rng.standard_normal(n1 + n2) * sigma)
        info = sh.step([g], lr)
        gd = torch.from_numpy(dec_f16(g))
        p1.grad, p2.grad = gd[:n1].clone(), gd[n1:].clone()
        tn = torch.nn.utils.clip_grad_norm_([p1, p2], 1.0, foreach=False)
        opt.step()
        assert info.norm == pytest.approx(tn.item(), rel=1e-12)
    ref = torch.cat([p1.detach(), p2.detach()]).numpy()
    np.testing.assert_allclose(sh.master, ref, rtol=1e-5, atol=1e-7)
    st = [opt.state[p] for p in (p1, p2)]
    m_ref = torch.cat([s["exp_avg"] for s in st]).numpy()
    v_ref = torch.cat([s["exp_avg_sq"] for s in st]).numpy()
    # moments near a sign change lose relative accuracy to cancellation; the
    # absolute floor is a millionth of the largest moment
    np.testing.assert_allclose(sh.m, m_ref, rtol=1e-5, atol=1e-6 * np.abs(m_ref).max())
    np.testing.assert_allclose(sh.v, v_ref, rtol=1e-5, atol=1e-6 * np.abs(v_ref).max())


# ---------------------------------------------------------------- float64 brute force

@pytest.mark.parametrize("gbf16,K,pre", [(False, 1, 1.0), (False, 3, 2.0), (True, 1, 1.0), (True, 4, 4.0)])
def test_fp32_oracle_tracks_float64_brute_force(orc, gbf16, K, pre):
    """100 calls on a 4096-element shard with three segments, overflows on
    scripted calls, the FP32 oracle stays within 1e-5 relative of the float64
    brute force; flags and scales agree exactly."""
    n = 4096
    rng = np.random.default_rng(10 + K)
    master = (rng.standard_normal(n) * 0.02).astype(np.float32)
    segs = [(0, 1000, 0.1), (1000, 96, 0.0), (1096, n - 1096, 0.05)]
    hp = orc.OracleHparams(clip_norm=0.3, predivide=pre, init_scale=2.0 ** 14, scale_window=7)
    o32 = orc.OracleShard(master, hp, wbf16=gbf16, gbf16=gbf16, segments=segs)
    o64 = orc.Oracle64Shard(master, hp, gbf16=gbf16, segments=segs)
    enc = bf16 if gbf16 else f16
    for s in range(1, 101):
        grads = [enc(rng.standard_normal(n) * 2e-3 * o32.scale) for _ in range(K)]
        if s in (5, 6, 40):
            grads[K - 1][rng.integers(n)] = enc([np.nan])[0]
        i32 = o32.step(grads, 1e-3)
        ov64, norm64 = o64.step(grads, 1e-3)
        assert bool(i32.overflow) == ov64
        assert o32.scale == o64.scaler.scale and o32.scaler.t == o64.scaler.t
        if not ov64:
            assert i32.norm == pytest.approx(norm64, rel=1e-6)
    for a32, a64 in ((o32.master, o64.master), (o32.m, o64.m), (o32.v, o64.v)):
        np.testing.assert_allclose(a32, a64, rtol=1e-5, atol=1e-7)
    np.testing.assert_allclose(o32.v, o64.v, rtol=1e-5, atol=0)


def test_philox_known_answers():
    """The input generator's Philox4x32-10 reproduces the published vectors."""
    with open(os.path.join(GOLDEN, "philox4x32_10_kat.txt")) as f:
        rows = [ln.split("->") for ln in f if ln.strip() and not ln.startswith("#")]
    for lhs, rhs in rows:
        c0, c1, c2, c3, k0, k1 = (int(x, 16) for x in lhs.split())
        want = [int(x, 16) for x in rhs.split()]
        got = [int(v) for v in synth.philox4x32(c0, c1, c2, c3, k0, k1)]
        assert got == want


def test_state_accounting_oracle_arrays(orc):
    """The oracle's per-element state: FP32 master/m/v, 16-bit working copy,
    16-bit grad = 16 bytes per parameter, as the bottleneck section states."""
    facts = dict(ln.split() for ln in open(os.path.join(GOLDEN, "state_accounting.txt"))
                 if ln.strip() and not ln.startswith("#"))
    sh = make_shard(orc, 1000)
    per = (sh.master.itemsize + sh.m.itemsize + sh.v.itemsize + sh.w.itemsize + np.dtype(np.uint16).itemsize)
    assert per == 16
    assert int(facts["params"]) * per == int(facts["state_bytes"])
    assert int(facts["params"]) * sh.w.itemsize == int(facts["fp16_weight_bytes"])


# ---------------------------------------------------------------- scaler / optimizer variants

def test_scaler_hysteresis_golden(orc):
    facts = {}
    for ln in open(os.path.join(GOLDEN, "scaler_hysteresis.txt")):
        if ln.strip() and not ln.startswith("#"):
            k, *v = ln.split()
            facts[k] = [float(x) for x in v]
    hp = orc.OracleHparams(init_scale=facts["init"][0], scale_factor=facts["factor"][0],
                           scale_window=int(facts["window"][0]), hysteresis=int(facts["hysteresis"][0]))
    ov = {int(x) for x in facts["overflows"]}
    s, g, t, h = hp.init_scale, 0, 0, hp.hyst0
    got = []
    for call in range(1, len(facts["scales"]) + 1):
        s, g, t, h = orc.scaler_update(hp, s, g, t, call in ov, hyst=h, with_hyst=True)
        if call not in ov:
            t += 1
        got.append(s)
    assert got == facts["scales"] and t == int(facts["applied"][0])
    # hysteresis 0 or 1 is the plain scaler: a back-off at every overflow
    # (same calls, worked by hand: 2, 3 halve; 6, 7, 8 halve; 11 grows; 12
    # halves; 15 grows)
    plain = [1024, 512, 256, 256, 256, 128, 64, 32, 32, 32, 64, 32, 32, 32, 64]
    for h1 in (0, 1):
        hp1 = orc.OracleHparams(init_scale=1024.0, scale_window=3, hysteresis=h1)
        s, g, t, h = 1024.0, 0, 0, hp1.hyst0
        got = []
        for call in range(1, 16):
            s, g, t, h = orc.scaler_update(hp1, s, g, t, call in ov, hyst=h, with_hyst=True)
            got.append(s)
        assert got == plain


def test_sgd_matches_torch_float64(orc):
    """The SGD fallback: clip_grad_norm_ + torch.optim.SGD(momentum=0,
    weight_decay=wd) in float64 (coupled decay equals decoupled decay for
    plain SGD in exact arithmetic)."""
    rng = np.random.default_rng(31)
    n1, n2 = 2000, 500
    lr, wd = float(F32(5e-3)), float(F32(0.1))
    master = (rng.standard_normal(n1 + n2) * 0.02).astype(np.float32)
    sh = orc.OracleShard(master, orc.OracleHparams(clip_norm=1.0, init_scale=1.0, scale_window=10 ** 6, optimizer=1),
                         segments=[(0, n1, wd), (n1, n2, 0.0)])
    p1 = torch.nn.Parameter(torch.from_numpy(master[:n1].astype(np.float64)))
    p2 = torch.nn.Parameter(torch.from_numpy(master[n1:].astype(np.float64)))
    opt = torch.optim.SGD([{"params": [p1], "weight_decay": wd}, {"params": [p2], "weight_decay": 0.0}], lr=lr,
                          momentum=0.0, foreach=False)
    for step in range(20):
        g = f16(rng.standard_normal(n1 + n2) * (0.05 if step % 2 else 1e-3))
        info = sh.step([g], lr)
        gd = torch.from_numpy(dec_f16(g))
        p1.grad, p2.grad = gd[:n1].clone(), gd[n1:].clone()
        torch.nn.utils.clip_grad_norm_([p1, p2], 1.0, foreach=False)
        opt.step()
    ref = torch.cat([p1.detach(), p2.detach()]).numpy()
    np.testing.assert_allclose(sh.master, ref, rtol=1e-5, atol=1e-7)


def test_sgd_closed_form_and_untouched_moments(orc):
    """wd = 0, clipping off, scale 1: one SGD step is p - lr*g to within the
    two roundings; m and v stay zero."""
    n, lr = 5000, 1e-2
    rng = np.random.default_rng(32)
    master = (rng.standard_normal(n) * 0.02).astype(np.float32)
    sh = orc.OracleShard(master, orc.OracleHparams(clip_norm=0.0, init_scale=1.0, optimizer=1), default_wd=0.0)
    g = f16(rng.standard_normal(n))
    sh.step([g], lr)
    expect = master.astype(np.float64) - F32(lr) * dec_f16(g)
    np.testing.assert_allclose(sh.master, expect, rtol=2.0 ** -22, atol=lr * 2.0 ** -22)
    assert not sh.m.any() and not sh.v.any()
    np.testing.assert_array_equal(sh.w, f16(sh.master))


@pytest.mark.parametrize("optimizer", [0, 1])
def test_threaded_step_equals_single_threaded(orc, optimizer):
    """The oracle split over host threads by contiguous chunks (the CPU
    baseline on all cores) gives the single-threaded step's state byte for
    byte, across segment and chunk boundaries and through an overflow; the
    norm differs only by the re-association of the chunk sums."""
    import synth
    n = 100_003
    segs = [(0, 40_000, 0.1), (40_000, 3, 0.0), (40_003, n - 40_003, 0.1)]
    hp = orc.OracleHparams(clip_norm=1.0, init_scale=2.0 ** 12, scale_window=2, optimizer=optimizer)
    master = synth.master_normal(n, 0.02, 5)
    a = orc.OracleShard(master, hp, wbf16=True, gbf16=False, segments=segs)
    b = orc.OracleShard(master, hp, wbf16=True, gbf16=False, segments=segs)
    for s in range(1, 6):
        g = synth.grad_normal16(n, 1e-3, a.scale, 5, 0, s)
        if s == 3:
            g[70_001] = 0x7C00
        ia = a.step([g], 1e-3)
        ib = b.step_threaded([g], 1e-3, threads=4, chunk=7_777)
        assert (ia.overflow, ia.scale_next, ia.t) == (ib.overflow, ib.scale_next, ib.t)
        assert ia.overflow == (1 if s == 3 else 0)
        if not ia.overflow:
            assert abs(ia.norm - ib.norm) <= 1e-12 * ia.norm
            assert ia.coef == ib.coef   # on these inputs the re-association does not reach the FP32 coefficient
    for x, y in ((a.master, b.master), (a.m, b.m), (a.v, b.v), (a.w, b.w)):
        assert x.tobytes() == y.tobytes()
