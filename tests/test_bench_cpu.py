"""bench.py's bookkeeping on CPU: the algorithmic bytes the roofline divides
by, and the source hash that ties recorded ncu counters to the kernel code."""
import os
import shutil

import pytest

import bench


def test_algorithmic_bytes_per_parameter():
    # AdamW, one 16-bit buffer: pass 1 reads the gradient; pass 2 reads it again
    # with master/m/v and writes master/m/v and the 16-bit weight
    assert bench.alg_bytes_per_param(1, False) == (2, 2 + 12 + 12 + 2)
    # eight buffers through the FP32 sum: pass 1 writes it, pass 2 reads it instead
    assert bench.alg_bytes_per_param(8, True) == (16 + 4, 4 + 12 + 12 + 2)
    # SGD leaves m and v alone
    assert bench.alg_bytes_per_param(1, False, sgd=True) == (2, 2 + 4 + 4 + 2)
    assert sum(bench.alg_bytes_per_param(1, False)) == 30


def test_source_hash_ignores_comments_but_not_code(tmp_path):
    copies = []
    for src in bench.KERNEL_SRCS:
        dst = tmp_path / os.path.basename(src)
        shutil.copy(src, dst)
        copies.append(str(dst))
    orig = bench.KERNEL_SRCS
    try:
        bench.KERNEL_SRCS = copies
        h0 = bench.kernel_source_hash()
        assert h0 == bench.kernel_source_hash() and len(h0) == 16
        with open(copies[0], "a") as f:
            f.write("\n// a comment\n/* a block\n   comment */\n\n   \n")
        assert bench.kernel_source_hash() == h0
        with open(copies[0], "a") as f:
            f.write("static int g_extra_symbol = 1;\n")
        assert bench.kernel_source_hash() != h0
    finally:
        bench.KERNEL_SRCS = orig


def test_zero2_plan_tiles_the_model():
    """Every rank's slice and segment table of the ZeRO-2 mode: equal slices
    that tile the model, segment tables that tile each slice with the
    model's weight decays, and the NVLink bytes of one step."""
    import bench
    from synth import workloads as W
    wl = W.pythia_1p4b()
    for world in (1, 2, 4, 8):
        covered = []
        for r in range(world):
            p = bench.zero2_plan(wl, world, r)
            assert p["n"] * world == wl.numel and p["lo"] == r * p["n"]
            pos = 0
            for off, cnt, wd in p["segments"]:
                assert off == pos and cnt > 0
                g = p["lo"] + off     # the model's segment containing this piece has the same decay
                src = [s for s in wl.segments if s[0] <= g < s[0] + s[1]][0]
                assert wd == src[2] and g + cnt <= src[0] + src[1]
                pos += cnt
            assert pos == p["n"]
            assert p["nvlink_read_bytes"] == p["nvlink_write_bytes"] == (world - 1) * 2 * p["n"]
            covered.append((p["lo"], p["n"]))
        assert sum(c for _, c in covered) == wl.numel
    with pytest.raises(ValueError):
        bench.zero2_plan(W.tiny(), 3, 0)


def test_parallel_generation_equals_one_call():
    """The reference arm draws its inputs in contiguous chunks on several
    threads; the counter-based generator makes that the same array as one
    call, chunk boundaries (not multiples of 4) included."""
    import numpy as np

    import synth
    n, lo = 50_021, 7
    one = synth.grad_normal16(n, 1e-3, 2.0 ** 12, 3, 1, 2, True, start=lo)
    par = bench.parallel_gen(synth.grad_normal16, n, 4, chunk=4_099, sigma=1e-3, scale=2.0 ** 12, seed=3,
                             tensor_id=1, step=2, bf16=True, start=lo)
    assert np.array_equal(one, par)
    m1 = synth.master_normal(n, 0.02, 5, start=lo)
    m2 = bench.parallel_gen(synth.master_normal, n, 3, chunk=10_001, sigma=0.02, seed=5, tensor_id=0, start=lo)
    assert np.array_equal(m1, m2)
