"""The five shard workloads, as seeded synthetic recipes (sizes, layouts, value
distributions, hyperparameters, step counts and scripted overflows).

No dataset is involved: the step consumes gradients only, and the gradients
here are drawn from the distributions the workloads state (normal or
Student-t values times the loss scale, rounded to the 16-bit type).
"""
from __future__ import annotations

from dataclasses import dataclass, field


@dataclass
class Workload:
    name: str
    numel: int
    K: int = 1                    # gradient buffers per step
    bf16: bool = False            # 16-bit type of weights and grads
    grad_dist: str = "normal"     # "normal" or "t3"
    grad_sigma: float = 1e-3      # std of the true (unscaled) gradient (normal)
    init_scale: float = 2.0 ** 16
    scale_window: int = 1000
    lr: float = 6e-4
    beta1: float = 0.9
    beta2: float = 0.95
    eps: float = 1e-8
    weight_decay: float = 0.1
    clip: float = 1.0
    predivide: float = 1.0
    steps: int = 10
    elem_offset: int = 0          # element offset of every array from a 256-byte boundary
    inject_steps: tuple = ()      # 1-based calls with one scripted non-finite value
    inject_rate: float = 0.0      # per-element injection probability ...
    inject_rate_steps: tuple = () # ... on these calls
    segments: list | None = None  # [(offset, numel, wd, init)] ; init in {"normal", "zero", "one"}
    master_sigma: float = 0.02
    bench_scale: float | None = None  # loss scale for throughput runs (None: init_scale)
    seed: int = 0
    cfg_id: int = 0
    extra: dict = field(default_factory=dict)

    def seg_table(self):
        if self.segments is None:
            return None
        return [(o, c, w) for o, c, w, _ in self.segments]


def pythia_like_segments(layers=24, hidden=2048, vocab=50304, ffn_mult=4):
    """Flat layout of a GPT-NeoX / Pythia-style decoder: embedding, `layers`
    blocks (LayerNorm, fused QKV, attention output, LayerNorm, MLP in/out, all
    with biases), un-embedding.  Biases and LayerNorm parameters get wd = 0."""
    segs = []
    off = 0

    def add(n, wd, init):
        nonlocal off
        segs.append((off, n, wd, init))
        off += n

    add(vocab * hidden, 0.1, "normal")
    ffn = ffn_mult * hidden
    for _ in range(layers):
        add(hidden, 0.0, "one")              # LN1 weight
        add(hidden, 0.0, "zero")             # LN1 bias
        add(hidden * 3 * hidden, 0.1, "normal")  # QKV weight
        add(3 * hidden, 0.0, "zero")         # QKV bias
        add(hidden * hidden, 0.1, "normal")  # attention dense weight
        add(hidden, 0.0, "zero")             # dense bias
        add(hidden, 0.0, "one")              # LN2 weight
        add(hidden, 0.0, "zero")             # LN2 bias
        add(hidden * ffn, 0.1, "normal")     # MLP h->4h weight
        add(ffn, 0.0, "zero")                # bias
        add(ffn * hidden, 0.1, "normal")     # MLP 4h->h weight
        add(hidden, 0.0, "zero")             # bias
    add(vocab * hidden, 0.1, "normal")
    return segs


def tiny() -> Workload:
    """1,048,576-element FP16 shard, N(0,1e-3) x 2^16 grads, an inf on call 4, window 2."""
    return Workload("tiny_1M_fp16", 1 << 20, grad_sigma=1e-3, init_scale=2.0 ** 16, scale_window=2,
                    steps=10, inject_steps=(4,), cfg_id=0)


def pythia_1p4b(layers=24, hidden=2048, vocab=50304) -> Workload:
    """Pythia-1.4B-shaped multi-tensor shard: 290 segments, wd 0 on biases / LayerNorms."""
    segs = pythia_like_segments(layers, hidden, vocab)
    n = segs[-1][0] + segs[-1][1]
    return Workload(f"pythia_1.4b_shaped_{layers}layer_fp16" if layers != 24 else "pythia_1.4b_shaped_fp16", n, grad_sigma=1e-4,
                    init_scale=2.0 ** 12, scale_window=1000, steps=10, segments=segs, cfg_id=1)


def neox20b_zero1_slice(numel=2_570_000_001) -> Workload:
    """Flat ZeRO-1 slice of a GPT-NeoX-20B-shaped buffer at DP=8, element offset 3."""
    return Workload("neox20b_dp8_slice_fp16", numel, grad_sigma=5e-5, init_scale=2.0 ** 16, scale_window=1000,
                    steps=50, elem_offset=3, cfg_id=2)


def accum8_predivide(numel=268_435_456) -> Workload:
    """K = 8 FP16 buffers of Student-t(3) x 2^10, predivide 8, clip 0.3, natural
    overflow plus 1e-7/element injection on calls 20 and 25."""
    # At 2^10 about 18,000 of the 2.1e9 FP16 values overflow per call and the
    # scaler walks down; throughput runs use 2^2, below where it settles (about
    # 0.001 expected overflows per call), so that every timed call is applied.
    return Workload("accum8_t3_predivide8_fp16", numel, K=8, grad_dist="t3", init_scale=2.0 ** 10,
                    predivide=8.0, clip=0.3, steps=30, inject_rate=1e-7, inject_rate_steps=(20, 25), cfg_id=3,
                    bench_scale=2.0 ** 2)


def opt_style_5b(numel=5_000_000_000) -> Workload:
    """OPT-175B-style ZeRO shard: BF16 weights and grads, N(0,1e-5) grads, lr 1.2e-4,
    clip 0.3, 100 calls, scripted overflows on calls 3, 4, 57."""
    return Workload("opt_style_5e9_bf16", numel, bf16=True, grad_sigma=1e-5, init_scale=2.0 ** 16,
                    scale_window=1000, lr=1.2e-4, clip=0.3, steps=100, inject_steps=(3, 4, 57), cfg_id=4)


def pythia_2layer() -> Workload:
    """The Pythia-1.4B layout cut to 2 layers (306,761,728 params, 4.9 GB of
    state): the same kernels and segment kinds at a size that detailed
    profiler captures handle."""
    return pythia_1p4b(layers=2)


def opt_5b_cut() -> Workload:
    """The OPT-style recipe at 2^28 parameters (4.8 GB on the device): the BF16
    kernel instances of the 5e9-element shard at a size that detailed profiler
    captures handle."""
    import dataclasses
    return dataclasses.replace(opt_style_5b(numel=1 << 28), name="opt_style_bf16_2e28")


def accum8_small() -> Workload:
    """The 8-buffer recipe at 2^26 parameters (2.4 GB on the device with the
    FP32 sum buffer): a size that detailed profiler captures handle."""
    import dataclasses
    return dataclasses.replace(accum8_predivide(numel=1 << 26), name="accum8_t3_predivide8_fp16_2e26")


ALL = {"tiny": tiny, "pythia_1p4b": pythia_1p4b, "neox20b_slice": neox20b_zero1_slice,
       "accum8": accum8_predivide, "opt_5b": opt_style_5b, "pythia_2layer": pythia_2layer,
       "accum8_small": accum8_small, "opt_5b_cut": opt_5b_cut}
