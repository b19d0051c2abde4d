"""The oracle's pins catch planted mistakes.

Each case copies ``oracle/oracle.c`` to a temporary directory, plants one
plausible mistake (a dropped term, a wrong sign, a swapped operand, an
off-by-one, a wrong rounding), builds it, routes the oracle module to that
build and runs the pins of ``test_oracle_step.py`` / ``test_oracle_codec.py``.
At least one pin must fail for every mutant.  Nothing here touches a GPU.
"""
import os
import subprocess

import numpy as np
import pytest

import oracle
from tests import test_oracle_codec as tc
from tests import test_oracle_step as ts

SRC = os.path.join(os.path.dirname(oracle.__file__), "oracle.c")

# (name, text in oracle.c, replacement)
MUTANTS = [
    ("predivide dropped", "float term = dec16(g[k][j], gbf16) * inv_pre;", "float term = dec16(g[k][j], gbf16);"),
    ("unscale dropped", "    return a * inv_us;\n}", "    return a;\n}"),
    ("only first buffer", "for (int32_t k = 0; k < K; k++) {\n        float term", "for (int32_t k = 0; k < 1; k++) {\n        float term"),
    ("post ignores predivide", "double post = (double)K / (double)predivide;", "double post = (double)K;"),
    ("m decays with beta2", "float mj = b1 * m[j];", "float mj = b2 * m[j];"),
    ("m gain beta1", "mj = mj + omb1 * gh;", "mj = mj + b1 * gh;"),
    ("v not squared", "vj = vj + gg * gh;", "vj = vj + gg;"),
    ("v gain 1-beta1", "float gg = omb2 * gh;", "float gg = omb1 * gh;"),
    ("bc2 dropped", "float den = sqrtf(vj) / bcs;", "float den = sqrtf(vj);"),
    ("eps dropped", "den = den + eps;", "den = den + 0.0f;"),
    ("decay sign", "float keep = 1.0f - lrwd;", "float keep = 1.0f + lrwd;"),
    ("decay dropped", "p = p * keep;", "p = p * 1.0f;"),
    ("update sign", "p = p - step_size * upd;", "p = p + step_size * upd;"),
    ("clip ignored", "float gh = gj * c;", "float gh = gj;"),
    ("bias correction t+1", "double bc1 = 1.0 - pow((double)hp->beta1, (double)sc->t);",
     "double bc1 = 1.0 - pow((double)hp->beta1, (double)(sc->t + 1));"),
    ("step uses bc2", "info->step_size = (float)((double)lr / bc1);", "info->step_size = (float)((double)lr / bc2);"),
    ("norm not rooted", "    double norm = sqrt(sumsq);\n    if (!overflow", "    double norm = sumsq;\n    if (!overflow"),
    ("clip margin dropped", "double c = (double)clip / (norm + 1e-6);", "double c = (double)clip / norm;"),
    ("inf not detected", "        if (!isfinite(x))\n            bad++;", "        if (isnan(x))\n            bad++;"),
    ("overflow applies update", "    if (!info->overflow) {\n        if (hp->optimizer == 1)",
     "    if (1) {\n        if (hp->optimizer == 1)"),
    ("overflow advances t", "        info->coef = 0.0f;\n        info->t = sc->t;", "        info->coef = 0.0f;\n        sc->t += 1;\n        info->t = sc->t;"),
    ("backoff grows", "float s = sc->scale / hp->scale_factor;", "float s = sc->scale * hp->scale_factor;"),
    ("counter kept on overflow", "    if (overflow) {\n        sc->good = 0;\n", "    if (overflow) {\n"),
    ("growth counter not reset", "            sc->scale = s;\n        sc->good = 0;", "            sc->scale = s;"),
    ("floor ignored", "sc->scale = s > hp->min_scale ? s : hp->min_scale;", "sc->scale = s;"),
    ("segment lookup off by one", "if (segs[mid].offset <= idx) lo = mid;", "if (segs[mid].offset < idx) lo = mid;"),
    ("f16 truncates", "uint32_t q = rne(sig >> 13, sig & 0x1fffu, 0x1000u);", "uint32_t q = sig >> 13;"),
    ("ties away from zero", "if (rem > half || (rem == half && (q & 1u)))", "if (rem >= half)"),
    ("f16 subnormal scale", "mag = ldexpf((float)frac, -24);", "mag = ldexpf((float)frac, -25);"),
    ("bf16 no rounding", "return (uint16_t)rne(x >> 16, x & 0xffffu, 0x8000u);", "return (uint16_t)(x >> 16);"),
    ("hysteresis ignored", "        if (sc->hyst == 0) {", "        if (1) {"),
    ("hysteresis never refilled", "        sc->hyst = orc_hysteresis(hp);", "        sc->hyst = 1;"),
    ("sgd step sign", "        q = q - delta;", "        q = q + delta;"),
    ("sgd ignores clip", "        float g_clipped = gj * c;", "        float g_clipped = gj;"),
    ("sgd decay dropped", "        q = q * retain;", "        q = q * 1.0f;"),
]

# pins run against each mutant, cheapest first
PINS = [
    (tc.test_encode_boundaries_fp16, {}),
    (tc.test_encode_boundaries_bf16, {}),
    (tc.test_decode_exhaustive_all_codes, {"bf16": False}),
    (ts.test_zero_grad_only_decays, {}),
    (ts.test_first_step_eps0_is_sign_update, {"wd": 0.1}),
    (ts.test_constant_grad_bias_corrected_update, {}),
    (ts.test_norm_closed_form_power_of_two, {}),
    (ts.test_predivide_gives_exact_mean, {"K": 8, "pre": 8.0, "S": 2.0 ** 10}),
    (ts.test_predivide_gives_exact_mean, {"K": 4, "pre": 2.0, "S": 2.0 ** 3}),
    (ts.test_clip_coefficient_invariants, {}),
    (ts.test_step_applies_clip_to_moments, {}),
    (ts.test_overflow_skips_and_backs_off, {"bad": np.inf}),
    (ts.test_unscale_overflow_counts, {}),
    (ts.test_nonfinite_count_exact, {}),
    (ts.test_skipped_step_does_not_advance_t, {}),
    (ts.test_scaler_trajectory_golden, {"name": "tiny"}),
    (ts.test_scaler_floor, {}),
    (ts.test_scaler_matches_torch_gradscaler, {}),
    (ts.test_matches_torch_adamw_float64, {}),
    (ts.test_fp32_oracle_tracks_float64_brute_force, {"gbf16": False, "K": 3, "pre": 2.0}),
    (ts.test_scaler_hysteresis_golden, {}),
    (ts.test_sgd_matches_torch_float64, {}),
    (ts.test_sgd_closed_form_and_untouched_moments, {}),
]


def test_mutant_table_applies():
    src = open(SRC).read()
    for name, old, _ in MUTANTS:
        assert src.count(old) == 1, f"mutant '{name}' does not match oracle.c exactly once"


@pytest.mark.parametrize("name,old,new", MUTANTS, ids=[m[0] for m in MUTANTS])
def test_pins_catch_mutant(tmp_path, name, old, new):
    src = open(SRC).read()
    assert src.count(old) == 1
    mut = tmp_path / "oracle_mutant.c"
    mut.write_text(src.replace(old, new))
    so = tmp_path / "liboracle_mutant.so"
    subprocess.check_call(["gcc", *oracle._CFLAGS, "-o", str(so), str(mut), "-lm"])
    caught = None
    with oracle.use_library(str(so)):
        for fn, kw in PINS:
            try:
                with np.errstate(all="ignore"):
                    fn(oracle, **kw)
            except (AssertionError, ValueError, FloatingPointError) as e:
                caught = f"{fn.__name__}: {type(e).__name__}"
                break
    assert caught is not None, f"no pin caught mutant '{name}'"
