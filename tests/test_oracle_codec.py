"""Pins of the oracle's 16-bit codecs (the a11 cast and the grad decode).

The oracle writes IEEE-754 binary16 / bfloat16 rounding itself; these tests
compare it with the library casts of torch (CPU, round-to-nearest-even)
exhaustively over every binary32 bit pattern and every 16-bit code.
"""
from concurrent.futures import ThreadPoolExecutor

import numpy as np
import pytest
import torch


def _lib_cast(x32: np.ndarray, dtype) -> np.ndarray:
    return torch.from_numpy(x32).to(dtype).view(torch.int16).numpy().view(np.uint16)


def _is_nan16(h: np.ndarray, bf16: bool) -> np.ndarray:
    if bf16:
        return ((h & 0x7F80) == 0x7F80) & ((h & 0x007F) != 0)
    return ((h & 0x7C00) == 0x7C00) & ((h & 0x03FF) != 0)


@pytest.mark.parametrize("bf16", [False, True], ids=["fp16", "bf16"])
def test_encode_exhaustive_all_f32_patterns(orc, bf16):
    """Every one of the 2^32 binary32 inputs rounds like torch's RNE cast
    (NaN inputs: both sides give a NaN code)."""
    base = np.arange(1 << 24, dtype=np.uint32)
    dtype = torch.bfloat16 if bf16 else torch.float16
    enc = orc.bf16_encode if bf16 else orc.f16_encode

    def chunk(hi):
        x = (base | np.uint32(hi << 24)).view(np.float32)
        a = enc(x)
        r = _lib_cast(x, dtype)
        nan_in = np.isnan(x)
        ok = (a == r) | (nan_in & _is_nan16(a, bf16) & _is_nan16(r, bf16))
        bad = np.flatnonzero(~ok)
        return hi, bad[:4], int(bad.size)

    with ThreadPoolExecutor(8) as ex:
        for hi, first, nbad in ex.map(chunk, range(256)):
            assert nbad == 0, f"chunk {hi:#x}: {nbad} mismatches, first offsets {first}"


@pytest.mark.parametrize("bf16", [False, True], ids=["fp16", "bf16"])
def test_decode_exhaustive_all_codes(orc, bf16):
    h = np.arange(1 << 16, dtype=np.uint32).astype(np.uint16)
    ours = orc.bf16_decode(h) if bf16 else orc.f16_decode(h)
    dtype = torch.bfloat16 if bf16 else torch.float16
    ref = torch.from_numpy(h.view(np.int16)).view(dtype).to(torch.float32).numpy()
    both_nan = np.isnan(ours) & np.isnan(ref)
    assert np.all((ours.view(np.uint32) == ref.view(np.uint32)) | both_nan)
    # NaN codes decode to NaN and nothing else does
    assert np.array_equal(np.isnan(ours), _is_nan16(h, bf16))


def test_encode_boundaries_fp16(orc):
    """Hand-checked binary16 facts: largest finite 65504, the overflow
    threshold 65520 (halfway to 2^16 rounds up to inf), smallest subnormal
    2^-24, and the tie at 2^-25 rounding to even (zero)."""
    cases = {
        65504.0: 0x7BFF, 65519.996: 0x7BFF, 65520.0: 0x7C00, -65520.0: 0xFC00,
        2.0 ** -24: 0x0001, 2.0 ** -25: 0x0000, 1.5 * 2.0 ** -25: 0x0001,
        3 * 2.0 ** -25: 0x0002,  # tie between codes 1 and 2 -> even (2)
        2.0 ** -14: 0x0400, 1.0: 0x3C00, 1.0 + 2.0 ** -11: 0x3C00,  # tie -> even
        1.0 + 3 * 2.0 ** -11: 0x3C02, -0.0: 0x8000,
    }
    x = np.array(list(cases.keys()), np.float32)
    got = orc.f16_encode(x)
    assert [int(v) for v in got] == list(cases.values())


def test_encode_boundaries_bf16(orc):
    cases = {
        1.0: 0x3F80, 1.0 + 2.0 ** -8: 0x3F80, 1.0 + 3 * 2.0 ** -8: 0x3F82,
        3.3895313892515355e38: 0x7F7F, 3.4028234663852886e38: 0x7F80, -0.0: 0x8000,
    }
    x = np.array(list(cases.keys()), np.float32)
    got = orc.bf16_encode(x)
    assert [int(v) for v in got] == list(cases.values())
