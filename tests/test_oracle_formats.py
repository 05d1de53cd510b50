"""Pins for the oracle's number-format helpers against library conversions.

bf16 and binary16 values are checked for all 65536 bit patterns against
torch / numpy; bf16 rounding against torch's float32 -> bfloat16 conversion
(a single rounding for float32-representable inputs) and constructed ties.
"""
import math

import numpy as np
import pytest
import torch

import oracle

ALL = np.arange(1 << 16, dtype=np.uint32).astype(np.uint16)


def test_bf16_value_all_patterns():
    ref = torch.from_numpy(ALL.view(np.int16)).view(torch.bfloat16).to(torch.float64).numpy()
    got = np.array([oracle.bf16_value(int(h)) for h in ALL])
    nan = np.isnan(ref)
    assert np.array_equal(np.isnan(got), nan)
    assert np.array_equal(got[~nan], ref[~nan])


def test_fp16_value_all_patterns():
    ref = ALL.view(np.float16).astype(np.float64)
    got = np.array([oracle.fp16_value(int(h)) for h in ALL])
    nan = np.isnan(ref)
    assert np.array_equal(np.isnan(got), nan)
    assert np.array_equal(got[~nan], ref[~nan])


def test_bf16_round_matches_torch_on_float32_inputs():
    rng = np.random.default_rng(5)
    bits = rng.integers(0, 1 << 32, size=20000, dtype=np.uint64).astype(np.uint32)
    f = bits.view(np.float32)
    f = f[np.isfinite(f)]
    ref = torch.from_numpy(f).to(torch.bfloat16).view(torch.int16).numpy().view(np.uint16)
    got = np.array([oracle.bf16_round(float(v)) for v in f], dtype=np.uint16)
    assert np.array_equal(got, ref)


def test_bf16_round_ties_to_even():
    # 1 + 2^-8 is halfway between 1 and 1 + 2^-7: even is 1.0 (0x3F80)
    assert oracle.bf16_round(1.0 + 2.0 ** -8) == 0x3F80
    # 1 + 3*2^-8 is halfway between 1+2^-7 (odd) and 1+2^-6 (even mantissa 2)
    assert oracle.bf16_round(1.0 + 3 * 2.0 ** -8) == 0x3F82
    # just above a tie rounds up
    assert oracle.bf16_round(1.0 + 2.0 ** -8 + 2.0 ** -40) == 0x3F81
    # subnormal boundary and overflow
    assert oracle.bf16_round(2.0 ** -134) == 0x0000          # tie below the smallest subnormal
    assert oracle.bf16_round(3 * 2.0 ** -134) == 0x0002      # 1.5 quanta -> 2 (even)
    assert oracle.bf16_round(-0.0) == 0x8000
    big = (2 - 2.0 ** -8) * 2.0 ** 127                      # halfway past the largest finite
    assert oracle.bf16_round(big) == 0x7F80
    assert oracle.bf16_round(math.nextafter(big, 0)) == 0x7F7F
    assert oracle.bf16_round(float("nan")) == 0x7FC0
