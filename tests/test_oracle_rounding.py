"""Pins for the oracle's storage rounding (CPU only)."""

import numpy as np
import torch

from oracle import rounding


def test_bf16_matches_library_on_binary32_inputs():
    """For values that are exact binary32 numbers, fp64 -> bf16 rounding must
    equal torch's binary32 -> bfloat16 round-to-nearest-even."""
    rng = np.random.default_rng(0)
    x32 = np.concatenate([
        rng.standard_normal(200000).astype(np.float32),
        (rng.standard_normal(20000) * 1e-30).astype(np.float32),
        (rng.standard_normal(20000) * 1e30).astype(np.float32),
        np.array([0.0, -0.0, 1.0, -1.0, 3.0e38], dtype=np.float32),
    ])
    ours = rounding.bf16_bits(x32.astype(np.float64))
    lib = torch.from_numpy(x32).to(torch.bfloat16).view(torch.int16).numpy().view(np.uint16)
    assert np.array_equal(ours, lib)


def test_bf16_ties_go_to_even():
    one = 1.0
    ulp = 2.0 ** -7                        # bf16 spacing in [1, 2)
    # halfway between 1 and 1+ulp -> 1 (even); between 1+ulp and 1+2ulp -> 1+2ulp
    assert rounding.to_bf16(one + ulp / 2) == one
    assert rounding.to_bf16(one + 1.5 * ulp) == one + 2 * ulp
    # just above halfway rounds up
    assert rounding.to_bf16(one + ulp / 2 + 2.0 ** -40) == one + ulp
    assert rounding.to_bf16(-(one + ulp / 2 + 2.0 ** -40)) == -(one + ulp)


def test_bf16_rounds_fp64_directly_not_through_fp32():
    # x lies just above a bf16 tie; rounding to fp32 first would land exactly on
    # the tie and then go to even (down).  Direct rounding must go up.
    x = 1.0 + 2.0 ** -8 + 2.0 ** -40
    assert rounding.to_bf16(x) == 1.0 + 2.0 ** -7


def test_bits_roundtrip():
    rng = np.random.default_rng(1)
    v = rounding.to_bf16(rng.standard_normal(1000))
    assert np.array_equal(rounding.from_bf16_bits(rounding.bf16_bits(v)), v)
