"""Pins for the oracle's bf16 conversions.

Widening is checked against the IEEE bit layout; rounding against torch's
binary32 -> bf16 conversion (ties to even) on values that are exact in
binary32, where one rounding from binary64 must agree, and against cases
worked by hand where a detour through binary32 would round twice.
"""
import numpy as np
import torch

import oracle


def test_widening_is_exact():
    bits = np.arange(0, 1 << 16, 7, dtype=np.uint16)
    with np.errstate(invalid="ignore"):      # signalling-NaN patterns widen to NaN
        ref = (bits.astype(np.uint32) << 16).view(np.float32).astype(np.float64)
    got = oracle.bf16_to_f64(bits)
    same = (got == ref) | (np.isnan(got) & np.isnan(ref))
    assert same.all()


def test_rounding_matches_torch_on_binary32_values():
    g = np.random.default_rng(0)
    x = np.concatenate([
        g.standard_normal(20000).astype(np.float32) * np.float32(10.0) ** g.integers(-30, 30, 20000),
        (np.arange(1, 4000, dtype=np.uint32) << 13).view(np.float32),      # many exact ties
        np.array([1e-40, -3e-39, 3.4e38, -3.39e38, 0.0, -0.0], dtype=np.float32),
    ])
    ref = torch.from_numpy(x).to(torch.bfloat16).view(torch.int16).numpy().view(np.uint16)
    got = oracle.f64_to_bf16(x.astype(np.float64))
    np.testing.assert_array_equal(got, ref)


def test_single_rounding_from_binary64():
    # 1 + 2^-8 + 2^-30 is just above the tie between 1 and 1 + 2^-7: one rounding gives 1 + 2^-7
    # (0x3f81); through binary32 it would first become the exact tie and then round to even, 1.0.
    assert oracle.f64_to_bf16(np.array([1 + 2.0 ** -8 + 2.0 ** -30]))[0] == 0x3F81
    assert oracle.f64_to_bf16(np.array([1 + 2.0 ** -8]))[0] == 0x3F80          # tie -> even
    assert oracle.f64_to_bf16(np.array([1 + 3 * 2.0 ** -8]))[0] == 0x3F82      # tie -> even (up)
    assert oracle.f64_to_bf16(np.array([np.inf, -np.inf]))[0] == 0x7F80
    assert oracle.f64_to_bf16(np.array([3.5e38]))[0] == 0x7F80                  # overflow
    assert oracle.f64_to_bf16(np.array([-0.0]))[0] == 0x8000
