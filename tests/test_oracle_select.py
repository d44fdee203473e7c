"""Pins for the oracle's importance update and top-k rank choice.

Checked by brute force (a token is selected iff fewer than k tokens beat it
under (key desc, index asc)), by constructed ties, -0/+0, NaN, and by the
moving average on values where one fp32 rounding is known exactly.
"""
import numpy as np
import pytest

import oracle


def _brute_force_bits(key, k):
    T = len(key)
    kk = np.where(np.isnan(key), -np.inf, key).astype(np.float64)
    nan = np.isnan(key)
    sel = np.zeros(T, dtype=bool)
    for t in range(T):
        better = 0
        for s in range(T):
            if s == t:
                continue
            if nan[t] and not nan[s]:
                better += 1
            elif nan[t] == nan[s] and not nan[t]:
                if kk[s] > kk[t] or (kk[s] == kk[t] and s < t):
                    better += 1
            elif nan[t] and nan[s] and s < t:
                better += 1
        sel[t] = better < k
    return sel


@pytest.mark.parametrize("T,k,seed", [(1, 1, 0), (7, 3, 1), (32, 8, 2), (33, 9, 3), (100, 25, 4), (70, 70, 5),
                                      (70, 0, 6), (45, 60, 7)])
def test_select_matches_brute_force(T, k, seed):
    g = np.random.default_rng(seed)
    mass = g.random(T).astype(np.float32)
    mask, _ = oracle.select(mass, k)
    np.testing.assert_array_equal(oracle.mask_bits(mask, T)[0], _brute_force_bits(mass, k))


def test_ties_go_to_lower_index():
    mass = np.array([0.5, 0.2, 0.5, 0.5, 0.1, 0.5], dtype=np.float32)
    mask, _ = oracle.select(mass, 2)
    assert list(np.nonzero(oracle.mask_bits(mask, 6)[0])[0]) == [0, 2]
    mask, _ = oracle.select(mass, 3)
    assert list(np.nonzero(oracle.mask_bits(mask, 6)[0])[0]) == [0, 2, 3]


def test_negative_zero_equals_positive_zero_and_nan_is_lowest():
    mass = np.array([np.nan, -0.0, 0.0, -1.0, np.nan, 0.0], dtype=np.float32)
    mask, _ = oracle.select(mass, 3)
    # 0.0 ties among {1 (-0), 2, 5}; -1 and NaN below
    assert list(np.nonzero(oracle.mask_bits(mask, 6)[0])[0]) == [1, 2, 5]
    mask, _ = oracle.select(mass, 5)
    assert list(np.nonzero(oracle.mask_bits(mask, 6)[0])[0]) == [0, 1, 2, 3, 5]


def test_bits_past_T_are_clear_and_count_is_k():
    g = np.random.default_rng(9)
    T = 77
    mass = g.random((3, T)).astype(np.float32)
    mask, _ = oracle.select(mass, 20)
    assert mask.shape == (3, 3)
    for u in range(3):
        assert int(np.unpackbits(mask[u].view(np.uint8)).sum()) == 20
        assert mask[u, 2] >> (T - 64) == 0


def test_moving_average_update():
    """alpha = 0.5: key = fma(0.5, s, 0.5 m); 0.5 s is exact, so it equals one fp32 rounding of s/2 + m/2."""
    g = np.random.default_rng(4)
    m = g.random(40).astype(np.float32)
    s = g.random(40).astype(np.float32)
    mask, new = oracle.select(m, 10, alpha=0.5, score=s)
    expect = (np.float32(0.5) * s + np.float32(0.5) * m).astype(np.float32)
    np.testing.assert_array_equal(new[0], expect)
    np.testing.assert_array_equal(oracle.mask_bits(mask, 40)[0], _brute_force_bits(expect, 10))


def test_alpha_zero_ignores_previous_score():
    m = np.array([0.1, 0.9, 0.3], dtype=np.float32)
    s = np.array([np.inf, np.nan, -5.0], dtype=np.float32)
    mask, new = oracle.select(m, 1, alpha=0.0, score=s)
    np.testing.assert_array_equal(new[0], m)
    assert list(np.nonzero(oracle.mask_bits(mask, 3)[0])[0]) == [1]
