"""Pins for the oracle's batched entry points and for the pages' decompression-FLOP figure.

* Batched calls over U = 3 different units give exactly what one call per
  unit gives (decode, select with a moving average, compress): a wrong
  per-unit offset in a batched routine would mix units and fail here.
* The decompression work of a step is proportional to the sum of the
  per-token ranks.  With all-ones coefficients, a basis that copies a sum of
  coefficients into one output feature and a zero query (uniform attention),
  the oracle's output equals the mean rank; the es summary's sensitivity
  analysis (§4) puts the cut at 67.5 %, which the arithmetic gives for 10 %
  of the tokens at full rank, and 56.25 % for 25 %.
"""
import numpy as np
import pytest

import oracle


def _units(seed, U, T, L, Hg, r=64):
    g = np.random.default_rng(seed)
    CK = g.standard_normal((U, T, r)) * (0.9 ** np.arange(r))
    CV = g.standard_normal((U, T, r)) * (0.9 ** np.arange(r))
    BK = np.stack([np.linalg.qr(g.standard_normal((512, r)))[0].T for _ in range(U)])
    BV = np.stack([np.linalg.qr(g.standard_normal((512, r)))[0].T for _ in range(U)])
    Kt = g.standard_normal((U, L, 4, 128))
    Vt = g.standard_normal((U, L, 4, 128))
    q = g.standard_normal((U, Hg, 128)) / np.sqrt(128)
    mask = g.integers(0, 2 ** 32, size=(U, (T + 31) // 32), dtype=np.uint64).astype(np.uint32)
    return CK, BK, CV, BV, Kt, Vt, mask, q


@pytest.mark.parametrize("r_lo", [16, 0])
def test_batched_decode_equals_per_unit_calls(r_lo):
    U, T, L, Hg = 3, 70, 9, 8
    CK, BK, CV, BV, Kt, Vt, mask, q = _units(11, U, T, L, Hg)
    out, mass = oracle.decode(CK, BK, CV, BV, Kt, Vt, mask, q, r_lo=r_lo, scale=0.9)
    for u in range(U):
        sl = slice(u, u + 1)
        o1, m1 = oracle.decode(CK[sl], BK[sl], CV[sl], BV[sl], Kt[sl], Vt[sl], mask[sl], q[sl], r_lo=r_lo,
                               scale=0.9)
        assert np.array_equal(out[u], o1[0])
        assert np.array_equal(mass[u], m1[0])
    # the units really differ, so a mix-up would show
    assert not np.allclose(out[0], out[1])


def test_batched_select_equals_per_unit_calls():
    U, T, k = 3, 100, 23
    g = np.random.default_rng(5)
    mass = g.random((U, T)).astype(np.float32)
    score = g.random((U, T)).astype(np.float32)
    mask, sc = oracle.select(mass, k, alpha=0.3, score=score)
    for u in range(U):
        m1, s1 = oracle.select(mass[u:u + 1], k, alpha=0.3, score=score[u:u + 1])
        assert np.array_equal(mask[u], m1[0])
        assert np.array_equal(sc[u], s1[0])
    assert not np.array_equal(mask[0], mask[1])


def test_batched_compress_equals_per_unit_calls():
    U, T = 3, 90
    g = np.random.default_rng(9)
    X = g.standard_normal((U, T, 512)) * np.linspace(2.0, 0.1, 512)
    C, B, sig = oracle.compress(X, r=64)
    for u in range(U):
        C1, B1, s1 = oracle.compress(X[u:u + 1], r=64)
        assert np.array_equal(C[u], C1[0])
        assert np.array_equal(B[u], B1[0])
        assert np.array_equal(sig[u], s1[0])
    assert not np.allclose(sig[0], sig[1])


@pytest.mark.parametrize("frac,cut", [(0.25, 0.5625), (0.10, 0.675)])
def test_decompression_flop_cut(frac, cut):
    T, Hg, r = 640, 4, 64
    k = int(np.ceil(frac * T))
    g = np.random.default_rng(3)
    mask, _ = oracle.select(g.random((1, T)).astype(np.float32), k)
    assert int(sum(bin(int(w)).count("1") for w in mask[0])) == k
    CK = np.ones((1, T, r))
    CV = np.ones((1, T, r))
    BK = np.zeros((1, r, 512))
    BV = np.zeros((1, r, 512))
    BV[0, :, 0] = 1.0                    # feature 0 of KV head 0 = sum of the token's kept coefficients
    q = np.zeros((1, Hg, 128))           # zero logits: uniform attention over the T tokens
    Kt = np.zeros((1, 0, 4, 128))
    out, _ = oracle.decode(CK, BK, CV, BV, Kt, Kt, mask, q, r_lo=16)
    mean_rank = out[0, 0, 0]             # = sum_t rho_t / T
    assert abs(mean_rank - (k * 64 + (T - k) * 16) / T) < 1e-12
    assert abs((1.0 - mean_rank / r) - cut) < 1e-12
