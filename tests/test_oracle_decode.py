"""Pins for the oracle's decode step (decompress at per-token rank, then attend).

Checks against closed forms (a single token, uniform attention, a dominant
key), against the rank-space route the pages' method reduces to by
associativity (q~ = B_K q, s = C_K q~, o = (sum p C_V) B_V) computed here in
numpy, and invariances (token permutation, r_lo = r, GQA head mapping).
"""
import math

import numpy as np
import pytest

import oracle


def _rand_unit(seed, T, L, Hg, r=64, hi_frac=0.25):
    g = np.random.default_rng(seed)
    CK = g.standard_normal((1, T, r)) * (0.9 ** np.arange(r))
    CV = g.standard_normal((1, T, r)) * (0.9 ** np.arange(r))
    BK = np.linalg.qr(g.standard_normal((512, r)))[0].T[None]
    BV = np.linalg.qr(g.standard_normal((512, r)))[0].T[None]
    Kt = g.standard_normal((1, L, 4, 128))
    Vt = g.standard_normal((1, L, 4, 128))
    q = g.standard_normal((1, Hg, 128)) / math.sqrt(128)
    bits = g.random(T) < hi_frac
    mask = np.zeros((1, (T + 31) // 32), dtype=np.uint32)
    for t in np.nonzero(bits)[0]:
        mask[0, t >> 5] |= np.uint32(1 << (t & 31))
    return CK, BK, CV, BV, Kt, Vt, mask, q, bits


def _rank_space_reference(CK, BK, CV, BV, Kt, Vt, bits, q, r_lo, scale):
    """The method's rank-space formulation, independent of the oracle's code path."""
    T, r = CK.shape
    Hg = q.shape[0]
    per = Hg // 4
    rho = np.where(bits, r, r_lo)
    cols = np.arange(r)[None, :] < rho[:, None]
    CKm, CVm = CK * cols, CV * cols
    out = np.zeros((Hg, 128))
    mass = np.zeros(T)
    for h in range(Hg):
        j = h // per
        sl = slice(j * 128, (j + 1) * 128)
        qt = BK[:, sl] @ q[h]                         # q~ = B_K[:, slice] q
        s = np.concatenate([CKm @ qt, Kt[:, j, :] @ q[h]]) * scale
        p = np.exp(s - s.max())
        p /= p.sum()
        u = p[:T] @ CVm                                # sum_t p_t C_V[t, :rho_t]
        out[h] = u @ BV[:, sl] + p[T:] @ Vt[:, j, :]
        mass += p[:T]
    return out, mass


@pytest.mark.parametrize("T,L,Hg", [(40, 7, 4), (64, 0, 16), (33, 12, 28), (1, 3, 8)])
def test_rank_space_equals_decompress_then_attend(T, L, Hg):
    CK, BK, CV, BV, Kt, Vt, mask, q, bits = _rand_unit(T * 7 + L, T, L, Hg)
    out, mass = oracle.decode(CK, BK, CV, BV, Kt, Vt, mask, q, r_lo=16, scale=1.3)
    ref_o, ref_m = _rank_space_reference(CK[0], BK[0], CV[0], BV[0], Kt[0], Vt[0], bits, q[0], 16, 1.3)
    np.testing.assert_allclose(out[0], ref_o, atol=1e-12, rtol=1e-10)
    np.testing.assert_allclose(mass[0], ref_m, atol=1e-13, rtol=1e-10)


def test_single_token_no_text_returns_its_value():
    """T = 1, L = 0: softmax weight 1, so o_h = Vhat_0[j(h)] and mass_0 = Hg."""
    CK, BK, CV, BV, Kt, Vt, mask, q, bits = _rand_unit(5, 1, 0, 8)
    mask[:] = 1
    out, mass = oracle.decode(CK, BK, CV, BV, Kt[:, :0], Vt[:, :0], mask, q)
    vhat = CV[0, 0] @ BV[0]                            # full rank: bit set
    for h in range(8):
        j = h // 2
        np.testing.assert_allclose(out[0, h], vhat[j * 128:(j + 1) * 128], atol=1e-13)
    assert abs(mass[0, 0] - 8.0) < 1e-13


def test_zero_query_gives_uniform_attention():
    """q = 0: every logit is 0, so each head averages all T + L value rows; mass_t = Hg/(T+L)."""
    T, L, Hg = 20, 5, 4
    CK, BK, CV, BV, Kt, Vt, mask, q, bits = _rand_unit(9, T, L, Hg)
    q[:] = 0.0
    out, mass = oracle.decode(CK, BK, CV, BV, Kt, Vt, mask, q, r_lo=16)
    rho = np.where(bits, 64, 16)
    vhat = np.stack([CV[0, t, :rho[t]] @ BV[0, :rho[t]] for t in range(T)])
    for h in range(Hg):
        sl = slice(h * 128, (h + 1) * 128)
        expect = (vhat[:, sl].sum(0) + Vt[0, :, h, :].sum(0)) / (T + L)
        np.testing.assert_allclose(out[0, h], expect, atol=1e-13)
    np.testing.assert_allclose(mass[0], Hg / (T + L), rtol=1e-13)


def test_dominant_key_selects_its_value():
    """One key equal to 1e4 * q_h takes all of head h's weight: o_h = Vhat_6, mass_6 = Hg."""
    T, L, Hg = 16, 4, 4
    g = np.random.default_rng(13)
    Bfull = np.linalg.qr(g.standard_normal((512, 512)))[0].T      # orthogonal: B B^T = B^T B = I
    q = g.standard_normal((1, Hg, 128)) / math.sqrt(128)
    CK = g.standard_normal((1, T, 512)) * 0.05
    CV = g.standard_normal((1, T, 512))
    CK[0, 6] = Bfull @ (1e4 * q[0].reshape(-1))                   # Khat_6 = C_K[6] B = 1e4 q
    Kt, Vt = g.standard_normal((1, L, 4, 128)), g.standard_normal((1, L, 4, 128))
    mask = np.array([[0xFFFF]], dtype=np.uint32)
    out, mass = oracle.decode(CK, Bfull[None], CV, Bfull[None], Kt, Vt, mask, q, r_lo=16)
    vhat6 = CV[0, 6] @ Bfull
    for h in range(Hg):
        np.testing.assert_allclose(out[0, h], vhat6[h * 128:(h + 1) * 128], atol=1e-9)
    assert abs(mass[0, 6] - Hg) < 1e-9


def test_token_permutation_invariance():
    T, L, Hg = 50, 9, 16
    CK, BK, CV, BV, Kt, Vt, mask, q, bits = _rand_unit(21, T, L, Hg)
    out, mass = oracle.decode(CK, BK, CV, BV, Kt, Vt, mask, q)
    perm = np.random.default_rng(2).permutation(T)
    pbits = bits[perm]
    pmask = np.zeros_like(mask)
    for t in np.nonzero(pbits)[0]:
        pmask[0, t >> 5] |= np.uint32(1 << (t & 31))
    out2, mass2 = oracle.decode(CK[:, perm], BK, CV[:, perm], BV, Kt, Vt, pmask, q)
    np.testing.assert_allclose(out2, out, atol=1e-13)
    np.testing.assert_allclose(mass2[0], mass[0, perm], atol=1e-15)


def test_full_low_rank_makes_mask_irrelevant():
    T, L, Hg = 37, 6, 8
    CK, BK, CV, BV, Kt, Vt, mask, q, bits = _rand_unit(4, T, L, Hg)
    o1, m1 = oracle.decode(CK, BK, CV, BV, Kt, Vt, mask, q, r_lo=64)
    o2, m2 = oracle.decode(CK, BK, CV, BV, Kt, Vt, np.zeros_like(mask), q, r_lo=64)
    np.testing.assert_array_equal(o1, o2)
    np.testing.assert_array_equal(m1, m2)


def test_low_rank_tokens_ignore_trailing_components():
    """A token with its mask bit clear reads only C[t, :r_lo]; with the bit set, all r."""
    T, L, Hg = 24, 3, 4
    CK, BK, CV, BV, Kt, Vt, mask, q, bits = _rand_unit(8, T, L, Hg)
    t_lo = int(np.nonzero(~bits)[0][0])
    t_hi = int(np.nonzero(bits)[0][0])
    o, m = oracle.decode(CK, BK, CV, BV, Kt, Vt, mask, q)
    CK2, CV2 = CK.copy(), CV.copy()
    CK2[0, t_lo, 16:] += 5.0
    CV2[0, t_lo, 16:] -= 3.0
    o2, m2 = oracle.decode(CK2, BK, CV2, BV, Kt, Vt, mask, q)
    np.testing.assert_array_equal(o, o2)
    CK3 = CK.copy()
    CK3[0, t_hi, 40] += 5.0
    o3, _ = oracle.decode(CK3, BK, CV, BV, Kt, Vt, mask, q)
    assert np.abs(o3 - o).max() > 1e-6


def test_gqa_head_to_kv_head_mapping():
    """Query head h reads KV head h // (Hg/4): only heads of KV head 2 see a nonzero text V."""
    T, L, Hg = 10, 5, 16
    CK, BK, CV, BV, Kt, Vt, mask, q, bits = _rand_unit(17, T, L, Hg)
    CV[:] = 0.0
    Vt[:] = 0.0
    Vt[0, :, 2, :] = 1.0
    out, _ = oracle.decode(CK, BK, CV, BV, Kt, Vt, mask, q)
    for h in range(Hg):
        if h // 4 == 2:
            assert out[0, h].min() > 0.0
        else:
            assert np.all(out[0, h] == 0.0)


def test_mass_is_a_probability_share():
    """Each head's softmax sums to 1 over visual + text, so sum_t mass_t + text share = Hg."""
    T, L, Hg = 30, 0, 28
    CK, BK, CV, BV, Kt, Vt, mask, q, bits = _rand_unit(31, T, L, Hg)
    _, mass = oracle.decode(CK, BK, CV, BV, Kt[:, :0], Vt[:, :0], mask, q)
    assert abs(mass.sum() - Hg) < 1e-12
    assert np.all(mass > 0)


def test_scale_is_a_query_scale():
    T, L, Hg = 19, 4, 8
    CK, BK, CV, BV, Kt, Vt, mask, q, bits = _rand_unit(2, T, L, Hg)
    o1, m1 = oracle.decode(CK, BK, CV, BV, Kt, Vt, mask, q, scale=2.5)
    o2, m2 = oracle.decode(CK, BK, CV, BV, Kt, Vt, mask, q * 2.5, scale=1.0)
    np.testing.assert_allclose(o1, o2, atol=1e-13)
    np.testing.assert_allclose(m1, m2, atol=1e-14)


def test_large_logits_do_not_overflow():
    T, L, Hg = 12, 2, 4
    CK, BK, CV, BV, Kt, Vt, mask, q, bits = _rand_unit(6, T, L, Hg)
    o, m = oracle.decode(CK, BK, CV, BV, Kt, Vt, mask, q * 1e5)
    assert np.all(np.isfinite(o)) and np.all(np.isfinite(m))


def test_rank_zero_tokens_act_as_zero_key_and_value():
    """r_lo = 0 (a low-importance token is not decompressed at all, de summary 2.B): such a
    token's reconstruction is zero, so the step equals a full-rank step in which those tokens'
    coefficients are zero; all of them get the same mass."""
    T, L, Hg = 45, 6, 8
    CK, BK, CV, BV, Kt, Vt, mask, q, bits = _rand_unit(77, T, L, Hg)
    out0, mass0 = oracle.decode(CK, BK, CV, BV, Kt, Vt, mask, q, r_lo=0)
    CKz, CVz = CK.copy(), CV.copy()
    CKz[0, ~bits] = 0.0
    CVz[0, ~bits] = 0.0
    ones = np.full_like(mask, 0xFFFFFFFF)
    ref_o, ref_m = oracle.decode(CKz, BK, CVz, BV, Kt, Vt, ones, q, r_lo=64)
    np.testing.assert_allclose(out0, ref_o, rtol=1e-12, atol=1e-14)
    np.testing.assert_allclose(mass0, ref_m, rtol=1e-12, atol=1e-16)
    m_low = mass0[0, ~bits]
    assert np.all(np.abs(m_low - m_low[0]) <= 1e-15 * abs(m_low[0]))


def test_all_rank_zero_without_text_is_uniform_and_zero():
    T, Hg = 37, 4
    CK, BK, CV, BV, Kt, Vt, mask, q, bits = _rand_unit(3, T, 0, Hg)
    zero = np.zeros_like(mask)
    out, mass = oracle.decode(CK, BK, CV, BV, Kt, Vt, zero, q, r_lo=0)
    assert np.all(out == 0.0)
    np.testing.assert_allclose(mass[0], np.full(T, Hg / T), rtol=1e-14)


# ----------------------------------------------------------------- text compressed too

def _text_factors(seed, L, exact_rank=64):
    """Text K / V of rank <= 64 with exact factors: K = C B, B with orthonormal rows."""
    g = np.random.default_rng(seed)
    out = []
    for _ in range(2):
        B = np.linalg.qr(g.standard_normal((512, 64)))[0].T
        C = g.standard_normal((L, 64)) * (np.arange(64) < exact_rank)
        out += [C[None], B[None]]
    return out   # CKt, BKt, CVt, BVt


def test_text_basis_equals_its_decompressed_tail():
    """The compressed text tokens act exactly like the uncompressed tokens C B they factor."""
    CK, BK, CV, BV, Kt, Vt, mask, q, _ = _rand_unit(71, 300, 9, 8)
    CKt, BKt, CVt, BVt = _text_factors(72, 40)
    Kd = (CKt[0] @ BKt[0]).reshape(1, 40, 4, 128)
    Vd = (CVt[0] @ BVt[0]).reshape(1, 40, 4, 128)
    o1, m1 = oracle.decode_tb(CK, BK, CV, BV, CKt, BKt, CVt, BVt, Kt, Vt, mask, q)
    o2, m2 = oracle.decode(CK, BK, CV, BV, np.concatenate([Kd, Kt], 1), np.concatenate([Vd, Vt], 1), mask, q)
    np.testing.assert_allclose(o1, o2, rtol=0, atol=1e-12)
    np.testing.assert_allclose(m1, m2, rtol=0, atol=1e-15)


def test_text_basis_without_text_tokens_is_the_plain_step():
    CK, BK, CV, BV, Kt, Vt, mask, q, _ = _rand_unit(73, 200, 5, 16)
    z = np.zeros((1, 0, 64))
    zb = np.linalg.qr(np.random.default_rng(74).standard_normal((512, 64)))[0].T[None]
    o1, m1 = oracle.decode_tb(CK, BK, CV, BV, z, zb, z, zb, Kt, Vt, mask, q)
    o2, m2 = oracle.decode(CK, BK, CV, BV, Kt, Vt, mask, q)
    assert np.array_equal(o1, o2) and np.array_equal(m1, m2)


def test_text_basis_rank_space_route():
    """Closed form of the text tokens' part: their logits are C_K' (B_K' q) and their value sum
    (sum p C_V') B_V', so a query orthogonal to every B_K' row gives them logit 0."""
    CK, BK, CV, BV, Kt, Vt, mask, q, _ = _rand_unit(75, 64, 0, 4)
    CKt, BKt, CVt, BVt = _text_factors(76, 30)
    # project the query of every head onto the orthogonal complement of its KV head's text basis slice
    qq = q.copy()
    for h in range(4):
        Bj = BKt[0][:, 128 * h:128 * h + 128]          # Hg = 4: one query head per KV head
        Pj = np.linalg.qr(Bj.T)[0]                      # orthonormal basis of span(B_j^T) (128 x 64)
        qq[0, h] -= Pj @ (Pj.T @ qq[0, h])
    big = 1e3 * np.ones_like(CKt)                        # any coefficients: the logits stay 0
    o1, _ = oracle.decode_tb(CK, BK, CV, BV, big, BKt, CVt, BVt, Kt, Vt, mask, qq)
    o2, _ = oracle.decode_tb(CK, BK, CV, BV, 0 * big, BKt, CVt, BVt, Kt, Vt, mask, qq)
    np.testing.assert_allclose(o1, o2, rtol=0, atol=1e-9)


# ----------------------------------------------------------------- 4-bit coefficients

def test_quantize4_exponent_and_codes_by_brute_force():
    """e is the smallest integer with 7 * 2^e >= max |c| (searched over all candidates), codes
    are c / 2^e rounded half to even, and |q| <= 7."""
    g = np.random.default_rng(81)
    C = g.standard_normal((40, 64)) * np.exp(g.uniform(-20, 20, size=(40, 1)))
    C[3] = 0.0                                  # an all-zero token
    C[5, :16] = 0.0                             # an all-zero plane
    C[7, :16] = np.linspace(-3.0, 3.0, 16)
    C[7, 0] = 7 * 2.0 ** 3                      # the maximum exactly on 7 * 2^e
    C[8, :16] = 0.0
    C[8, 1] = 2.5 * 2.0 ** -4                   # a tie, rounded to even
    C[8, 0] = 7 * 2.0 ** -4
    q, e = oracle.quantize4(C)
    for t in range(C.shape[0]):
        for pl, (a, b) in enumerate(((0, 16), (16, 64))):
            amax = np.abs(C[t, a:b]).max()
            if amax == 0:
                assert e[t, pl] == 0 and np.all(q[t, a:b] == 0)
                continue
            best = min(x for x in range(-200, 200) if 7 * 2.0 ** x >= amax)
            assert e[t, pl] == best
            assert np.all(np.abs(q[t, a:b]) <= 7)
            for i in range(a, b):
                v = C[t, i] / 2.0 ** best
                r = np.floor(v + 0.5)
                if r - v == 0.5 and r % 2 == 1:   # a tie goes to the even neighbour
                    r -= 1
                assert q[t, i] == r
    assert e[7, 0] == 3 and q[7, 0] == 7
    assert q[8, 1] == 2                          # 2.5 -> 2


def test_quantize4_round_trip_and_error_bound():
    g = np.random.default_rng(82)
    C = g.standard_normal((100, 64))
    q, e = oracle.quantize4(C)
    D = oracle.dequantize4(q, e)
    step = np.concatenate([np.repeat(2.0 ** e[:, :1], 16, axis=1), np.repeat(2.0 ** e[:, 1:], 48, axis=1)], axis=1)
    assert np.all(np.abs(D - C) <= step / 2)    # half a step at most
    q2, e2 = oracle.quantize4(D)                 # grid values are fixed points
    assert np.array_equal(q2, q) and np.array_equal(e2, e)


def test_pack4_layout():
    codes = np.arange(-7, 8).tolist() * 5
    codes = np.array(codes[:64], dtype=np.int8)[None]
    lo, hi = oracle.pack4(codes)
    assert lo.shape == (1, 8) and hi.shape == (1, 24)
    flat = np.concatenate([lo, hi], axis=1)[0]
    for k in range(32):
        low, high = int(flat[k]) & 0xF, int(flat[k]) >> 4
        sx = lambda v: v - 16 if v >= 8 else v
        assert sx(low) == codes[0, 2 * k] and sx(high) == codes[0, 2 * k + 1]
