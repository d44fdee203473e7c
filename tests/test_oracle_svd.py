"""Pins for the oracle's compression: Householder QR + one-sided Jacobi SVD.

Each test checks the oracle against something other than itself: a closed
form, LAPACK (numpy.linalg.svd, an independent implementation), or a theorem
(Eckart-Young, exact reconstruction at full rank), and the generator's
known singular values.
"""
import math

import numpy as np
import pytest

import oracle
import synth


def _closed_form_2x2(A):
    a, b = A[0]
    c, d = A[1]
    s1 = a * a + b * b + c * c + d * d
    det = a * d - b * c
    disc = math.sqrt(max(s1 * s1 - 4 * det * det, 0.0))
    return np.array([math.sqrt((s1 + disc) / 2), math.sqrt(max((s1 - disc) / 2, 0.0))])


@pytest.mark.parametrize("seed", range(6))
def test_2x2_closed_form(seed):
    A = np.random.default_rng(seed).standard_normal((2, 2))
    s, V = oracle.svd(A)
    np.testing.assert_allclose(s, _closed_form_2x2(A), rtol=1e-13, atol=1e-14)
    np.testing.assert_allclose(V.T @ V, np.eye(2), atol=1e-14)


def test_diagonal_input():
    d = np.array([0.5, -3.0, 2.0, 0.0, 7.0])
    s, V = oracle.svd(np.diag(d))
    np.testing.assert_allclose(s, [7.0, 3.0, 2.0, 0.5, 0.0], atol=1e-15)
    # the leading right singular vector is the coordinate of the largest |d|
    assert abs(abs(V[4, 0]) - 1.0) < 1e-15 and abs(abs(V[1, 1]) - 1.0) < 1e-15


def test_rank_one_outer_product():
    g = np.random.default_rng(3)
    u, v = g.standard_normal(9), g.standard_normal(5)
    s, V = oracle.svd(np.outer(u, v))
    assert abs(s[0] - np.linalg.norm(u) * np.linalg.norm(v)) < 1e-12
    assert np.all(np.abs(s[1:]) < 1e-12)
    assert abs(abs(V[:, 0] @ v) / np.linalg.norm(v) - 1.0) < 1e-12


@pytest.mark.parametrize("shape", [(8, 4), (4, 8), (40, 6), (300, 64), (64, 64)])
def test_against_lapack(shape):
    X = np.random.default_rng(sum(shape)).standard_normal(shape)
    s, V = oracle.svd(X)
    s_ref = np.linalg.svd(X, compute_uv=False)
    np.testing.assert_allclose(s, s_ref, rtol=1e-12, atol=1e-12)
    np.testing.assert_allclose(V.T @ V, np.eye(shape[1]), atol=1e-12)
    # columns of X V are orthogonal with norms sigma (definition of right singular vectors)
    k = min(shape)
    XV = X @ V[:, :k]
    np.testing.assert_allclose(np.linalg.norm(XV, axis=0), s, rtol=1e-11, atol=1e-11)
    G = XV.T @ XV
    off = G - np.diag(np.diag(G))
    assert np.abs(off).max() < 1e-10 * s[0] ** 2


def test_full_rank_reconstructs_to_1e10():
    """r = g*d = 512 reconstructs the 576 x 512 unit to within 1e-10 (fp64)."""
    w = synth.WORKLOADS["C0"]
    X = oracle.bf16_to_f64(synth.visual_kv(w, 0, 0, 0, synth.K_VIS))
    C, B, sig = oracle.compress(X, r=512)
    err = np.abs(C[0] @ B[0] - X).max()
    assert err <= 1e-10 * np.abs(X).max()
    np.testing.assert_allclose(B[0] @ B[0].T, np.eye(512), atol=1e-12)


@pytest.mark.parametrize("r", [1, 16, 64, 200])
def test_eckart_young_truncation_error(r):
    """||X - C B||_F equals sqrt(sum of the discarded sigma_i^2)."""
    X = np.random.default_rng(r).standard_normal((260, 96)) @ np.diag(0.97 ** np.arange(96))
    rr = min(r, 96)
    C, B, sig = oracle.compress(X, r=rr)
    lhs = np.linalg.norm(X - C[0] @ B[0])
    rhs = math.sqrt(float(np.sum(sig[0][rr:] ** 2)))
    assert abs(lhs - rhs) <= 1e-10 * max(1.0, rhs)


def test_coefficients_are_U_sigma():
    """C = X V_r has orthogonal columns of norm sigma_i (C = U_r Sigma_r)."""
    X = np.random.default_rng(11).standard_normal((120, 32))
    C, B, sig = oracle.compress(X, r=8)
    np.testing.assert_allclose(np.linalg.norm(C[0], axis=0), sig[0][:8], rtol=1e-12)
    np.testing.assert_allclose(C[0], X @ B[0].T, atol=1e-12)


@pytest.mark.parametrize("name", ["C0", "C3"])
def test_generator_signal_sigmas_exact(name):
    """The noise-free generated signal has exactly the generator's singular values (pin P5)."""
    w = synth.WORKLOADS[name]
    T = 576 if name == "C0" else 196 * 4
    if name == "C3":
        w = synth.Workload(**{**w.__dict__, "T": T, "frames": 4})
    S, sig = synth.visual_signal(w, 0, 0, 0, synth.K_VIS)
    s, _ = oracle.svd(S)
    k = len(sig)
    np.testing.assert_allclose(s[:k], sig, rtol=1e-10)
    assert np.all(s[k:] < 1e-9 * sig[0])
    # signal RMS 1 per element
    assert abs(np.sqrt(np.mean(S ** 2)) - 1.0) < 1e-12
