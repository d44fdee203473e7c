"""GPU compression (Gram -> subspace iteration -> projection) vs the fp64 oracle
(Householder QR + one-sided Jacobi SVD) on the same bf16 X.

The cases include the full visual lengths of the video workload (32 frames x
196 = 6272 tokens, shared rank-24 structure) and of the long-context workload
(65536 tokens), where the eigen-solver works hardest.

Signs of singular vectors and rotations inside clusters are arbitrary, so only
sign-invariant quantities are compared: singular values (<= 1e-2 relative),
the angle between matching singular vectors where sigma is well separated
(relative gap > 5 %; <= 1e-2 rad), the truncation error against the
Eckart-Young optimum, orthonormality of B and consistency of C with X B^T."""
import math

import numpy as np
import pytest
import torch

import oracle
import synth
from gpu_util import DEV, bf

pytestmark = pytest.mark.gpu


def _gpu_compress(kv, X_bits, T):
    """X_bits: uint16 [U, T, 512]; returns sigma [U,64], B [U,64,512], C [U,T,64] (float64 of the bf16 results)."""
    U = X_bits.shape[0]
    dims = kv.Dims(batch=U, n_q_heads=4, n_kv_heads=4, T_vis=T, L_text_cap=0)
    X = bf(X_bits)
    C_lo = torch.empty(U, T, 16, dtype=torch.bfloat16, device=DEV)
    C_hi = torch.empty(U, T, 48, dtype=torch.bfloat16, device=DEV)
    B = torch.empty(U, 64, 512, dtype=torch.bfloat16, device=DEV)
    sig = torch.empty(U, 64, dtype=torch.float32, device=DEV)
    ws = torch.empty(kv.compress_workspace(dims, 1), dtype=torch.uint8, device=DEV)
    kv.compress(dims, 1, X, C_lo, C_hi, B, sig, ws)
    st = kv.last_device_status()
    assert st == 0, kv.STATUS_NAMES[st]
    C = torch.cat([C_lo, C_hi], dim=2).double().cpu().numpy()
    return sig.double().cpu().numpy(), B.double().cpu().numpy(), C


def _check_unit(Xf, sig_g, B_g, C_g, sig_r, B_r, structure_rank):
    T = Xf.shape[0]
    k = min(64, T)
    # singular values
    rel = np.abs(sig_g[:k] - sig_r[:k]) / np.maximum(sig_r[:k], 1e-12 * sig_r[0])
    assert rel.max() <= 1e-2, f"sigma rel error {rel.max():.3e} at {rel.argmax()}"
    if T < 64:
        assert np.all(sig_g[T:] <= 1e-2 * sig_r[0])
    # well-separated singular vectors
    s = sig_r
    for i in range(min(k, structure_rank)):
        lo_gap = (s[i - 1] - s[i]) / s[i] if i > 0 else np.inf
        hi_gap = (s[i] - s[i + 1]) / s[i]
        if min(lo_gap, hi_gap) <= 0.05:
            continue
        cosang = abs(B_g[i] @ B_r[i]) / np.linalg.norm(B_g[i])
        ang = math.acos(min(1.0, cosang))
        assert ang <= 1e-2, f"vector {i}: angle {ang:.3e} rad"
    # basis rows orthonormal (bf16 storage)
    Gm = B_g[:k] @ B_g[:k].T
    assert np.abs(Gm - np.eye(k)).max() <= 1e-2
    # coefficients are X B^T (bf16 storage, relative to the coefficient scale)
    ref_C = Xf @ B_g.T
    assert np.abs(C_g - ref_C).max() <= 1e-2 * np.abs(ref_C).max()
    # truncation error near the Eckart-Young optimum
    opt = math.sqrt(float(np.sum(sig_r[64:] ** 2))) if T > 64 else 0.0
    err = np.linalg.norm(Xf - C_g @ B_g)
    assert err <= 1.02 * opt + 1e-2 * np.linalg.norm(Xf) * (T <= 64), f"truncation {err:.4e} vs optimum {opt:.4e}"


@pytest.mark.parametrize("name,T,units", [("C0", 576, 2), ("C0", 1000, 3), ("C2", 2304, 1), ("C3", 784, 2),
                                          ("C0", 50, 1), ("C0", 96, 1), ("C3", 6272, 1), ("C4", 65536, 1)])
def test_compress_matches_oracle(name, T, units):
    import rank_compressed_kv_b200 as kv
    w = synth.WORKLOADS[name]
    if w.structure == "video24":
        w = synth.Workload(**{**w.__dict__, "T": T, "frames": T // 196})
    X_bits = np.stack([synth.visual_kv(w, 0, 0, u, synth.K_VIS if u % 2 == 0 else synth.V_VIS, T) for u in range(units)])
    sig_g, B_g, C_g = _gpu_compress(kv, X_bits, T)
    Xf = oracle.bf16_to_f64(X_bits)
    C_r, B_r, sig_r = oracle.compress(Xf, r=min(64, T, 512))
    rank = 32 if w.structure == "lowrank32" else 24
    for u in range(units):
        sr = np.zeros(max(64, sig_r.shape[1]) + 1)
        sr[:sig_r.shape[1]] = sig_r[u]
        Br = np.zeros((64, 512))
        Br[:B_r.shape[1]] = B_r[u]
        _check_unit(Xf[u], sig_g[u], B_g[u], C_g[u], sr, Br, rank)
