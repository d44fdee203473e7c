"""fp64 CPU oracle for the AttentionPack decode hot path (numpy front end).

TEST INFRASTRUCTURE ONLY.  Only tests/, __graft_entry__.smoke() and the
cpu_baseline / reference leg of bench.py may import this package.  It shares
no code with the product (rank_compressed_kv_b200), and neither imports the
other.

The arithmetic lives in oracle.c (plain C, fp64, OpenMP over independent
units); this module converts numpy arrays and calls it.  What each routine
computes, and the passage of the method it follows:

  compress  -- multi-head SVD compression (AttentionPack pages, Technical
               summary 2.A): K (T x 512, the 4 KV heads of a group side by
               side) = C . B with C = U_r Sigma_r and B = V_r^T, by Householder
               QR followed by one-sided Jacobi (Hestenes) SVD.
  decode    -- one decode step with attention-aware partial decompression
               (pages 2.B): each visual token decompressed at rank r or r_lo
               by its mask bit, then dense softmax attention over visual
               tokens plus the uncompressed text tail; also the attention
               mass each visual token received.
  decode_tb -- the same step with the text tokens compressed too, by a basis
               of their own (pages 2.A): they are decompressed at the full
               rank and attended together with the uncompressed tail.
  quantize4 -- 4-bit coefficients (int4 codes, a power-of-two scale per token
               and plane) and their exact dequantisation.
  select    -- importance = moving average (alpha) of attention mass; the k
               largest get the full rank next step, ties to the lower index.

Parity pins for every routine are in tests/test_oracle_*.py.
"""
import ctypes
import os

import numpy as np

from . import build as _build

_lib = None

_dp = ctypes.POINTER(ctypes.c_double)
_fp = ctypes.POINTER(ctypes.c_float)
_u32p = ctypes.POINTER(ctypes.c_uint32)
_u16p = ctypes.POINTER(ctypes.c_uint16)
_i64 = ctypes.c_int64


def lib():
    global _lib
    if _lib is None:
        path = _build.build()
        L = ctypes.CDLL(path)
        L.ora_bf16_to_f64_array.argtypes = [_u16p, _dp, _i64]
        L.ora_f64_to_bf16_array.argtypes = [_dp, _u16p, _i64]
        L.ora_svd.argtypes = [_dp, _i64, ctypes.c_int, _dp, _dp]
        L.ora_svd.restype = ctypes.c_int
        L.ora_compress_units.argtypes = [_i64, _dp, _i64, ctypes.c_int, ctypes.c_int, _dp, _dp, _dp]
        L.ora_compress_units.restype = ctypes.c_int
        L.ora_decode_units.argtypes = [_i64, _i64, _i64, ctypes.c_int, ctypes.c_int, ctypes.c_int,
                                       _dp, _dp, _dp, _dp, _dp, _dp, _u32p, _dp, ctypes.c_double, _dp, _dp]
        L.ora_select_units.argtypes = [_i64, _i64, _fp, _fp, ctypes.c_float, _i64, _u32p]
        L.ora_num_threads.restype = ctypes.c_int
        _lib = L
    return _lib


def num_threads() -> int:
    """OpenMP threads the oracle runs on."""
    return int(lib().ora_num_threads())


def _ptr(a, t):
    return a.ctypes.data_as(t)


def _f64(a):
    return np.ascontiguousarray(a, dtype=np.float64)


# ------------------------------------------------------------------ bf16

def bf16_to_f64(bits) -> np.ndarray:
    """Exact widening of bf16 bit patterns (uint16) to float64."""
    b = np.ascontiguousarray(bits, dtype=np.uint16)
    out = np.empty(b.shape, dtype=np.float64)
    lib().ora_bf16_to_f64_array(_ptr(b, _u16p), _ptr(out, _dp), b.size)
    return out


def f64_to_bf16(x) -> np.ndarray:
    """Round float64 to the nearest bf16 (ties to even), one rounding step; uint16 bits."""
    a = _f64(x)
    out = np.empty(a.shape, dtype=np.uint16)
    lib().ora_f64_to_bf16_array(_ptr(a, _dp), _ptr(out, _u16p), a.size)
    return out


# ------------------------------------------------------------- compress

def svd(X):
    """Singular values (descending) and right singular vectors (columns of V) of X (T x n)."""
    X = _f64(X)
    T, n = X.shape
    sig = np.empty(min(T, n), dtype=np.float64)
    V = np.empty((n, n), dtype=np.float64)
    sweeps = lib().ora_svd(_ptr(X, _dp), T, n, _ptr(sig, _dp), _ptr(V, _dp))
    if sweeps < 0:
        raise RuntimeError("oracle Jacobi SVD did not converge")
    return sig, V


def compress(X, r=64):
    """Truncated factors of units X [U, T, n] (fp64): C [U,T,r], B [U,r,n], sigma [U,min(T,n)]."""
    X = _f64(X)
    if X.ndim == 2:
        X = X[None]
    U, T, n = X.shape
    C = np.empty((U, T, r))
    B = np.empty((U, r, n))
    sig = np.empty((U, min(T, n)))
    s = lib().ora_compress_units(U, _ptr(X, _dp), T, n, r, _ptr(C, _dp), _ptr(B, _dp), _ptr(sig, _dp))
    if s < 0:
        raise RuntimeError("oracle Jacobi SVD did not converge")
    return C, B, sig


# --------------------------------------------------------------- decode

def decode(CK, BK, CV, BV, Ktext, Vtext, mask, q, r_lo=16, scale=1.0, want_mass=True):
    """One decode step over U independent units (fp64).

    CK, CV [U,T,r]; BK, BV [U,r,512]; Ktext, Vtext [U,L,4,128]; mask uint32
    [U, ceil(T/32)]; q [U,Hg,128].  Returns out [U,Hg,128] and mass [U,T].
    """
    CK, BK, CV, BV = (_f64(a) for a in (CK, BK, CV, BV))
    Ktext, Vtext, q = _f64(Ktext), _f64(Vtext), _f64(q)
    U, T, r = CK.shape
    L = Ktext.shape[1]
    Hg = q.shape[1]
    assert BK.shape == (U, r, 512) and Ktext.shape == (U, L, 4, 128) and q.shape == (U, Hg, 128)
    assert Hg % 4 == 0
    m = np.ascontiguousarray(mask, dtype=np.uint32).reshape(U, (T + 31) // 32)
    out = np.empty((U, Hg, 128))
    mass = np.empty((U, T)) if want_mass else None
    if L == 0:   # keep valid pointers for empty tails
        Ktext = np.zeros((U, 1, 4, 128))
        Vtext = np.zeros((U, 1, 4, 128))
    lib().ora_decode_units(U, T, L, Hg, r, r_lo, _ptr(CK, _dp), _ptr(BK, _dp), _ptr(CV, _dp), _ptr(BV, _dp),
                           _ptr(Ktext, _dp), _ptr(Vtext, _dp), _ptr(m, _u32p), _ptr(q, _dp), float(scale),
                           _ptr(out, _dp), _ptr(mass, _dp) if want_mass else None)
    return out, mass


def decode_tb(CK, BK, CV, BV, CKt, BKt, CVt, BVt, Ktail, Vtail, mask, q, r_lo=16, scale=1.0, want_mass=True):
    """One decode step when the text tokens are compressed too, with a basis of their own
    (technical summaries 2.A on the es / fr / de pages: visual and text tokens are factored
    separately).  The L_c compressed text tokens are decompressed at the full rank,
    K' = C_K' B_K' and V' = C_V' B_V' (fp64 products, reshaped to [L_c, 4, 128]), and placed
    before the uncompressed tail; the step is then decode() over T visual + L_c + L_tail tokens.

    CKt, CVt [U,L_c,64]; BKt, BVt [U,64,512]; Ktail, Vtail [U,L,4,128].  Returns out, mass [U,T].
    """
    CKt, BKt, CVt, BVt = (_f64(a) for a in (CKt, BKt, CVt, BVt))
    U, Lc, _ = CKt.shape
    Kd = np.matmul(CKt, BKt).reshape(U, Lc, 4, 128)
    Vd = np.matmul(CVt, BVt).reshape(U, Lc, 4, 128)
    Kall = np.concatenate([Kd, _f64(Ktail)], axis=1)
    Vall = np.concatenate([Vd, _f64(Vtail)], axis=1)
    return decode(CK, BK, CV, BV, Kall, Vall, mask, q, r_lo=r_lo, scale=scale, want_mass=want_mass)


# --------------------------------------------------------------- 4-bit coefficients

def quantize4(C):
    """4-bit coefficients with a power-of-two scale per token and plane (the pages' composition of
    the compression with 4-bit quantisation: es page 3 Contribuciones, fr page 4 Compatibilite;
    they fix no format, so this build takes symmetric int4 codes with a shared power-of-two scale,
    the block format of the OCP microscaling (MX) specification with E8M0 scales).

    C: [..., T, 64] coefficients (bf16 values as float64).  For each token the planes of ranks
    0..15 and 16..63 get their own exponent e = the smallest integer with 7 * 2^e >= max |c|
    (e = 0 for an all-zero plane), and codes q = round-half-even(c / 2^e) in [-7, 7].  Returns
    codes int8 [..., T, 64] and exponents int8 [..., T, 2]."""
    C = np.asarray(C, dtype=np.float64)
    codes = np.zeros(C.shape, dtype=np.int8)
    exps = np.zeros(C.shape[:-1] + (2,), dtype=np.int8)
    for pl, (a, b) in enumerate(((0, 16), (16, 64))):
        X = C[..., a:b]
        amax = np.abs(X).max(axis=-1)
        nz = amax > 0
        # amax = m 2^k with m in [0.5, 1): the smallest e with 7 * 2^e >= amax is k - 3 or k - 2
        _, k = np.frexp(np.where(nz, amax, 1.0))
        k = k.astype(np.int64)
        e = np.where(np.ldexp(7.0, k - 3) >= amax, k - 3, k - 2)
        e = np.where(nz, e, 0)
        e = np.clip(e, -127, 127)
        q = np.rint(X / np.ldexp(1.0, e)[..., None])
        codes[..., a:b] = np.clip(q, -7, 7).astype(np.int8)
        exps[..., pl] = e.astype(np.int8)
    return codes, exps


def dequantize4(codes, exps):
    """c = q * 2^e per plane (exact in binary floating point)."""
    codes = np.asarray(codes, dtype=np.float64)
    e = np.asarray(exps, dtype=np.int64)
    out = codes.copy()
    out[..., :16] *= np.ldexp(1.0, e[..., 0])[..., None]
    out[..., 16:] *= np.ldexp(1.0, e[..., 1])[..., None]
    return out


def pack4(codes):
    """int4 codes [..., 64] -> bytes: lo plane [..., 8], hi plane [..., 24]; code 2k in the low nibble of
    byte k, two's complement."""
    u = (np.asarray(codes, dtype=np.int16) & 0xF).astype(np.uint8)
    packed = (u[..., 0::2] | (u[..., 1::2] << 4)).astype(np.uint8)
    return np.ascontiguousarray(packed[..., :8]), np.ascontiguousarray(packed[..., 8:])


# --------------------------------------------------------------- select

def select(mass, k, alpha=0.0, score=None):
    """Rank mask for the next step from fp32 mass [U,T] (and EMA score, updated in place).

    Returns (mask uint32 [U, ceil(T/32)], score fp32 [U,T]).
    """
    mass = np.ascontiguousarray(mass, dtype=np.float32)
    if mass.ndim == 1:
        mass = mass[None]
    U, T = mass.shape
    if score is None:
        score = np.zeros_like(mass)
    score = np.ascontiguousarray(score, dtype=np.float32).reshape(U, T).copy()
    mask = np.empty((U, (T + 31) // 32), dtype=np.uint32)
    lib().ora_select_units(U, T, _ptr(mass, _fp), _ptr(score, _fp), ctypes.c_float(alpha), int(k),
                           _ptr(mask, _u32p))
    return mask, score


def mask_bits(mask, T) -> np.ndarray:
    """Bool [.., T] view of a packed rank mask (bit t of word t>>5)."""
    m = np.asarray(mask, dtype=np.uint32)
    idx = np.arange(T)
    return ((m[..., idx >> 5] >> (idx & 31).astype(np.uint32)) & 1).astype(bool)
