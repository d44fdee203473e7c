// quant.cuh -- 4-bit coefficients (the pages' composition of the compression with 4-bit
// quantisation: es page 3 Contribuciones, fr page 4 Compatibilite, de page 4 Ergebnisse).
//
// Format (the pages fix none): per token and plane (ranks 0..15, ranks 16..63) symmetric int4
// codes q in [-7, 7] with one power-of-two scale 2^e, e the smallest integer with
// 7 * 2^e >= max |c| (e = 0 for an all-zero plane) -- the block format of the OCP microscaling
// (MX) specification with an E8M0 scale.  q = round-half-even(c / 2^e); c is recovered as
// q * 2^e, exactly representable in bf16, so the decode's tensor-core operands carry no
// rounding of their own.  Codes are packed two per byte, code 2k in the low nibble of byte k:
//   Q_lo [units][T][8], Q_hi [units][T][24], E [units][T][2] (int8: e_lo, e_hi).
#pragma once

#include "common.cuh"

#include <cuda_bf16.h>

namespace kvpack {
namespace quant {

// e of a plane: max |c| = m 2^k with m in [0.5, 1) puts it at k - 3 or k - 2; the comparison
// with 7 * 2^(k-3) is exact.
__device__ __forceinline__ int plane_exponent(float amax) {
    if (!(amax > 0.f)) return 0;
    int k;
    frexpf(amax, &k);
    int e = ldexpf(7.f, k - 3) >= amax ? k - 3 : k - 2;
    return e < -127 ? -127 : (e > 127 ? 127 : e);
}

__device__ __forceinline__ uint32_t code4(float c, int e) {
    float q = rintf(ldexpf(c, -e));   // exact scaling; rounding half to even
    q = fminf(fmaxf(q, -7.f), 7.f);
    return (uint32_t)((int)q) & 0xFu;
}

// One thread per (unit, token): reads the token's 64 bf16 coefficients, writes its codes and
// exponents.
__global__ void __launch_bounds__(256) quantize4_kernel(const uint16_t *__restrict__ C_lo,
                                                        const uint16_t *__restrict__ C_hi, uint8_t *__restrict__ Q_lo,
                                                        uint8_t *__restrict__ Q_hi, int8_t *__restrict__ E,
                                                        long long rows) {
    const long long row = (long long)blockIdx.x * blockDim.x + threadIdx.x;
    if (row >= rows) return;
    float c[64];
    #pragma unroll
    for (int i = 0; i < 2; ++i) {
        const uint4 v = __ldg(reinterpret_cast<const uint4 *>(C_lo + row * 16) + i);
        const uint32_t w[4] = {v.x, v.y, v.z, v.w};
        #pragma unroll
        for (int k = 0; k < 4; ++k) {
            c[8 * i + 2 * k] = __uint_as_float(w[k] << 16);
            c[8 * i + 2 * k + 1] = __uint_as_float(w[k] & 0xffff0000u);
        }
    }
    #pragma unroll
    for (int i = 0; i < 6; ++i) {
        const uint4 v = __ldg(reinterpret_cast<const uint4 *>(C_hi + row * 48) + i);
        const uint32_t w[4] = {v.x, v.y, v.z, v.w};
        #pragma unroll
        for (int k = 0; k < 4; ++k) {
            c[16 + 8 * i + 2 * k] = __uint_as_float(w[k] << 16);
            c[16 + 8 * i + 2 * k + 1] = __uint_as_float(w[k] & 0xffff0000u);
        }
    }
    float a0 = 0.f, a1 = 0.f;
    #pragma unroll
    for (int i = 0; i < 16; ++i) a0 = fmaxf(a0, fabsf(c[i]));
    #pragma unroll
    for (int i = 16; i < 64; ++i) a1 = fmaxf(a1, fabsf(c[i]));
    const int e0 = plane_exponent(a0), e1 = plane_exponent(a1);
    uint32_t pk[8];
    #pragma unroll
    for (int wd = 0; wd < 8; ++wd) {
        uint32_t x = 0u;
        #pragma unroll
        for (int k = 0; k < 8; ++k) {
            const int i = 8 * wd + k;
            x |= code4(c[i], i < 16 ? e0 : e1) << (4 * k);
        }
        pk[wd] = x;
    }
    *reinterpret_cast<uint2 *>(Q_lo + row * 8) = make_uint2(pk[0], pk[1]);
    uint2 *qh = reinterpret_cast<uint2 *>(Q_hi + row * 24);
    qh[0] = make_uint2(pk[2], pk[3]);
    qh[1] = make_uint2(pk[4], pk[5]);
    qh[2] = make_uint2(pk[6], pk[7]);
    *reinterpret_cast<char2 *>(E + row * 2) = make_char2((signed char)e0, (signed char)e1);
}

// 2^e as a float for e in [-127, 127] (2^-127 is subnormal)
__device__ __forceinline__ float pow2f(int e) {
    return e > -127 ? __int_as_float((e + 127) << 23) : __int_as_float(1 << 22);
}

// 8 codes times 2^e through fp32 (exact for every e): the path for exponents whose bf16
// intermediates below could leave the normal range
__device__ __noinline__ uint4 dq8_wide(uint32_t w, int e) {
    const float sc = pow2f(e);
    uint32_t b[8];
    #pragma unroll
    for (int k = 0; k < 8; ++k) b[k] = __float_as_uint(__int2float_rn((int)(w << (28 - 4 * k)) >> 28) * sc);
    return make_uint4((b[0] >> 16) | (b[1] & 0xffff0000u), (b[2] >> 16) | (b[3] & 0xffff0000u),
                      (b[4] >> 16) | (b[5] & 0xffff0000u), (b[6] >> 16) | (b[7] & 0xffff0000u));
}

// 2^e as a bf16 pair for e in [-119, 119]
__device__ __forceinline__ uint32_t pow2_bf16x2(int e) {
    const uint32_t h = (uint32_t)(e + 127) << 7;
    return h | (h << 16);
}

// 8 codes of a packed word -> 8 bf16 values as 4 packed pairs.  A code's nibble n, made offset-binary
// (n ^ 8 = q + 8), is placed under the bf16 bits of 128 (0x4300), which reads as 128 + q + 8 exactly;
// one bf16 fused multiply-add per pair then forms (128 + q + 8) 2^e - 136 2^e = q 2^e, exact because
// every intermediate has at most eight significant bits and the result three.
__device__ __forceinline__ uint4 dq8(uint32_t w, int e) {
    if (e < -119 || e > 119) return dq8_wide(w, e);   // keeps every bf16 intermediate normal and finite
    const uint32_t x = w ^ 0x88888888u;
    const uint32_t s2 = pow2_bf16x2(e);
    __nv_bfloat162 sc = *reinterpret_cast<const __nv_bfloat162 *>(&s2);
    const __nv_bfloat162 c136 = __floats2bfloat162_rn(-136.f, -136.f);
    const __nv_bfloat162 bias = __hmul2(c136, sc);
    uint32_t r[4];
    #pragma unroll
    for (int k = 0; k < 4; ++k) {
        const uint32_t t = x >> (8 * k);
        const uint32_t v = 0x43004300u | (t & 0xFu) | ((t << 12) & 0xF0000u);
        const __nv_bfloat162 y = __hfma2(*reinterpret_cast<const __nv_bfloat162 *>(&v), sc, bias);
        r[k] = *reinterpret_cast<const uint32_t *>(&y);
    }
    return make_uint4(r[0], r[1], r[2], r[3]);
}

// One plane set of LO rows: codes of ranks 0..15 of tokens tok .. tok + n - 1 (row base `base`) into
// 32-byte rows of a tile with the 32-byte swizzle (16-byte chunk c of row t at c ^ ((t >> 2) & 1));
// R rows per thread, thread `t0` of `NT`; rows past n are zero.  Every load is issued before the
// first is used.
template <int R, int NT>
__device__ __forceinline__ void lo_rows(unsigned char *dst, const uint8_t *__restrict__ Q, const int8_t *__restrict__ E,
                                        size_t base, int n, int t0) {
    uint2 w[R];
    int ex[R];
    #pragma unroll
    for (int i = 0; i < R; ++i) {
        const int t = t0 + NT * i;
        w[i] = make_uint2(0u, 0u);
        ex[i] = 0;
        if (t < n) {
            w[i] = __ldg(reinterpret_cast<const uint2 *>(Q + (base + t) * 8));
            ex[i] = __ldg(E + (base + t) * 2);
        }
    }
    #pragma unroll
    for (int i = 0; i < R; ++i) {
        const int t = t0 + NT * i;
        const int sw = (t >> 2) & 1;
        *reinterpret_cast<uint4 *>(dst + t * 32 + (sw << 4)) = dq8(w[i].x, ex[i]);
        *reinterpret_cast<uint4 *>(dst + t * 32 + ((1 ^ sw) << 4)) = dq8(w[i].y, ex[i]);
    }
}

// The same for the K and the V planes of the same rows, the loads of eight rows first
template <int R, int NT>
__device__ __forceinline__ void lo_rows_kv(unsigned char *dk, unsigned char *dv, const uint8_t *__restrict__ QK,
                                           const int8_t *__restrict__ EK, const uint8_t *__restrict__ QV,
                                           const int8_t *__restrict__ EV, size_t base, int n, int t0) {
    if constexpr (R > 8) {
        lo_rows_kv<8, NT>(dk, dv, QK, EK, QV, EV, base, n, t0);
        lo_rows_kv<R - 8, NT>(dk, dv, QK, EK, QV, EV, base, n, t0 + 8 * NT);
    } else {
    uint2 wk[R], wv[R];
    int ek[R], ev[R];
    #pragma unroll
    for (int i = 0; i < R; ++i) {
        const int t = t0 + NT * i;
        wk[i] = wv[i] = make_uint2(0u, 0u);
        ek[i] = ev[i] = 0;
        if (t < n) {
            wk[i] = __ldg(reinterpret_cast<const uint2 *>(QK + (base + t) * 8));
            ek[i] = __ldg(EK + (base + t) * 2);
            wv[i] = __ldg(reinterpret_cast<const uint2 *>(QV + (base + t) * 8));
            ev[i] = __ldg(EV + (base + t) * 2);
        }
    }
    #pragma unroll
    for (int i = 0; i < R; ++i) {
        const int t = t0 + NT * i;
        const int sw = (t >> 2) & 1;
        *reinterpret_cast<uint4 *>(dk + t * 32 + (sw << 4)) = dq8(wk[i].x, ek[i]);
        *reinterpret_cast<uint4 *>(dk + t * 32 + ((1 ^ sw) << 4)) = dq8(wk[i].y, ek[i]);
        *reinterpret_cast<uint4 *>(dv + t * 32 + (sw << 4)) = dq8(wv[i].x, ev[i]);
        *reinterpret_cast<uint4 *>(dv + t * 32 + ((1 ^ sw) << 4)) = dq8(wv[i].y, ev[i]);
    }
    }
}

}  // namespace quant
}  // namespace kvpack
