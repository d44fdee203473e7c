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
    float q = rintf(ldexpf(c, -e));
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

// bf16 bits of q * 2^e (exact: |q| <= 7 has three significant bits)
__device__ __forceinline__ uint32_t dq_bf16(uint32_t nib, int e) {
    const int q = (int)(nib ^ 8u) - 8;        // sign-extended code
    return __float_as_uint(ldexpf((float)q, e)) >> 16;
}

// 8 codes of a packed word -> 8 bf16 values as 4 packed pairs
__device__ __forceinline__ uint4 dq8(uint32_t w, int e) {
    uint4 r;
    r.x = dq_bf16(w & 0xFu, e) | (dq_bf16((w >> 4) & 0xFu, e) << 16);
    r.y = dq_bf16((w >> 8) & 0xFu, e) | (dq_bf16((w >> 12) & 0xFu, e) << 16);
    r.z = dq_bf16((w >> 16) & 0xFu, e) | (dq_bf16((w >> 20) & 0xFu, e) << 16);
    r.w = dq_bf16((w >> 24) & 0xFu, e) | (dq_bf16((w >> 28) & 0xFu, e) << 16);
    return r;
}

}  // namespace quant
}  // namespace kvpack
