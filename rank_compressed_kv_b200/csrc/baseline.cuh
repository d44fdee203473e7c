// baseline.cuh -- the two routes the fused rank-space decode is measured against
// (the fr summary's results, §4, compare the fused kernels with a standard
// implementation; the method's own alternative is to decompress and then attend):
//
//   decompress_kernel   K^_t = C_K[t, :rho_t] B_K[:rho_t, :] and V^_t likewise for every
//                       visual token, written as a dense bf16 cache [units][L_cap][4][128]
//                       (rows 0 .. T-1; rho_t = 64 if the token's mask bit is set, else
//                       r_lo = 16 or 0): a (128 tokens x 64) x (64 x 512) product per tile
//                       on mma.sync, staged through shared memory for 16-byte stores
//   dense_finish_kernel out_h = sum_c 2^(m_c - M) w_c / L over the chunk partials the
//                       text kernel leaves when it attends over a dense cache
// The dense decode itself reuses the text kernel (decode.cuh) over the whole
// cache with long chunks, so both baselines attend with the same streaming
// kernel that the rank-space decode uses for its text tail.
#pragma once

#include "common.cuh"
#include "decode.cuh"

namespace kvpack {
namespace baseline {

constexpr int kDenseChunk = 1024;   // tokens per text-kernel item over a dense cache

// ------------------------------------------------------------------ decompress

constexpr int kDecThreads = 256;    // 8 warps x 16 tokens
constexpr int kDecTok = 128;

struct DecompressParams {
    const uint16_t *C_lo[2], *C_hi[2], *B[2];   // K side, V side
    const uint32_t *mask;
    uint16_t *out[2];                           // [units][L_cap][512]
    int T, L_cap, nwords, tiles, rank_lo;
};

struct DecSmem {
    alignas(128) unsigned char b[64 * 1024];     // B of one side: [64 ranks][512 features] bf16, 1 KB rows
    alignas(128) unsigned char c[kDecTok * 128];  // C rows [128 tokens][64] bf16, 16-byte chunk c at c ^ (r & 7)
    alignas(128) unsigned char st[8][16 * 256];   // per warp: 16 tokens x 128 features bf16 for the stores
};

__global__ void __launch_bounds__(kDecThreads, 1) decompress_kernel(const DecompressParams p) {
    extern __shared__ __align__(128) unsigned char dec_smem_raw[];
    DecSmem &sm = *reinterpret_cast<DecSmem *>(dec_smem_raw);
    const int unit = blockIdx.x / p.tiles, t0 = (blockIdx.x % p.tiles) * kDecTok;
    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const int g = lane >> 2, tig = lane & 3;
    for (int side = 0; side < 2; ++side) {
        // B (64 KB) and the tile's coefficient rows; a token's components past its rank are zero
        const uint16_t *bsrc = p.B[side] + (size_t)unit * 64 * 512;
        for (int i = tid; i < 64 * 512 / 8; i += kDecThreads) {
            const int k = i >> 6, c = i & 63;        // 16-byte chunk c of rank row k, stored at c ^ (k & 7)
            cp_async16(sm.b + k * 1024 + ((c ^ (k & 7)) << 4), bsrc + 8 * i);
        }
        for (int i = tid; i < kDecTok * 8; i += kDecThreads) {
            const int r = i >> 3, ch = i & 7, t = t0 + r;
            bool keep = t < p.T;
            if (keep) {
                const bool hi = (__ldg(p.mask + (size_t)unit * p.nwords + (t >> 5)) >> (t & 31)) & 1u;
                const int rho = hi ? 64 : p.rank_lo;
                keep = 8 * ch < rho;
            }
            const size_t row = (size_t)unit * p.T + (t < p.T ? t : 0);
            const uint16_t *src = ch < 2 ? p.C_lo[side] + row * 16 + ch * 8 : p.C_hi[side] + row * 48 + (ch - 2) * 8;
            cp_async16_zfill(sm.c + r * 128 + ((ch ^ (r & 7)) << 4), src, keep);
        }
        cp_async_wait_all();
        __syncthreads();
        // warp w: tokens 16 w .. 16 w + 15; four 128-feature chunks (one KV head each)
        uint32_t a[4][4];
        #pragma unroll
        for (int kb = 0; kb < 4; ++kb) {
            const int row = 16 * warp + (lane & 7) + (((lane >> 3) & 1) << 3);
            const int ch = 2 * kb + (lane >> 4);
            ldsm_x4(smem_u32(sm.c) + row * 128 + ((ch ^ (row & 7)) << 4), a[kb][0], a[kb][1], a[kb][2], a[kb][3]);
        }
        for (int j = 0; j < 4; ++j) {
            float acc[16][4];
            #pragma unroll
            for (int nt = 0; nt < 16; ++nt) acc[nt][0] = acc[nt][1] = acc[nt][2] = acc[nt][3] = 0.f;
            #pragma unroll
            for (int kb = 0; kb < 4; ++kb) {
                #pragma unroll
                for (int np = 0; np < 8; ++np) {
                    // B[k = rank][n = feature]: rows of 1 KB, features 128 j + 16 np ..
                    uint32_t b0, b1, b2, b3;
                    const int k = 16 * kb + (lane & 7) + (((lane >> 3) & 1) << 3);
                    const int c = 16 * j + 2 * np + (lane >> 4);   // 16-byte chunk of features 8c ..
                    ldsm_x4_t(smem_u32(sm.b) + k * 1024 + ((c ^ (k & 7)) << 4), b0, b1, b2, b3);
                    mma_bf16(acc[2 * np], a[kb], b0, b1);
                    mma_bf16(acc[2 * np + 1], a[kb], b2, b3);
                }
            }
            // stage as bf16 [16 tokens][128 features] (16-byte chunk c of row r at c ^ (r & 7)),
            // then 16-byte stores of whole rows
            unsigned char *stw = sm.st[warp];
            #pragma unroll
            for (int nt = 0; nt < 16; ++nt) {
                *reinterpret_cast<uint32_t *>(stw + g * 256 + ((nt ^ (g & 7)) << 4) + 4 * tig) =
                    pack_bf16(acc[nt][0], acc[nt][1]);
                *reinterpret_cast<uint32_t *>(stw + (g + 8) * 256 + ((nt ^ (g & 7)) << 4) + 4 * tig) =
                    pack_bf16(acc[nt][2], acc[nt][3]);
            }
            __syncwarp();
            #pragma unroll
            for (int i = 0; i < 8; ++i) {
                const int idx = lane + 32 * i;          // 16 rows x 16 chunks of 16 bytes
                const int r = idx >> 4, c = idx & 15;
                const int t = t0 + 16 * warp + r;
                if (t < p.T) {
                    uint16_t *dst = p.out[side] + ((size_t)unit * p.L_cap + t) * 512 + 128 * j + 8 * c;
                    *reinterpret_cast<uint4 *>(dst) = *reinterpret_cast<const uint4 *>(stw + r * 256 + ((c ^ (r & 7)) << 4));
                }
            }
            __syncwarp();
        }
        __syncthreads();
    }
}

// ------------------------------------------------------------------ dense finish

struct DenseFinishParams {
    const float *tpart;       // [units][Sc][Hg][kTxtPart] from text_kernel
    uint16_t *out;            // [(layer, batch)][n_q][128]
    int Hg, n_q, groups, Sc;
};

// One block of 128 threads per (unit, KV head j): per query head of j, the max M and sum L
// over the chunk partials, then o_h = sum_c 2^(m_c - M) w_c / L, thread t owning feature t.
template <int PK>
__global__ void __launch_bounds__(128) dense_finish_kernel(const DenseFinishParams p) {
    const int unit = blockIdx.x >> 2, j = blockIdx.x & 3, tid = threadIdx.x;
    const int lb = unit / p.groups, G = unit % p.groups;
    #pragma unroll
    for (int hh = 0; hh < PK; ++hh) {
        const int h = j * PK + hh;
        const float *tp = p.tpart + ((size_t)unit * p.Sc * p.Hg + h) * decode::kTxtPart;
        float mx = -INFINITY;
        for (int c = 0; c < p.Sc; ++c) mx = fmaxf(mx, __ldcg(tp + (size_t)c * p.Hg * decode::kTxtPart));
        float sum = 0.f, acc = 0.f;
        for (int c = 0; c < p.Sc; ++c) {
            const float *r = tp + (size_t)c * p.Hg * decode::kTxtPart;
            const float mc = __ldcg(r);
            if (mc == -INFINITY) continue;
            const float e = ex2(mc - mx);
            sum = fmaf(__ldcg(r + 1), e, sum);
            acc = fmaf(__ldcg(r + 2 + tid), e, acc);
        }
        p.out[((size_t)lb * p.n_q + (size_t)G * p.Hg + h) * 128 + tid] = float_to_bf16_bits(acc / sum);
    }
}

}  // namespace baseline
}  // namespace kvpack
