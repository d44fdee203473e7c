// compress.cuh -- multi-head SVD compression of the visual K (or V) cache
// (AttentionPack, technical summaries 2.A on the es / fr / de pages: the K
// vectors of a group of heads, concatenated along the feature axis, are
// factored by SVD into per-token coefficients and a decompression matrix;
// storage falls from T x H x D to T x R + R x H x D).
//
// Per unit X (T x 512, bf16) the rank-64 truncated SVD X ~ C B is computed as
//   1. gram_tc_kernel  G = X^T X (512 x 512, fp32 accumulation) on the 5th-
//                      generation tensor cores (tcgen05.mma, accumulator in tensor
//                      memory, operands staged by TMA); only the upper 128-row bands
//                      right of the diagonal are computed, then mirrored.
//   2. eig_kernel      top-64 eigenpairs of G by blocked subspace iteration
//                      with p = 96 columns: Y = G Q (three-product bf16 split
//                      on the tensor cores, ~fp32 accurate), then Y is
//                      orthonormalised by one-sided Jacobi in shared memory,
//                      which also aligns the basis with the Ritz vectors of G
//                      (the column norms are the Ritz estimates of lambda).
//                      Stops when the leading 64 estimates move by less than
//                      5e-4 relative; sigma_i = sqrt(lambda_i), B = Q_r^T.
//   3. project_kernel  C = X Q_r (Q_r carried as a bf16 hi + lo pair), rounded
//                      to bf16 and written as the C_lo / C_hi planes.
#pragma once

#include "common.cuh"

namespace kvpack {
namespace compress {

constexpr int kN = 512;               // features per unit (4 KV heads x 128)
constexpr int kP = 96;                // subspace dimension (64 + 32 oversampling)
constexpr int kR = 64;                // rank kept
constexpr int kQPitch = 400;          // bytes per row of the bf16 Q layout: hi[96] | lo[96] | pad
constexpr int kMaxIter = 40;
constexpr int kMaxSweeps = 12;
constexpr float kConvTol = 2e-3f;     // estimated remaining relative error of the top-64 sigma
constexpr float kJacobiTol = 2e-5f;   // off-orthogonality tolerance (fp32 dot products of length 512)

struct Workspace {
    float *G;            // [units][512][512]
    float *Yt;           // [units][96][512]   Y = G Q, column-major
    unsigned char *Qg;   // [units][512][kQPitch]  Q as bf16 hi / lo, columns sorted by Ritz value
    float *info;         // [units][4]: iterations, Jacobi sweeps of the last iteration, last change, error estimate
};

inline size_t align256(size_t x) { return (x + 255) & ~size_t(255); }

inline size_t ws_G(int units) { return align256((size_t)units * kN * kN * 4); }
inline size_t ws_Yt(int units) { return align256((size_t)units * kP * kN * 4); }
inline size_t ws_Qg(int units) { return align256((size_t)units * kN * kQPitch); }

inline size_t ws_info(int units) { return align256((size_t)units * 4 * 4); }

inline size_t workspace_bytes(int units, int T) {
    (void)T;
    return ws_G(units) + ws_Yt(units) + ws_Qg(units) + ws_info(units);
}

inline Workspace carve(void *ws, int units) {
    unsigned char *p = static_cast<unsigned char *>(ws);
    Workspace w;
    w.G = reinterpret_cast<float *>(p);
    w.Yt = reinterpret_cast<float *>(p + ws_G(units));
    w.Qg = p + ws_G(units) + ws_Yt(units);
    w.info = reinterpret_cast<float *>(p + ws_G(units) + ws_Yt(units) + ws_Qg(units));
    return w;
}


__device__ __forceinline__ void cp_async_commit() { asm volatile("cp.async.commit_group;" ::: "memory"); }

template <int N>
__device__ __forceinline__ void cp_async_wait() { asm volatile("cp.async.wait_group %0;" :: "n"(N) : "memory"); }



// ================================================================== eigen-solver

constexpr int kEigThreads = 512;
constexpr int kEigWarps = kEigThreads / 32;

struct EigSmem {
    alignas(128) unsigned char buf[kN * kQPitch];   // Q (bf16 hi/lo rows) or Y^T (fp32 columns)
    float lam[kP];          // Ritz estimates of this iteration (unsorted, by column)
    float lam_sorted[kP];
    float prev_sorted[kP];
    int rank[kP];           // sorted position of each column
    int inv[kP];            // column at each sorted position
    int rotations;
    int done;
    int sweeps;
    float prev_change;
};
static_assert(kN * kQPitch >= kP * kN * 4, "buffer must hold Y^T too");

// Deterministic +-1 start vectors (a multiplicative hash of row and column).
__device__ __forceinline__ float start_entry(int r, int c) {
    uint32_t h = (uint32_t)(r * 2654435761u) ^ (uint32_t)((c + 1) * 2246822519u);
    h ^= h >> 15; h *= 2654435761u; h ^= h >> 13;
    return (h & 1u) ? 0.04419417382415922f : -0.04419417382415922f;   // +-1/sqrt(512)
}

// Y = G Q for one matrix: warp w computes rows [32w, 32w+32) x 96 columns with
// three bf16 products per tile (G_hi Q_hi + G_hi Q_lo + G_lo Q_hi), fp32 accumulation;
// Y is written column-major to global memory.
__device__ void eig_gemm(const float *__restrict__ Gu, const unsigned char *qbuf, float *__restrict__ Ytu) {
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int g = lane >> 2, tig = lane & 3;
    const uint32_t qb = smem_u32(qbuf);
    float acc[2][12][4];
    #pragma unroll
    for (int a = 0; a < 2; ++a)
        #pragma unroll
        for (int b = 0; b < 12; ++b) acc[a][b][0] = acc[a][b][1] = acc[a][b][2] = acc[a][b][3] = 0.f;
    const int r0 = 32 * warp;
    float2 ga[2][4], gn[2][4];
    auto fetch = [&](int k0, float2 (&dst)[2][4]) {
        #pragma unroll
        for (int mt = 0; mt < 2; ++mt) {
            const float *row0 = Gu + (size_t)(r0 + 16 * mt + g) * kN + k0 + 2 * tig;
            const float *row1 = row0 + 8 * kN;
            dst[mt][0] = __ldcg(reinterpret_cast<const float2 *>(row0));
            dst[mt][1] = __ldcg(reinterpret_cast<const float2 *>(row1));
            dst[mt][2] = __ldcg(reinterpret_cast<const float2 *>(row0 + 8));
            dst[mt][3] = __ldcg(reinterpret_cast<const float2 *>(row1 + 8));
        }
    };
    fetch(0, ga);
    for (int k0 = 0; k0 < kN; k0 += 16) {
        if (k0 + 16 < kN) fetch(k0 + 16, gn);
        uint32_t ah[2][4], al[2][4];
        #pragma unroll
        for (int mt = 0; mt < 2; ++mt)
            #pragma unroll
            for (int e = 0; e < 4; ++e) split2(ga[mt][e].x, ga[mt][e].y, ah[mt][e], al[mt][e]);
        #pragma unroll
        for (int np = 0; np < 6; ++np) {
            uint32_t bh[4], bl[4];
            const int row = k0 + (lane & 7) + 8 * ((lane >> 3) & 1);
            const int col = 16 * np + 8 * (lane >> 4);
            const uint32_t a = qb + row * kQPitch + col * 2;
            ldsm_x4_t(a, bh[0], bh[1], bh[2], bh[3]);
            ldsm_x4_t(a + kP * 2, bl[0], bl[1], bl[2], bl[3]);
            #pragma unroll
            for (int mt = 0; mt < 2; ++mt) {
                mma_bf16(acc[mt][2 * np], ah[mt], bh[0], bh[1]);
                mma_bf16(acc[mt][2 * np], ah[mt], bl[0], bl[1]);
                mma_bf16(acc[mt][2 * np], al[mt], bh[0], bh[1]);
                mma_bf16(acc[mt][2 * np + 1], ah[mt], bh[2], bh[3]);
                mma_bf16(acc[mt][2 * np + 1], ah[mt], bl[2], bl[3]);
                mma_bf16(acc[mt][2 * np + 1], al[mt], bh[2], bh[3]);
            }
        }
        #pragma unroll
        for (int mt = 0; mt < 2; ++mt)
            #pragma unroll
            for (int e = 0; e < 4; ++e) ga[mt][e] = gn[mt][e];
    }
    #pragma unroll
    for (int mt = 0; mt < 2; ++mt)
        #pragma unroll
        for (int nt = 0; nt < 12; ++nt)
            #pragma unroll
            for (int e = 0; e < 4; ++e) {
                const int r = r0 + 16 * mt + g + 8 * (e >> 1);
                const int c = 8 * nt + 2 * tig + (e & 1);
                Ytu[(size_t)c * kN + r] = acc[mt][nt][e];
            }
}

// One-sided Jacobi on the columns of Y^T (96 columns of 512 fp32 in shared
// memory), parallel round-robin pair order: 48 disjoint pairs per round, 95
// rounds per sweep; a warp rotates 3 pairs per round.  Returns the sweeps used,
// or -1 if kMaxSweeps passed without convergence.
__device__ int eig_jacobi(float *Y, EigSmem &sm) {
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    for (int sweep = 1; sweep <= kMaxSweeps; ++sweep) {
        if (threadIdx.x == 0) sm.rotations = 0;
        __syncthreads();
        int mine = 0;
        for (int r = 0; r < kP - 1; ++r) {
            for (int k = warp; k < kP / 2; k += kEigWarps) {
                int a, b;
                if (k == 0) { a = r; b = kP - 1; }
                else { a = (r + k) % (kP - 1); b = (r - k + kP - 1) % (kP - 1); }
                float *ya = Y + a * kN, *yb = Y + b * kN;
                float al = 0.f, be = 0.f, ga = 0.f;
                float va[16], vb[16];
                #pragma unroll
                for (int j = 0; j < 16; ++j) {
                    va[j] = ya[lane + 32 * j];
                    vb[j] = yb[lane + 32 * j];
                    al = fmaf(va[j], va[j], al);
                    be = fmaf(vb[j], vb[j], be);
                    ga = fmaf(va[j], vb[j], ga);
                }
                #pragma unroll
                for (int d = 16; d > 0; d >>= 1) {
                    al += __shfl_xor_sync(0xffffffffu, al, d);
                    be += __shfl_xor_sync(0xffffffffu, be, d);
                    ga += __shfl_xor_sync(0xffffffffu, ga, d);
                }
                if (al > 0.f && be > 0.f && fabsf(ga) > kJacobiTol * sqrtf(al * be)) {
                    ++mine;
                    const float zeta = (be - al) / (2.f * ga);
                    const float t = copysignf(1.f, zeta) / (fabsf(zeta) + sqrtf(1.f + zeta * zeta));
                    const float c = rsqrtf(1.f + t * t), s = c * t;
                    #pragma unroll
                    for (int j = 0; j < 16; ++j) {
                        ya[lane + 32 * j] = c * va[j] - s * vb[j];
                        yb[lane + 32 * j] = s * va[j] + c * vb[j];
                    }
                }
            }
            __syncthreads();
        }
        if (lane == 0 && mine) atomicAdd(&sm.rotations, mine);
        __syncthreads();
        const int rot = sm.rotations;
        __syncthreads();
        if (rot == 0) return sweep;
    }
    return -1;
}

struct EigParams {
    Workspace ws;
    int max_iter;       // iteration cap (at most kMaxIter)
    uint16_t *B;        // [units][64][512]
    float *sigma;       // [units][64] or null
    int units;
};

__global__ void __launch_bounds__(kEigThreads, 1) eig_kernel(EigParams p) {
    extern __shared__ __align__(128) unsigned char eig_smem_raw[];
    EigSmem &sm = *reinterpret_cast<EigSmem *>(eig_smem_raw);
    const int unit = blockIdx.x;
    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const float *Gu = p.ws.G + (size_t)unit * kN * kN;
    float *Ytu = p.ws.Yt + (size_t)unit * kP * kN;
    unsigned char *Qgu = p.ws.Qg + (size_t)unit * kN * kQPitch;
    float *Ys = reinterpret_cast<float *>(sm.buf);

    // Q0 in the bf16 layout: row r = [hi 96 | lo 96]
    for (int i = tid; i < kN * kP; i += kEigThreads) {
        const int r = i / kP, c = i % kP;
        const float v = start_entry(r, c);
        const uint16_t h = float_to_bf16_bits(v);
        uint16_t *row = reinterpret_cast<uint16_t *>(sm.buf + r * kQPitch);
        row[c] = h;
        row[kP + c] = float_to_bf16_bits(v - bf16_bits_to_float(h));
    }
    if (tid < kP) sm.prev_sorted[tid] = 0.f;
    if (tid == 0) { sm.done = 0; sm.prev_change = 1.f; }
    __syncthreads();

    bool converged = false, jacobi_ok = true;
    for (int it = 0; it < p.max_iter; ++it) {
        // Y = G Q  (Q in the smem buffer), Y^T to global
        eig_gemm(Gu, sm.buf, Ytu);
        __threadfence_block();
        __syncthreads();
        // Y^T into shared memory (column-major fp32)
        for (int i = tid; i < kP * kN / 4; i += kEigThreads)
            reinterpret_cast<float4 *>(Ys)[i] = __ldcg(reinterpret_cast<const float4 *>(Ytu) + i);
        __syncthreads();
        const int sw = eig_jacobi(Ys, sm);
        jacobi_ok = sw >= 0;
        if (tid == 0) sm.sweeps = sw;
        // column norms = Ritz estimates of lambda
        for (int c = warp; c < kP; c += kEigWarps) {
            float s = 0.f;
            for (int j = lane; j < kN; j += 32) s = fmaf(Ys[c * kN + j], Ys[c * kN + j], s);
            #pragma unroll
            for (int d = 16; d > 0; d >>= 1) s += __shfl_xor_sync(0xffffffffu, s, d);
            if (lane == 0) sm.lam[c] = sqrtf(s);
        }
        __syncthreads();
        if (tid < kP) {
            const float v = sm.lam[tid];
            int rk = 0;
            for (int c = 0; c < kP; ++c) {
                const float u = sm.lam[c];
                rk += (u > v || (u == v && c < tid)) ? 1 : 0;
            }
            sm.rank[tid] = rk;
            sm.inv[rk] = tid;
            sm.lam_sorted[rk] = v;
        }
        __syncthreads();
        if (tid == 0) {
            // components below 1e-6 of the largest are numerically zero (rank-deficient G) and
            // are left out of the test
            // largest relative change of sigma = sqrt(lambda) among the leading 64; with the
            // ratio of successive changes as the contraction rate rho, the remaining error is
            // about change * rho / (1 - rho)
            float worst = 0.f;
            const float floor_l = 1e-6f * sm.lam_sorted[0];
            for (int i = 0; i < kR; ++i) {
                if (sm.lam_sorted[i] <= floor_l) continue;
                const float a = sqrtf(sm.lam_sorted[i]), b = sqrtf(sm.prev_sorted[i]);
                worst = fmaxf(worst, fabsf(a - b) / a);
            }
            const float rho = fminf(worst / fmaxf(sm.prev_change, 1e-30f), 0.95f);
            const float est = worst * rho / (1.f - rho);
            sm.done = (it >= 2 && est < kConvTol && worst < kConvTol) ? 1 : 0;
            sm.prev_change = worst;
            float *inf = p.ws.info + (size_t)unit * 4;
            inf[0] = (float)(it + 1); inf[1] = (float)sm.sweeps; inf[2] = worst; inf[3] = est;
        }
        __syncthreads();
        if (tid < kP) sm.prev_sorted[tid] = sm.lam_sorted[tid];
        converged = sm.done != 0;
        const bool last = converged || it == p.max_iter - 1;

        // Q for the next iteration: normalised columns in sorted order, bf16 hi / lo rows
        {
            const int r = tid;   // one row per thread
            unsigned char *dst = Qgu + (size_t)r * kQPitch;
            for (int c8 = 0; c8 < kP; c8 += 8) {
                uint32_t hw[4], lw[4];
                #pragma unroll
                for (int e = 0; e < 4; ++e) {
                    const int c0 = sm.inv[c8 + 2 * e], c1 = sm.inv[c8 + 2 * e + 1];
                    const float x0 = sm.lam[c0] > 0.f ? Ys[c0 * kN + r] / sm.lam[c0] : 0.f;
                    const float x1 = sm.lam[c1] > 0.f ? Ys[c1 * kN + r] / sm.lam[c1] : 0.f;
                    split2(x0, x1, hw[e], lw[e]);
                }
                *reinterpret_cast<uint4 *>(dst + c8 * 2) = make_uint4(hw[0], hw[1], hw[2], hw[3]);
                *reinterpret_cast<uint4 *>(dst + kP * 2 + c8 * 2) = make_uint4(lw[0], lw[1], lw[2], lw[3]);
            }
        }
        if (last) {
            // basis B = Q_r^T (bf16) and singular values sigma_i = sqrt(lambda_i)
            uint16_t *Bu = p.B + (size_t)unit * kR * kN;
            for (int i = tid; i < kR * kN; i += kEigThreads) {
                const int row = i / kN, col = i % kN;
                const int c = sm.inv[row];
                Bu[i] = float_to_bf16_bits(sm.lam[c] > 0.f ? Ys[c * kN + col] / sm.lam[c] : 0.f);
            }
            if (p.sigma != nullptr && tid < kR) p.sigma[(size_t)unit * kR + tid] = sqrtf(sm.lam_sorted[tid]);
            break;
        }
        __syncthreads();
        // reload Q into shared memory for the next product
        for (int i = tid; i < kN * kQPitch / 16; i += kEigThreads)
            reinterpret_cast<uint4 *>(sm.buf)[i] = __ldcg(reinterpret_cast<const uint4 *>(Qgu) + i);
        __syncthreads();
    }
    if (tid == 0 && (!converged || !jacobi_ok)) report_error(KVPACK_ERR_NOCONVERGE);
}

// ================================================================== projection

constexpr int kProjThreads = 256;
constexpr int kProjTok = 128;     // tokens per block (16 per warp)
constexpr int kProjKC = 64;       // features per chunk
constexpr int kProjQPitch = 272;  // bytes per row of the smem Q_r copy: hi[64] | lo[64] | pad

struct ProjSmem {
    alignas(128) unsigned char q[kN * kProjQPitch];            // Q_r hi / lo, rows = features
    alignas(128) unsigned char x[2][kProjTok * kProjKC * 2];  // X chunk [128 tokens][64 features], swizzled
};

__global__ void __launch_bounds__(kProjThreads, 1) project_kernel(const uint16_t *__restrict__ X, int T,
                                                                  Workspace ws, uint16_t *__restrict__ C_lo,
                                                                  uint16_t *__restrict__ C_hi, int tiles) {
    extern __shared__ __align__(128) unsigned char proj_smem_raw[];
    ProjSmem &sm = *reinterpret_cast<ProjSmem *>(proj_smem_raw);
    const int unit = blockIdx.x / tiles, tile = blockIdx.x % tiles;
    const int t0 = tile * kProjTok;
    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const int g = lane >> 2, tig = lane & 3;
    const uint16_t *xu = X + (size_t)unit * T * kN;
    const unsigned char *Qgu = ws.Qg + (size_t)unit * kN * kQPitch;

    // Q_r (first 64 sorted columns): hi at bytes [0,128), lo at [128,256) of each 272-byte row
    for (int i = tid; i < kN * 16; i += kProjThreads) {
        const int r = i >> 4, c = i & 15;
        const unsigned char *src = Qgu + (size_t)r * kQPitch + ((c < 8) ? c * 16 : kP * 2 + (c - 8) * 16);
        cp_async16(sm.q + r * kProjQPitch + c * 16, src);
    }
    auto load_x = [&](int stage, int f0) {
        for (int i = tid; i < kProjTok * 8; i += kProjThreads) {
            const int r = i >> 3, c = i & 7;
            const int tok = t0 + r;
            const bool ok = tok < T;
            cp_async16_zfill(sm.x[stage] + r * 128 + ((c ^ (r & 7)) << 4), xu + (size_t)(ok ? tok : 0) * kN + f0 + c * 8, ok);
        }
        cp_async_commit();
    };
    load_x(0, 0);

    float acc[8][4];
    #pragma unroll
    for (int a = 0; a < 8; ++a) acc[a][0] = acc[a][1] = acc[a][2] = acc[a][3] = 0.f;
    const uint32_t qb = smem_u32(sm.q);
    constexpr int nchunks = kN / kProjKC;
    for (int ch = 0; ch < nchunks; ++ch) {
        if (ch + 1 < nchunks) load_x((ch + 1) & 1, (ch + 1) * kProjKC);
        else cp_async_commit();
        cp_async_wait<1>();
        __syncthreads();
        const uint32_t xb = smem_u32(sm.x[ch & 1]);
        #pragma unroll
        for (int kk = 0; kk < kProjKC; kk += 16) {
            uint32_t a[4];
            {
                const int row = 16 * warp + (lane & 7) + 8 * ((lane >> 3) & 1);
                const int c = kk / 8 + (lane >> 4);
                ldsm_x4(xb + row * 128 + ((c ^ (row & 7)) << 4), a[0], a[1], a[2], a[3]);
            }
            #pragma unroll
            for (int np = 0; np < 4; ++np) {
                uint32_t bh[4], bl[4];
                const int row = ch * kProjKC + kk + (lane & 7) + 8 * ((lane >> 3) & 1);
                const int col = 16 * np + 8 * (lane >> 4);
                const uint32_t ad = qb + row * kProjQPitch + col * 2;
                ldsm_x4_t(ad, bh[0], bh[1], bh[2], bh[3]);
                ldsm_x4_t(ad + 128, bl[0], bl[1], bl[2], bl[3]);
                mma_bf16(acc[2 * np], a, bh[0], bh[1]);
                mma_bf16(acc[2 * np], a, bl[0], bl[1]);
                mma_bf16(acc[2 * np + 1], a, bh[2], bh[3]);
                mma_bf16(acc[2 * np + 1], a, bl[2], bl[3]);
            }
        }
        __syncthreads();
    }
    cp_async_wait<0>();
    #pragma unroll
    for (int nt = 0; nt < 8; ++nt)
        #pragma unroll
        for (int h = 0; h < 2; ++h) {
            const int tok = t0 + 16 * warp + g + 8 * h;
            if (tok >= T) continue;
            const int col = 8 * nt + 2 * tig;
            const uint32_t v = pack_bf16(acc[nt][2 * h], acc[nt][2 * h + 1]);
            const size_t row = (size_t)unit * T + tok;
            if (col < 16) *reinterpret_cast<uint32_t *>(C_lo + row * 16 + col) = v;
            else *reinterpret_cast<uint32_t *>(C_hi + row * 48 + (col - 16)) = v;
        }
}

// ================================================================== host side

// ------------------------------------------------------------ Gram on tcgen05
//
// G = X^T X per unit with the 5th-generation tensor cores.  A block owns one
// 128-row band I of G (feature rows 128 I ..) and its columns 128 I .. 511 (the
// upper triangle and the diagonal block), for one range of tokens:
//   * TMA streams 64-token chunks of X restricted to features 128 I .. 511
//     (boxes of 64 features x 64 tokens, 128-byte swizzle) through a 3-stage ring;
//   * one thread issues tcgen05.mma kind::f16 (bf16 in, fp32 accumulate in tensor
//     memory), M = 128 (the band's features), N <= 256 (columns), K = 16 tokens,
//     both operands read "MN-major" straight from the swizzled X tiles (a token is a
//     K row; the band's own 128 features are the first two boxes of the stage);
//   * tcgen05.commit releases a stage once its MMAs have read it;
//   * four warps move the accumulator (one tensor-memory lane per feature row) to
//     G and mirror the off-diagonal part into the lower triangle.
// Long token ranges are split 4:3:2:1 over the bands (equal work per block) and
// the splits add into a zeroed G with fp32 atomics.
constexpr int kGtTok = 64;         // tokens per stage
constexpr int kGtStages = 3;
constexpr int kGtThreads = 128;
constexpr uint32_t kGtStageBytes = 64 * 1024;   // the widest band: 8 boxes of 64 features x 64 tokens

struct GramTcParams {
    CUtensorMap tm_x;      // 3D {512, T, units} bf16, box {64, 64, 1}, 128-byte swizzle
    float *G;              // [units][512][512]
    int T, units;
    int splits[4];         // token splits of band I (the block count per unit is their sum)
    int atomic;            // add into a zeroed G (any band split) instead of storing
};

struct GramTcSmem {
    alignas(1024) unsigned char stage[kGtStages][kGtStageBytes];
    uint64_t full[kGtStages], empty[kGtStages], done;
    uint32_t tmem_base;
};

// tcgen05 shared-memory descriptor of an MN-major operand in 128-byte-swizzled
// tiles: 64-element MN blocks kLbo bytes apart, 8-row K groups 1024 bytes apart.
__device__ __forceinline__ uint64_t umma_desc_mn_sw128(uint32_t saddr, uint32_t lbo_bytes) {
    uint64_t d = 0;
    d |= (uint64_t)((saddr >> 4) & 0x3FFFu);
    d |= (uint64_t)((lbo_bytes >> 4) & 0x3FFFu) << 16;
    d |= (uint64_t)((1024u >> 4) & 0x3FFFu) << 32;
    d |= (uint64_t)1 << 46;          // descriptor version of sm_100
    d |= (uint64_t)2 << 61;          // 128-byte swizzle
    return d;
}

// tcgen05 instruction descriptor: bf16 x bf16 -> fp32, both operands MN-major, M x N
__device__ __forceinline__ uint32_t umma_idesc_bf16_mn(int M, int N) {
    return (1u << 4) | (1u << 7) | (1u << 10) | (1u << 15) | (1u << 16) | ((uint32_t)(N >> 3) << 17) |
           ((uint32_t)(M >> 4) << 24);
}




__global__ void __launch_bounds__(kGtThreads, 1) gram_tc_kernel(const __grid_constant__ GramTcParams p) {
    extern __shared__ __align__(1024) unsigned char smem_raw[];
    const uint32_t base0 = smem_u32(smem_raw);
    GramTcSmem &sm = *reinterpret_cast<GramTcSmem *>(smem_raw + ((1024u - (base0 & 1023u)) & 1023u));
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    __shared__ int abort_flag;
    volatile int *abort = &abort_flag;

    // block -> (unit, band I, split s)
    const int per_unit = p.splits[0] + p.splits[1] + p.splits[2] + p.splits[3];
    const int unit = blockIdx.x / per_unit;
    int r = blockIdx.x % per_unit, I = 0;
    while (r >= p.splits[I]) { r -= p.splits[I]; ++I; }
    const int nsplit = p.splits[I], s = r;
    const int nch = (p.T + kGtTok - 1) / kGtTok;
    const int c0 = (int)(((long long)s * nch) / nsplit), c1 = (int)(((long long)(s + 1) * nch) / nsplit);
    const int NI = 512 - 128 * I;          // accumulator columns (features 128 I .. 511)
    const int nbox = NI / 64;
    const uint32_t sbytes = (uint32_t)nbox * 8192u;

    if (threadIdx.x == 0) {
        for (int i = 0; i < kGtStages; ++i) { mbar_init(&sm.full[i], 1); mbar_init(&sm.empty[i], 1); }
        mbar_init(&sm.done, 1);
        abort_flag = 0;
        asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
    }
    if (warp == 1) tmem_alloc(&sm.tmem_base, 512);
    tmem_fence_before();
    __syncthreads();
    tmem_fence_after();
    const uint32_t tmem = sm.tmem_base;

    if (c1 > c0) {
        if (warp == 0 && lane == 0) {
            // producer
            for (int c = c0; c < c1; ++c) {
                const int i = c - c0, slot = i % kGtStages;
                if (i >= kGtStages && !mbar_wait(&sm.empty[slot], ((i / kGtStages) - 1) & 1u, abort)) break;
                mbar_arrive_tx(&sm.full[slot], sbytes);
                for (int b = 0; b < nbox; ++b)
                    tma_3d(sm.stage[slot] + 8192 * b, &p.tm_x, 128 * I + 64 * b, kGtTok * c, unit, &sm.full[slot]);
            }
        } else if (warp == 1 && lane == 0) {
            // MMA issuer
            const uint32_t id256 = umma_idesc_bf16_mn(128, 256), id128 = umma_idesc_bf16_mn(128, 128);
            for (int c = c0; c < c1; ++c) {
                const int i = c - c0, slot = i % kGtStages;
                if (!mbar_wait(&sm.full[slot], (i / kGtStages) & 1u, abort)) break;
                tmem_fence_after();
                const uint32_t st = smem_u32(sm.stage[slot]);
                #pragma unroll
                for (int k = 0; k < kGtTok / 16; ++k) {
                    const uint64_t a = umma_desc_mn_sw128(st + 2048u * k, 8192u);
                    for (int n0 = 0; n0 < NI; n0 += 256) {
                        const int nn = min(256, NI - n0);
                        const uint64_t b = umma_desc_mn_sw128(st + 8192u * (n0 / 64) + 2048u * k, 8192u);
                        umma_bf16(tmem + (uint32_t)n0, a, b, nn == 256 ? id256 : id128, (c > c0 || k > 0) ? 1u : 0u);
                    }
                }
                umma_commit(&sm.empty[slot]);
            }
            umma_commit(&sm.done);
        }
        __syncwarp();
        // epilogue: warp w holds feature rows 32 w .. 32 w + 31 of the band (tensor-memory lanes)
        const bool ok = mbar_wait(&sm.done, 0u, abort);
        tmem_fence_after();
        if (ok) {
            const int row = 128 * I + 32 * warp + lane;
            float *grow = p.G + ((size_t)unit * 512 + row) * 512;
            for (int col0 = 0; col0 < NI; col0 += 32) {
                float v[32];
                tmem_ld32(tmem + ((uint32_t)(32 * warp) << 16) + (uint32_t)col0, v);
                tmem_wait_ld();
                const int J0 = 128 * I + col0;
                if (p.atomic) {
                    #pragma unroll
                    for (int j = 0; j < 32; ++j) atomicAdd(grow + J0 + j, v[j]);
                } else {
                    #pragma unroll
                    for (int j = 0; j < 32; j += 4)
                        *reinterpret_cast<float4 *>(grow + J0 + j) = make_float4(v[j], v[j + 1], v[j + 2], v[j + 3]);
                }
                if (J0 >= 128 * (I + 1)) {   // off the diagonal block: mirror (lanes write consecutive rows)
                    float *gcol = p.G + (size_t)unit * 512 * 512 + row;
                    #pragma unroll
                    for (int j = 0; j < 32; ++j) {
                        if (p.atomic) atomicAdd(gcol + (size_t)(J0 + j) * 512, v[j]);
                        else gcol[(size_t)(J0 + j) * 512] = v[j];
                    }
                }
            }
        }
    }
    tmem_fence_before();
    __syncthreads();
    if (warp == 1) {
        tmem_fence_after();
        tmem_dealloc(tmem, 512);
    }
}

// block counts of the four bands: equal work per block (4:3:2:1) once T is long
inline void gram_tc_splits(int T, int (&sp)[4]) {
    const int f = T >= 8192 ? (T + 8191) / 8192 : 0;
    for (int I = 0; I < 4; ++I) sp[I] = f ? f * (4 - I) : 1;
}

inline size_t gram_tc_smem() { return sizeof(GramTcSmem) + 1024; }

inline kvpack_status prepare_device() {
    if (cudaFuncSetAttribute(gram_tc_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)gram_tc_smem()) != cudaSuccess)
        return KVPACK_ERR_CUDA;
    if (cudaFuncSetAttribute(eig_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)sizeof(EigSmem)) != cudaSuccess)
        return KVPACK_ERR_CUDA;
    if (cudaFuncSetAttribute(project_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)sizeof(ProjSmem)) !=
        cudaSuccess)
        return KVPACK_ERR_CUDA;
    return KVPACK_OK;
}

inline kvpack_status run(int units, int T, const uint16_t *X, const CUtensorMap &tm_x, uint16_t *C_lo,
                         uint16_t *C_hi, uint16_t *B, float *sigma, void *ws, int sms, int max_iter, cudaStream_t st) {
    (void)sms;
    Workspace w = carve(ws, units);
    GramTcParams gp;
    gp.tm_x = tm_x;
    gp.G = w.G;
    gp.T = T;
    gp.units = units;
    gram_tc_splits(T, gp.splits);
    gp.atomic = gp.splits[3] > 1 ? 1 : 0;
    if (gp.atomic && cudaMemsetAsync(w.G, 0, (size_t)units * 512 * 512 * sizeof(float), st) != cudaSuccess)
        return KVPACK_ERR_CUDA;
    const int per_unit = gp.splits[0] + gp.splits[1] + gp.splits[2] + gp.splits[3];
    gram_tc_kernel<<<units * per_unit, kGtThreads, gram_tc_smem(), st>>>(gp);
    if (cudaGetLastError() != cudaSuccess) return KVPACK_ERR_CUDA;
    EigParams ep{w, max_iter, B, sigma, units};
    eig_kernel<<<units, kEigThreads, sizeof(EigSmem), st>>>(ep);
    if (cudaGetLastError() != cudaSuccess) return KVPACK_ERR_CUDA;
    const int tiles = (T + kProjTok - 1) / kProjTok;
    project_kernel<<<units * tiles, kProjThreads, sizeof(ProjSmem), st>>>(X, T, w, C_lo, C_hi, tiles);
    if (cudaGetLastError() != cudaSuccess) return KVPACK_ERR_CUDA;
    return KVPACK_OK;
}

}  // namespace compress
}  // namespace kvpack
