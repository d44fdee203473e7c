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
//   2. eig_kernel      top-64 eigenpairs of G by blocked subspace (orthogonal)
//                      iteration with p = 96 columns: Y = G Q (three-product bf16
//                      split on the tensor cores, ~fp32 accurate), Rayleigh-Ritz
//                      every third iteration (96 x 96 Jacobi), Cholesky QR of the
//                      columns scaled by their Ritz values; sigma_i = sqrt(theta_i),
//                      B = the leading 64 Ritz vectors.
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
constexpr int kMaxIter = 60;
constexpr int kMaxSweeps = 16;        // Jacobi sweeps of one 96 x 96 Rayleigh-Ritz problem
constexpr float kConvTol = 3e-3f;     // estimated remaining relative error of the top-64 sigma (bound: 1e-2)

struct Workspace {
    float *G;            // [units][512][512]
    float *Yt;           // [units][96][512]   Y = G Q, column-major
    float *Zt;           // [units][96][512]   Z = Y V Theta^-1 (Rayleigh-Ritz iterations), column-major
    float *Qt;           // [units][96][512]   Q in fp32, column-major
    unsigned char *Qg;   // [units][512][kQPitch]  Q as bf16 hi / lo, columns sorted by Ritz value
    float *info;         // [units][4]: iterations, Jacobi sweeps of the last Rayleigh-Ritz step, last change, error estimate
};

inline size_t align256(size_t x) { return (x + 255) & ~size_t(255); }

inline size_t ws_G(int units) { return align256((size_t)units * kN * kN * 4); }
inline size_t ws_Yt(int units) { return align256((size_t)units * kP * kN * 4); }
inline size_t ws_Qg(int units) { return align256((size_t)units * kN * kQPitch); }

inline size_t ws_info(int units) { return align256((size_t)units * 4 * 4); }

inline size_t workspace_bytes(int units, int T) {
    (void)T;
    return ws_G(units) + 3 * ws_Yt(units) + ws_Qg(units) + ws_info(units);
}

inline Workspace carve(void *ws, int units) {
    unsigned char *p = static_cast<unsigned char *>(ws);
    Workspace w;
    w.G = reinterpret_cast<float *>(p);
    p += ws_G(units);
    w.Yt = reinterpret_cast<float *>(p);
    p += ws_Yt(units);
    w.Zt = reinterpret_cast<float *>(p);
    p += ws_Yt(units);
    w.Qt = reinterpret_cast<float *>(p);
    p += ws_Yt(units);
    w.Qg = p;
    p += ws_Qg(units);
    w.info = reinterpret_cast<float *>(p);
    return w;
}


__device__ __forceinline__ void cp_async_commit() { asm volatile("cp.async.commit_group;" ::: "memory"); }

template <int N>
__device__ __forceinline__ void cp_async_wait() { asm volatile("cp.async.wait_group %0;" :: "n"(N) : "memory"); }



// ================================================================== eigen-solver
//
// Orthogonal (blocked subspace) iteration on G with p = 96 columns and a Rayleigh-Ritz step
// on the first and every third iteration:
//   Y = G Q                       tensor cores, three-product bf16 split (~fp32 accurate)
//   Rayleigh-Ritz iterations:     H = Q^T Y (96 x 96) = V Theta V^T by cyclic two-sided Jacobi;
//                                 Z = Y V Theta^-1, columns sorted by Ritz value
//   other iterations:             Z = Y D^-1, D = diag(Q^T Y) (the columns' Rayleigh quotients)
//   Q = Z R^-1 with Z^T Z = R^T R (Cholesky QR)
// Dividing each column by its Ritz value / Rayleigh quotient leaves Z's columns near unit
// length and near orthogonal, so a single fp32 Cholesky QR pass is accurate; the triangular R
// keeps Gram-Schmidt order (largest first), so between Rayleigh-Ritz steps the columns stay
// close to eigenvectors, as in orthogonal iteration.  The iteration stops when the Ritz
// estimates of the leading 64 sigma move by less than kConvTol between Rayleigh-Ritz steps
// (extrapolated with the observed contraction rate); B = the leading 64 Ritz vectors,
// sigma_i = sqrt(theta_i).
//
// One 512-thread block per unit.  The 96 x 96 work (H, Z^T Z, Jacobi, Cholesky, R^-1) lives in
// shared memory; Y, Z and Q (96 columns of 512 fp32, one column per row of the array) live in
// the workspace, which stays in L2.

constexpr int kEigThreads = 512;
constexpr int kEigWarps = kEigThreads / 32;
constexpr int kStageRows = 32;          // contraction rows per staged chunk of a 96 x 96 product
constexpr int kStagePitch = kP + 1;     // the staging buffer: 2 x 32 x 97 floats, room for four bf16 planes
constexpr float kJacTol = 1e-6f;        // rotate when |a_pq| > kJacTol sqrt(|a_pp a_qq|) ...
constexpr float kJacFloor = 1e-7f;      // ... and |a_pq| > kJacFloor max |a_ii| (fp32 rounding level)
constexpr float kJacQuad = 1e-3f;       // a sweep whose largest ratio is below this is the last (~sqrt(kJacTol))
constexpr float kPivTol = 1e-4f;        // Cholesky pivot below this fraction of its diagonal: dependent column
constexpr float kThetaFloor = 1e-7f;    // Ritz values below this fraction of the largest are taken as zero

struct EigWork {                        // the 96 x 96 phase, laid over the Q buffer
    float A[kP * kP];                   // H or W = Z^T Z (row-major)
    float V[kP * kP];                   // Jacobi rotations, then the Cholesky factor R
    float M[kP * kP];                   // the matrix that mixes the columns of Y or Z
    float st[2][kStageRows * kStagePitch];
};

struct EigSmem {
    alignas(128) unsigned char buf[kN * kQPitch];   // Q as bf16 hi / lo rows for the product | EigWork
    float theta[kP];        // Ritz values, sorted (descending)
    float prev[kP];         // the previous Rayleigh-Ritz step's sorted values
    float scale[kP];        // column scale of Z (1 / Rayleigh quotient), 0 for a dead column
    float diag0[kP];        // diagonal of W before the Cholesky updates
    int inv[kP];            // column of H at each sorted position
    int rot_p[kP / 2], rot_q[kP / 2];
    float rot_c[kP / 2], rot_s[kP / 2];
    float amax;
    float red2[2];
    int done;
    float prev_change;
};
static_assert(sizeof(EigWork) <= kN * kQPitch, "the 96 x 96 phase must fit in the Q buffer");

// Start vectors: 96 columns of a 512 x 512 Sylvester-Hadamard matrix with hashed row signs,
// scaled by 1/sqrt(512) (exactly orthonormal).
__device__ __forceinline__ float start_entry(int r, int c) {
    uint32_t h = (uint32_t)(r + 1) * 2654435761u;
    h ^= h >> 15; h *= 2246822519u; h ^= h >> 13;
    const int par = (__popc((uint32_t)r & (uint32_t)(c + 1)) + (int)(h & 1u)) & 1;
    return par ? -0.04419417382415922f : 0.04419417382415922f;
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

// C[i][j] = sum_r At[i][r] Bt[j][r] for i, j < 96, where At and Bt hold 96 columns of 512
// fp32 (column i contiguous), on the tensor cores: both operands split into bf16 hi + lo
// planes, three products (hi hi, hi lo, lo hi) with fp32 accumulation (~2^-16 relative, as the
// G Q product).
// 32-row chunks of the contraction are staged in shared memory as bf16 rows of 32 (one row per
// column i or j: K-major for both mma.sync operands; the 16-byte chunk c of row x sits at
// c ^ ((x >> 1) & 3), so the 8-row ldmatrix reads are free of bank conflicts); warp w < 12
// computes columns 8w .. 8w + 7 of C for all 96 rows.
__device__ void small_gram(const float *__restrict__ At, const float *__restrict__ Bt, float *C, EigWork &wk) {
    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const int g = lane >> 2, tig = lane & 3;
    // planes of 96 rows x 64 bytes: A hi, A lo, B hi, B lo
    unsigned char *st = reinterpret_cast<unsigned char *>(&wk.st[0][0]);
    const uint32_t st_s = smem_u32(st);
    constexpr uint32_t kPlane = kP * 64;
    static_assert(4 * kPlane <= sizeof(wk.st), "staging planes");
    float acc[6][4];
    #pragma unroll
    for (int mt = 0; mt < 6; ++mt) acc[mt][0] = acc[mt][1] = acc[mt][2] = acc[mt][3] = 0.f;
    for (int r0 = 0; r0 < kN; r0 += 32) {
        __syncthreads();
        // stage: thread t takes operand t / 256, column c, rows 4 q4 .. 4 q4 + 3 of the chunk
        for (int i = tid; i < 2 * kP * 8; i += kEigThreads) {
            const int op = i / (kP * 8), c = (i / 8) % kP, q4 = i % 8;
            const float4 v = __ldcg(reinterpret_cast<const float4 *>((op ? Bt : At) + (size_t)c * kN + r0 + 4 * q4));
            uint32_t h01, l01, h23, l23;
            split2(v.x, v.y, h01, l01);
            split2(v.z, v.w, h23, l23);
            const uint32_t off = (uint32_t)c * 64 + ((((q4 >> 1) ^ ((c >> 1) & 3))) << 4) + (q4 & 1) * 8;
            unsigned char *hp = st + (2 * op) * kPlane + off, *lp = st + (2 * op + 1) * kPlane + off;
            *reinterpret_cast<uint2 *>(hp) = make_uint2(h01, h23);
            *reinterpret_cast<uint2 *>(lp) = make_uint2(l01, l23);
        }
        __syncthreads();
        if (warp < 12) {
            #pragma unroll
            for (int ks = 0; ks < 2; ++ks) {
                // B (the warp's 8 columns, k 16 ks ..): rows n = 8 warp + (lane & 7), chunk 2 ks + ((lane >> 3) & 1)
                const int nrow = 8 * warp + (lane & 7);
                const uint32_t boff = (uint32_t)nrow * 64 + (((2 * ks + ((lane >> 3) & 1)) ^ ((nrow >> 1) & 3)) << 4);
                uint32_t bh0, bh1, bl0, bl1;
                asm volatile("ldmatrix.sync.aligned.m8n8.x2.shared.b16 {%0,%1}, [%2];"
                             : "=r"(bh0), "=r"(bh1) : "r"(st_s + 2 * kPlane + boff));
                asm volatile("ldmatrix.sync.aligned.m8n8.x2.shared.b16 {%0,%1}, [%2];"
                             : "=r"(bl0), "=r"(bl1) : "r"(st_s + 3 * kPlane + boff));
                #pragma unroll
                for (int mt = 0; mt < 6; ++mt) {
                    // A (rows 16 mt ..): matrices (rows 0-7, k 0-7), (8-15, 0-7), (0-7, 8-15), (8-15, 8-15)
                    const int arow = 16 * mt + (lane & 7) + (((lane >> 3) & 1) << 3);
                    const uint32_t aoff =
                        (uint32_t)arow * 64 + (((2 * ks + ((lane >> 4) & 1)) ^ ((arow >> 1) & 3)) << 4);
                    uint32_t ah[4], al[4];
                    ldsm_x4(st_s + aoff, ah[0], ah[1], ah[2], ah[3]);
                    ldsm_x4(st_s + kPlane + aoff, al[0], al[1], al[2], al[3]);
                    mma_bf16(acc[mt], ah, bh0, bh1);
                    mma_bf16(acc[mt], ah, bl0, bl1);
                    mma_bf16(acc[mt], al, bh0, bh1);
                }
            }
        }
    }
    if (warp < 12) {
        #pragma unroll
        for (int mt = 0; mt < 6; ++mt) {
            const int r = 16 * mt + g, c = 8 * warp + 2 * tig;
            C[r * kP + c] = acc[mt][0];
            C[r * kP + c + 1] = acc[mt][1];
            C[(r + 8) * kP + c] = acc[mt][2];
            C[(r + 8) * kP + c + 1] = acc[mt][3];
        }
    }
    __syncthreads();
}

// out[j][r] = sum_i in[i][r] M[i][j] for the 96 columns j (in and out: 96 columns of 512 fp32,
// column-contiguous; one thread per row r).  Optional outputs: out (fp32), the bf16 hi / lo row
// layout qg, and the bf16 rows of the basis B (its first 64 columns, B[j][r]).
__device__ void rowmix(const float *__restrict__ in, const float *M, float *__restrict__ out,
                       unsigned char *__restrict__ qg, uint16_t *__restrict__ Bout) {
    const int r = threadIdx.x;
    #pragma unroll 1
    for (int h = 0; h < kP; h += 48) {
        float acc[48];
        #pragma unroll
        for (int j = 0; j < 48; ++j) acc[j] = 0.f;
        #pragma unroll 4
        for (int i = 0; i < kP; ++i) {
            const float x = __ldcg(in + (size_t)i * kN + r);
            const float4 *m = reinterpret_cast<const float4 *>(M + i * kP + h);
            #pragma unroll
            for (int q = 0; q < 12; ++q) {
                const float4 v = m[q];
                acc[4 * q + 0] = fmaf(x, v.x, acc[4 * q + 0]);
                acc[4 * q + 1] = fmaf(x, v.y, acc[4 * q + 1]);
                acc[4 * q + 2] = fmaf(x, v.z, acc[4 * q + 2]);
                acc[4 * q + 3] = fmaf(x, v.w, acc[4 * q + 3]);
            }
        }
        if (out != nullptr) {
            #pragma unroll
            for (int j = 0; j < 48; ++j) out[(size_t)(h + j) * kN + r] = acc[j];
        }
        if (qg != nullptr) {
            unsigned char *row = qg + (size_t)r * kQPitch;
            #pragma unroll
            for (int c8 = 0; c8 < 48; c8 += 8) {
                uint32_t hw[4], lw[4];
                #pragma unroll
                for (int e = 0; e < 4; ++e) split2(acc[c8 + 2 * e], acc[c8 + 2 * e + 1], hw[e], lw[e]);
                *reinterpret_cast<uint4 *>(row + (h + c8) * 2) = make_uint4(hw[0], hw[1], hw[2], hw[3]);
                *reinterpret_cast<uint4 *>(row + kP * 2 + (h + c8) * 2) = make_uint4(lw[0], lw[1], lw[2], lw[3]);
            }
        }
        if (Bout != nullptr) {
            #pragma unroll
            for (int j = 0; j < 48; ++j)
                if (h + j < kR) Bout[(size_t)(h + j) * kN + r] = float_to_bf16_bits(acc[j]);
        }
    }
}

// Cyclic two-sided Jacobi on the symmetric 96 x 96 matrix A (row-major, both triangles),
// V = the product of the rotations (A -> V^T A V).  Parallel round-robin order: 48 disjoint
// pairs per round, 95 rounds per sweep; each 2 x 2 block of A is rotated in place by one
// thread.  The largest relative off-diagonal |a_pq| / sqrt(|a_pp a_qq|) met in a sweep decides
// the end: none above kJacTol means converged; all below sqrt(kJacTol) means this sweep's
// rotations leave them near kJacTol (Jacobi converges quadratically), so no further sweep is
// run.  Returns the sweeps used, or -1 after kMaxSweeps without convergence.
__device__ int jacobi96(float *A, float *V, EigSmem &sm) {
    const int tid = threadIdx.x, lane = tid & 31;
    constexpr int kPairs = kP / 2;
    for (int e = tid; e < kP * kP; e += kEigThreads) V[e] = (e / kP == e % kP) ? 1.f : 0.f;
    for (int sweep = 1; sweep <= kMaxSweeps; ++sweep) {
        __syncthreads();
        if (tid < 32) {
            float m = 0.f;
            for (int i = lane; i < kP; i += 32) m = fmaxf(m, fabsf(A[i * kP + i]));
            #pragma unroll
            for (int d = 16; d > 0; d >>= 1) m = fmaxf(m, __shfl_xor_sync(0xffffffffu, m, d));
            if (lane == 0) sm.amax = m;
        }
        __syncthreads();
        const float floor_a = kJacFloor * sm.amax;
        float worst = 0.f;                      // rotating threads: largest relative off-diagonal seen
        for (int rd = 0; rd < kP - 1; ++rd) {
            if (tid < kPairs) {
                const int k = tid;
                int p, q;
                if (k == 0) { p = rd; q = kP - 1; }
                else { p = (rd + k) % (kP - 1); q = (rd - k + kP - 1) % (kP - 1); }
                const float app = A[p * kP + p], aqq = A[q * kP + q], apq = A[p * kP + q];
                float c = 1.f, s = 0.f;
                const float ref = sqrtf(fabsf(app * aqq));
                if (fabsf(apq) > floor_a) worst = fmaxf(worst, fabsf(apq) / fmaxf(ref, 1e-30f));
                if (fabsf(apq) > kJacTol * ref && fabsf(apq) > floor_a) {
                    const float zeta = (aqq - app) / (2.f * apq);
                    const float t = copysignf(1.f, zeta) / (fabsf(zeta) + sqrtf(1.f + zeta * zeta));
                    c = 1.f / sqrtf(1.f + t * t);
                    s = c * t;
                }
                sm.rot_p[k] = p; sm.rot_q[k] = q; sm.rot_c[k] = c; sm.rot_s[k] = s;
            }
            __syncthreads();
            for (int blk = tid; blk < kPairs * kPairs; blk += kEigThreads) {
                const int a = blk / kPairs, b = blk - a * kPairs;
                const float sa = sm.rot_s[a], sb = sm.rot_s[b];
                if (sa == 0.f && sb == 0.f) continue;
                const float ca = sm.rot_c[a], cb = sm.rot_c[b];
                const int pa = sm.rot_p[a], qa = sm.rot_q[a], pb = sm.rot_p[b], qb = sm.rot_q[b];
                const float x11 = A[pa * kP + pb], x12 = A[pa * kP + qb];
                const float x21 = A[qa * kP + pb], x22 = A[qa * kP + qb];
                const float y11 = ca * x11 - sa * x21, y12 = ca * x12 - sa * x22;   // rows
                const float y21 = sa * x11 + ca * x21, y22 = sa * x12 + ca * x22;
                float z11 = cb * y11 - sb * y12, z12 = sb * y11 + cb * y12;          // columns
                float z21 = cb * y21 - sb * y22, z22 = sb * y21 + cb * y22;
                if (a == b) z12 = z21 = 0.f;                                        // the annihilated pair
                A[pa * kP + pb] = z11; A[pa * kP + qb] = z12;
                A[qa * kP + pb] = z21; A[qa * kP + qb] = z22;
            }
            for (int e = tid; e < kP * kPairs; e += kEigThreads) {
                const int i = e / kPairs, k = e - i * kPairs;
                const float s = sm.rot_s[k];
                if (s == 0.f) continue;
                const float c = sm.rot_c[k];
                const int p = sm.rot_p[k], q = sm.rot_q[k];
                const float vp = V[i * kP + p], vq = V[i * kP + q];
                V[i * kP + p] = c * vp - s * vq;
                V[i * kP + q] = s * vp + c * vq;
            }
            __syncthreads();
        }
        // the sweep's largest relative off-diagonal over the 48 rotating threads (warps 0 and 1)
        if (tid < 64) {
            float m = worst;
            #pragma unroll
            for (int d = 16; d > 0; d >>= 1) m = fmaxf(m, __shfl_xor_sync(0xffffffffu, m, d));
            if (lane == 0) sm.red2[tid >> 5] = m;
        }
        __syncthreads();
        const float sweep_worst = fmaxf(sm.red2[0], sm.red2[1]);
        if (sweep_worst <= kJacTol || sweep_worst < kJacQuad) return sweep;
    }
    return -1;
}

// W = R^T R (R upper triangular, written to R; the lower triangle is zeroed).  A holds W on
// entry and is overwritten by the trailing updates.  A pivot at or below kPivTol of its
// column's original diagonal marks a dependent (or dead) column: its row of R is zero.
// Trailing updates: thread (ti, tj) of a 16 x 32 grid takes rows k+1+ti+16m, columns k+1+tj+32n.
__device__ void cholesky96(float *A, float *R, EigSmem &sm) {
    const int tid = threadIdx.x, ti = tid >> 5, tj = tid & 31;
    if (tid < kP) sm.diag0[tid] = A[tid * kP + tid];
    for (int e = tid; e < kP * kP; e += kEigThreads) R[e] = 0.f;
    __syncthreads();
    for (int k = 0; k < kP; ++k) {
        const float piv = A[k * kP + k];
        const bool ok = piv > kPivTol * sm.diag0[k] && piv > 0.f;
        if (ok) {
            const float rk = sqrtf(piv), inv_piv = 1.f / piv, inv_rk = 1.f / rk;
            if (tid >= k && tid < kP) R[k * kP + tid] = tid == k ? rk : A[k * kP + tid] * inv_rk;
            for (int i = k + 1 + ti; i < kP; i += 16) {
                const float aki = A[k * kP + i] * inv_piv;
                for (int j = i + ((tj - (i - k - 1)) & 31); j < kP; j += 32) {
                    // columns j >= i of row i, each thread a fixed residue of j - (k + 1) mod 32
                    A[i * kP + j] -= aki * A[k * kP + j];
                }
            }
        }
        __syncthreads();
    }
}

// X = R^-1 for the upper-triangular R of cholesky96 (a zero row of R gives a zero row and
// column of X), by 16 x 16 blocks: the six diagonal blocks are inverted by back substitution,
// one warp each, a column per lane; then, block row by block row from the bottom,
// X_IJ = -X_II (sum_{I<K<=J} R_IK X_KJ) for every J > I at once.
__device__ void tri_inverse96(const float *R, float *X, float *T) {
    constexpr int kB = 16, kNB = kP / kB;
    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    for (int e = tid; e < kP * kP; e += kEigThreads) X[e] = 0.f;
    __syncthreads();
    if (warp < kNB && lane < kB) {
        const int o = warp * kB, j = o + lane;
        for (int i = j; i >= o; --i) {
            const float rii = R[i * kP + i];
            float sum = i == j ? 1.f : 0.f;
            for (int k = i + 1; k <= j; ++k) sum = fmaf(-R[i * kP + k], X[k * kP + j], sum);
            X[i * kP + j] = rii > 0.f ? sum / rii : 0.f;
        }
    }
    __syncthreads();
    for (int I = kNB - 2; I >= 0; --I) {
        const int oI = I * kB, ncol = kP - (oI + kB);        // columns right of the diagonal block
        // T = R[I rows, (I, J] ] X[(I, J], J cols] for every column of the blocks right of I
        for (int e = tid; e < kB * ncol; e += kEigThreads) {
            const int i = e / ncol, jc = oI + kB + (e - (e / ncol) * ncol);
            const int kend = jc;                               // X[k][jc] = 0 for k > jc
            float sum = 0.f;
            for (int k = oI + kB; k <= kend; ++k) sum = fmaf(R[(oI + i) * kP + k], X[k * kP + jc], sum);
            T[i * kP + jc] = sum;
        }
        __syncthreads();
        for (int e = tid; e < kB * ncol; e += kEigThreads) {
            const int i = e / ncol, jc = oI + kB + (e - (e / ncol) * ncol);
            float sum = 0.f;
            for (int k = i; k < kB; ++k) sum = fmaf(X[(oI + i) * kP + oI + k], T[k * kP + jc], sum);
            X[(oI + i) * kP + jc] = -sum;
        }
        __syncthreads();
    }
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
    EigWork &wk = *reinterpret_cast<EigWork *>(sm.buf);
    const int unit = blockIdx.x;
    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const float *Gu = p.ws.G + (size_t)unit * kN * kN;
    float *Yt = p.ws.Yt + (size_t)unit * kP * kN;
    float *Zt = p.ws.Zt + (size_t)unit * kP * kN;
    float *Qt = p.ws.Qt + (size_t)unit * kP * kN;
    unsigned char *Qgu = p.ws.Qg + (size_t)unit * kN * kQPitch;

    // the Gram kernel writes the diagonal 128-row blocks of G and the blocks right of them; the
    // blocks left of the diagonal are their transposes
    {
        float *Gw = p.ws.G + (size_t)unit * kN * kN;
        for (int e = tid; e < kN * kN; e += kEigThreads) {
            const int r = e / kN, c = e % kN;
            if ((c >> 7) < (r >> 7)) Gw[e] = __ldcg(Gw + (size_t)c * kN + r);
        }
    }
    __syncthreads();

    // Q0: fp32 columns in Qt and bf16 hi / lo rows in shared memory (thread = row)
    {
        const int r = tid;
        uint16_t *row = reinterpret_cast<uint16_t *>(sm.buf + r * kQPitch);
        for (int c = 0; c < kP; ++c) {
            const float v = start_entry(r, c);
            Qt[(size_t)c * kN + r] = v;
            const uint16_t h = float_to_bf16_bits(v);
            row[c] = h;
            row[kP + c] = float_to_bf16_bits(v - bf16_bits_to_float(h));
        }
    }
    if (tid == 0) { sm.done = 0; sm.prev_change = 1.f; }
    __syncthreads();

    bool converged = false, jacobi_ok = true, have_prev = false;
    int sweeps = 0;
    for (int it = 1; it <= p.max_iter; ++it) {
        eig_gemm(Gu, sm.buf, Yt);                       // Y = G Q
        __syncthreads();
        const bool rr = it == 1 || (it % 3) == 0 || it == p.max_iter;   // measured: every third beats every second
        const float *zsrc;
        if (rr) {
            small_gram(Qt, Yt, wk.A, wk);            // H = Q^T Y
            for (int e = tid; e < kP * kP; e += kEigThreads) {
                const int i = e / kP, j = e % kP;
                if (i < j) {
                    const float v = 0.5f * (wk.A[e] + wk.A[j * kP + i]);
                    wk.A[e] = v;
                    wk.A[j * kP + i] = v;
                }
            }
            __syncthreads();
            sweeps = jacobi96(wk.A, wk.V, sm);
            if (sweeps < 0) jacobi_ok = false;
            __syncthreads();
            if (tid < kP) {                              // sort the Ritz values, descending
                const float v = wk.A[tid * kP + tid];
                int rk = 0;
                for (int c = 0; c < kP; ++c) {
                    const float u = wk.A[c * kP + c];
                    rk += (u > v || (u == v && c < tid)) ? 1 : 0;
                }
                sm.inv[rk] = tid;
                sm.theta[rk] = v;
            }
            __syncthreads();
            if (tid == 0) {
                // largest relative change of sigma = sqrt(theta) among the leading 64 since the
                // previous Rayleigh-Ritz step (components below kThetaFloor of the largest are
                // numerically zero and left out); with the ratio of successive changes as the
                // contraction rate rho, the remaining error is about change * rho / (1 - rho)
                float worst = 0.f;
                const float floor_t = kThetaFloor * sm.theta[0];
                for (int i = 0; i < kR; ++i) {
                    if (sm.theta[i] <= floor_t) continue;
                    const float a = sqrtf(sm.theta[i]), b = sqrtf(fmaxf(sm.prev[i], 0.f));
                    worst = fmaxf(worst, fabsf(a - b) / a);
                }
                const float rho = fminf(worst / fmaxf(sm.prev_change, 1e-30f), 0.95f);
                const float est = worst * rho / (1.f - rho);
                sm.done = (have_prev && est < kConvTol && worst < kConvTol) ? 1 : 0;
                sm.prev_change = worst;
                float *inf = p.ws.info + (size_t)unit * 4;
                inf[0] = (float)it; inf[1] = (float)sweeps; inf[2] = worst; inf[3] = est;
            }
            __syncthreads();
            if (tid < kP) sm.prev[tid] = sm.theta[tid];
            have_prev = true;
            converged = sm.done != 0;
            const bool last = converged || it == p.max_iter;
            const float floor_t = kThetaFloor * fmaxf(sm.theta[0], 0.f);
            // M = V (sorted columns), scaled by 1 / theta for Z; plain for the final Ritz vectors
            for (int e = tid; e < kP * kP; e += kEigThreads) {
                const int i = e / kP, j = e % kP;
                const float th = sm.theta[j];
                const float v = wk.V[i * kP + sm.inv[j]];
                wk.M[e] = last ? v : (th > floor_t ? v / th : 0.f);
            }
            __syncthreads();
            if (last) {
                // Ritz vectors U = Q V: basis B = U_r^T (bf16) and Q_r for the projection
                rowmix(Qt, wk.M, nullptr, Qgu, p.B + (size_t)unit * kR * kN);
                if (p.sigma != nullptr && tid < kR) p.sigma[(size_t)unit * kR + tid] = sqrtf(fmaxf(sm.theta[tid], 0.f));
                break;
            }
            rowmix(Yt, wk.M, Zt, nullptr, nullptr);     // Z = Y V Theta^-1
            if (tid < kP) sm.scale[tid] = 1.f;
            zsrc = Zt;
        } else {
            // Rayleigh quotients d_j = q_j . y_j; Z = Y D^-1
            for (int c = warp; c < kP; c += kEigWarps) {
                float s = 0.f;
                for (int j = lane; j < kN; j += 32) s = fmaf(__ldcg(Qt + (size_t)c * kN + j), __ldcg(Yt + (size_t)c * kN + j), s);
                #pragma unroll
                for (int d = 16; d > 0; d >>= 1) s += __shfl_xor_sync(0xffffffffu, s, d);
                if (lane == 0) sm.scale[c] = s;
            }
            __syncthreads();
            if (tid < kP) {
                const float d = sm.scale[tid];
                sm.scale[tid] = d > kThetaFloor * sm.prev[0] ? 1.f / d : 0.f;
            }
            zsrc = Yt;
        }
        __syncthreads();
        // Cholesky QR of Z = zsrc * diag(scale): W = S^T (zsrc^T zsrc) S = R^T R, Q = zsrc S R^-1
        small_gram(zsrc, zsrc, wk.A, wk);
        for (int e = tid; e < kP * kP; e += kEigThreads) wk.A[e] *= sm.scale[e / kP] * sm.scale[e % kP];
        __syncthreads();
        cholesky96(wk.A, wk.V, sm);
        tri_inverse96(wk.V, wk.M, wk.A);
        for (int e = tid; e < kP * kP; e += kEigThreads) wk.M[e] *= sm.scale[e / kP];
        __syncthreads();
        rowmix(zsrc, wk.M, Qt, Qgu, nullptr);
        __syncthreads();
        // Q (bf16 hi / lo rows) into shared memory for the next product
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
//     G (the eigen-solver fills the lower triangle from it).
// When the units alone leave SMs idle, the bands' token ranges are split (more
// splits for the wider bands, equal work per block, one wave of blocks) and the
// splits add into a zeroed G with fp32 atomics.
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

// Token splits of the four bands (band I has 4 - I column blocks of work per token): while a further
// split of every unit still fits one wave of blocks, split the band whose blocks are the longest
// (at least 16 chunks of 64 tokens per split)
inline void gram_tc_splits(int units, int T, int sms, int (&sp)[4]) {
    for (int I = 0; I < 4; ++I) sp[I] = 1;
    const int nch = (T + kGtTok - 1) / kGtTok;
    while (true) {
        int total = 0, best = -1;
        for (int I = 0; I < 4; ++I) total += sp[I];
        if ((long long)units * (total + 1) > sms) break;
        for (int I = 0; I < 4; ++I)
            if (nch >= 16 * (sp[I] + 1) &&
                (best < 0 || (4 - I) * sp[best] > (4 - best) * sp[I])) best = I;
        if (best < 0) break;
        ++sp[best];
    }
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
    Workspace w = carve(ws, units);
    GramTcParams gp;
    gp.tm_x = tm_x;
    gp.G = w.G;
    gp.T = T;
    gp.units = units;
    gram_tc_splits(units, T, sms, gp.splits);
    gp.atomic = (gp.splits[0] > 1 || gp.splits[1] > 1 || gp.splits[2] > 1 || gp.splits[3] > 1) ? 1 : 0;
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
