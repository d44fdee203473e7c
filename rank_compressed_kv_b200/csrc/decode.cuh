// decode.cuh -- one AttentionPack decode step over the rank-compressed visual
// cache plus the uncompressed text tail.
//
// Method ("Attention-aware Inference Optimizations for Large Vision-Language
// Models with Memory-efficient Decoding", technical summaries 2.B, fr/es/de
// pages): tokens whose importance is high are decompressed at the full rank,
// the others at a quarter of it.  Decompression is folded into the attention
// by associativity: the query goes to rank space once (q~ = B_K[:, slice] q),
// a token's logit is C_K[t, :rho_t] . q~[:rho_t], the softmax-weighted V
// coefficients are summed in rank space and projected back through B_V once
// per head.  K and V are never materialised.
//
// Four launches, each streaming its own bytes once:
//   qproj_kernel   q~ = scale * log2(e) * B_K[:, 128 j(h) ..] q_h per unit, split into bf16 hi + lo
//   text_kernel    the text tail (plain bf16 K/V) per (unit, KV head, chunk of tokens):
//                  partial (max, sum, w = sum p V) per query head
//   vis_kernel     the compressed visual tokens per (unit, split of tokens): partial
//                  (max, sum, u = sum p C_V) per query head, then -- once every split
//                  of the unit has published -- the attention mass of each token
//   finish_kernel  combines the partials of a unit and projects: o_h = (u B_V + w) / l
// Logits are kept in the log2 domain (the scale folds log2(e)).
#pragma once

#include <cuda.h>

#include "common.cuh"

namespace kvpack {
namespace decode {

constexpr int kMaxHeads = 32;
constexpr int kTxtPart = 130;   // per (unit, text chunk, head): max, sum, w[128]
constexpr int kVisPart = 66;    // per (unit, visual split, head): max, sum, u[64]

// ======================================================================== qproj

struct QProjParams {
    const uint16_t *q;     // [(layer, batch)][n_q][128]
    const uint16_t *BK;    // [units][64][512]
    uint16_t *qt;          // [units][2][Hg][64]: hi then lo, 128-byte rows, 16-byte chunk c stored at c ^ (h & 7)
    int Hg, per_kv, n_q, groups;
    float scale2;
};

// One block per unit.  Warp w takes rank rows 8w..8w+7 of B_K; lane L holds
// columns 8L..8L+7 and 256+8L..256+8L+7 of a row, so a 16-lane half covers one
// KV head's 128 columns and a shuffle tree finishes each dot product.
__global__ void __launch_bounds__(256) qproj_kernel(const QProjParams p) {
    __shared__ float qs[kMaxHeads][128];
    const int unit = blockIdx.x, warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int lb = unit / p.groups, G = unit % p.groups;
    const uint16_t *qsrc = p.q + ((size_t)lb * p.n_q + (size_t)G * p.Hg) * 128;
    for (int i = threadIdx.x; i < p.Hg * 128; i += 256) qs[i >> 7][i & 127] = bf16_bits_to_float(qsrc[i]);

    uint4 raw[8][2];
    const uint16_t *bk = p.BK + (size_t)unit * 64 * 512;
    #pragma unroll
    for (int r = 0; r < 8; ++r)
        #pragma unroll
        for (int sg = 0; sg < 2; ++sg)
            raw[r][sg] = __ldcs(reinterpret_cast<const uint4 *>(bk + (size_t)(8 * warp + r) * 512 + 256 * sg + 8 * lane));
    __syncthreads();

    uint16_t *qt = p.qt + (size_t)unit * 2 * p.Hg * 64;
    #pragma unroll
    for (int r = 0; r < 8; ++r) {
        const int i = 8 * warp + r;
        #pragma unroll
        for (int sg = 0; sg < 2; ++sg) {
            const int j = 2 * sg + (lane >> 4), dd = 8 * (lane & 15);
            const uint32_t w4[4] = {raw[r][sg].x, raw[r][sg].y, raw[r][sg].z, raw[r][sg].w};
            float b[8];
            #pragma unroll
            for (int e = 0; e < 4; ++e) {
                b[2 * e] = __uint_as_float(w4[e] << 16);
                b[2 * e + 1] = __uint_as_float(w4[e] & 0xffff0000u);
            }
            for (int hh = 0; hh < p.per_kv; ++hh) {
                const int h = j * p.per_kv + hh;
                const float *qr = &qs[h][dd];
                float acc = 0.f;
                #pragma unroll
                for (int e = 0; e < 8; ++e) acc = fmaf(b[e], qr[e], acc);
                #pragma unroll
                for (int d = 1; d < 16; d <<= 1) acc += __shfl_xor_sync(0xffffffffu, acc, d);
                if ((lane & 15) == 0) {
                    const float v = acc * p.scale2;
                    const uint16_t hi = float_to_bf16_bits(v);
                    const uint16_t lo = float_to_bf16_bits(v - bf16_bits_to_float(hi));
                    const int off = h * 64 + ((((i >> 3) ^ (h & 7)) & 7) << 3) + (i & 7);
                    qt[off] = hi;
                    qt[p.Hg * 64 + off] = lo;
                }
            }
        }
    }
}

// ========================================================================= text

namespace text {

constexpr int kWarps = 8;
constexpr int kThreads = kWarps * 32;
constexpr int kSlots = 3;
constexpr int kSlotBytes = 8192;   // 16 tokens x (K 256 B + V 256 B) of one KV head
constexpr int kTile = 16;

struct Params {
    CUtensorMap tm_k, tm_v;    // 4D {128, 4, L, units}, box {64, 1, 16, 1}, 128-byte swizzle
    const uint16_t *q;
    float *part;               // [units][Sc][Hg][kTxtPart]
    unsigned int *counter;     // work counter, zero at launch
    int n_units, L, Hg, per_kv, n_q, groups, Sc, ct, n_items;
    float scale2;
};

struct Smem {
    alignas(1024) unsigned char ring[kWarps][kSlots][kSlotBytes];
    uint64_t full[kWarps][kSlots];
    int itemq[kWarps][8];
    int abort;
};

constexpr size_t smem_bytes() { return sizeof(Smem) + 1024; }

// Every warp streams whole work items -- (unit, KV head j, chunk of ct text
// tokens) -- through its own 3-slot ring, fetched from a global counter.  Per
// 16-token tile: S = K q^T with tokens on M and the KV head's query heads on N
// (mma.sync m16n8k16), an online softmax over the columns, and w^T += V^T P
// (the transposed P comes from movmatrix).  At the end of an item the warp
// writes the partial (max, sum, w) of each of its query heads.
__global__ void __launch_bounds__(kThreads, 1) text_kernel(const __grid_constant__ Params p) {
    extern __shared__ __align__(1024) unsigned char smem_raw[];
    const uint32_t base = smem_u32(smem_raw);
    Smem &sm = *reinterpret_cast<Smem *>(smem_raw + ((1024u - (base & 1023u)) & 1023u));
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int g = lane >> 2, tig = lane & 3;
    if (threadIdx.x == 0) {
        for (int w = 0; w < kWarps; ++w)
            for (int s = 0; s < kSlots; ++s) mbar_init(&sm.full[w][s], 1);
        sm.abort = 0;
        asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
    }
    __syncthreads();
    volatile int *abort = &sm.abort;

    auto fetch = [&]() -> int {
        int v = 0;
        if (lane == 0) v = (int)atomicAdd(p.counter, 1u);
        return __shfl_sync(0xffffffffu, v, 0);
    };
    auto n_tok = [&](int it) { const int c = it % p.Sc; return min(p.ct, p.L - c * p.ct); };

    // ---- issue side
    int i_item = -1, i_tile = 0, i_ntiles = 0, q_push = 0;
    bool i_done = false;
    uint32_t i_seq = 0, c_seq = 0;
    auto issue = [&]() {
        if (i_done) return;
        if (i_tile == i_ntiles) {
            const int it = fetch();
            if (it >= p.n_items) { i_done = true; return; }
            i_item = it; i_tile = 0; i_ntiles = (n_tok(it) + kTile - 1) / kTile;
            if (lane == 0) sm.itemq[warp][q_push & 7] = it;
            ++q_push;
        }
        const int slot = i_seq % kSlots;
        const int unit = i_item / (4 * p.Sc), j = (i_item / p.Sc) % 4, c = i_item % p.Sc;
        const int tok = c * p.ct + i_tile * kTile;
        __syncwarp();
        if (lane == 0) {
            unsigned char *dst = sm.ring[warp][slot];
            uint64_t *bar = &sm.full[warp][slot];
            fence_proxy_async();
            mbar_arrive_tx(bar, kSlotBytes);
            tma_4d(dst, &p.tm_k, 0, j, tok, unit, bar);
            tma_4d(dst + 2048, &p.tm_k, 64, j, tok, unit, bar);
            tma_4d(dst + 4096, &p.tm_v, 0, j, tok, unit, bar);
            tma_4d(dst + 6144, &p.tm_v, 64, j, tok, unit, bar);
        }
        ++i_tile;
        ++i_seq;
    };

    // query rows of (unit, j) as B fragments: b0 = q[g][16 kb + 2 tig ..], b1 = q[g][16 kb + 8 + 2 tig ..]
    auto load_q = [&](int it, uint32_t (&qf)[8][2]) {
        const int unit = it / (4 * p.Sc), j = (it / p.Sc) % 4;
        const int lb = unit / p.groups, G = unit % p.groups;
        const bool ok = g < p.per_kv;
        const uint32_t *row = reinterpret_cast<const uint32_t *>(
            p.q + ((size_t)lb * p.n_q + (size_t)G * p.Hg + j * p.per_kv + (ok ? g : 0)) * 128);
        #pragma unroll
        for (int kb = 0; kb < 8; ++kb) {
            qf[kb][0] = ok ? __ldg(row + 8 * kb + tig) : 0u;
            qf[kb][1] = ok ? __ldg(row + 8 * kb + 4 + tig) : 0u;
        }
    };

    for (int s = 0; s < kSlots; ++s) issue();

    uint32_t qf[8][2], qn[8][2];
    int qn_item = -1, q_pop = 0;
    int c_item = -1, c_tile = 0, c_ntiles = 0, c_n = 0;
    float m[2], l[2], wt[8][4];

    while (c_seq < i_seq) {
        if (c_tile == c_ntiles) {
            c_item = sm.itemq[warp][q_pop & 7];
            ++q_pop;
            c_tile = 0;
            c_n = n_tok(c_item);
            c_ntiles = (c_n + kTile - 1) / kTile;
            if (qn_item == c_item) {
                #pragma unroll
                for (int kb = 0; kb < 8; ++kb) { qf[kb][0] = qn[kb][0]; qf[kb][1] = qn[kb][1]; }
            } else {
                load_q(c_item, qf);
            }
            m[0] = m[1] = -INFINITY;
            l[0] = l[1] = 0.f;
            #pragma unroll
            for (int a = 0; a < 8; ++a) wt[a][0] = wt[a][1] = wt[a][2] = wt[a][3] = 0.f;
        }
        // prefetch the next item's query rows once the issue side has fetched it
        if (q_pop < q_push && qn_item != sm.itemq[warp][q_pop & 7]) {
            qn_item = sm.itemq[warp][q_pop & 7];
            load_q(qn_item, qn);
        }
        const int slot = c_seq % kSlots;
        if (!mbar_wait(&sm.full[warp][slot], (c_seq / kSlots) & 1u, abort)) break;
        const uint32_t sb = smem_u32(sm.ring[warp][slot]);
        const int n = min(kTile, c_n - c_tile * kTile);

        // S[tok][h] = K[tok][:] . q_h
        float s[4] = {0.f, 0.f, 0.f, 0.f};
        #pragma unroll
        for (int kb = 0; kb < 8; ++kb) {
            uint32_t a[4];
            const int row = (lane & 7) + (((lane >> 3) & 1) << 3);
            const int ch = 2 * (kb & 3) + (lane >> 4);
            ldsm_x4(sb + (kb >> 2) * 2048 + row * 128 + ((ch ^ (row & 7)) << 4), a[0], a[1], a[2], a[3]);
            mma_bf16(s, a, qf[kb][0], qf[kb][1]);
        }
        const bool v0 = g < n, v1 = g + 8 < n;
        s[0] = v0 ? s[0] * p.scale2 : -INFINITY;
        s[1] = v0 ? s[1] * p.scale2 : -INFINITY;
        s[2] = v1 ? s[2] * p.scale2 : -INFINITY;
        s[3] = v1 ? s[3] * p.scale2 : -INFINITY;
        float mx0 = fmaxf(s[0], s[2]), mx1 = fmaxf(s[1], s[3]);
        #pragma unroll
        for (int d = 4; d < 32; d <<= 1) {
            mx0 = fmaxf(mx0, __shfl_xor_sync(0xffffffffu, mx0, d));
            mx1 = fmaxf(mx1, __shfl_xor_sync(0xffffffffu, mx1, d));
        }
        const float mn0 = fmaxf(m[0], mx0), mn1 = fmaxf(m[1], mx1);   // finite: the tile has a valid token
        const float a0 = ex2(m[0] - mn0), a1 = ex2(m[1] - mn1);
        const float p0 = ex2(s[0] - mn0), p1 = ex2(s[1] - mn1), p2 = ex2(s[2] - mn0), p3 = ex2(s[3] - mn1);
        l[0] = l[0] * a0 + (p0 + p2);
        l[1] = l[1] * a1 + (p1 + p3);
        m[0] = mn0;
        m[1] = mn1;
        #pragma unroll
        for (int mt = 0; mt < 8; ++mt) {
            wt[mt][0] *= a0; wt[mt][1] *= a1; wt[mt][2] *= a0; wt[mt][3] *= a1;
        }
        const uint32_t b0 = movmatrix_t(pack_bf16(p0, p1));
        const uint32_t b1 = movmatrix_t(pack_bf16(p2, p3));
        // w^T[d][h] += V^T[d][tok] P[tok][h]
        #pragma unroll
        for (int mt = 0; mt < 8; ++mt) {
            uint32_t a[4];
            const int mi = lane >> 3;
            const int tok = (lane & 7) + ((mi >> 1) << 3);
            const int ch = 2 * (mt & 3) + (mi & 1);
            ldsm_x4_t(sb + 4096 + (mt >> 2) * 2048 + tok * 128 + ((ch ^ (tok & 7)) << 4), a[0], a[1], a[2], a[3]);
            mma_bf16(wt[mt], a, b0, b1);
        }
        ++c_tile;
        ++c_seq;

        if (c_tile == c_ntiles) {
            // partial of this item: per head h = 2 tig + e of KV head j
            #pragma unroll
            for (int e = 0; e < 2; ++e)
                #pragma unroll
                for (int d = 4; d < 32; d <<= 1) l[e] += __shfl_xor_sync(0xffffffffu, l[e], d);
            const int unit = c_item / (4 * p.Sc), j = (c_item / p.Sc) % 4, c = c_item % p.Sc;
            float *dst = p.part + (((size_t)unit * p.Sc + c) * p.Hg + j * p.per_kv) * kTxtPart;
            #pragma unroll
            for (int e = 0; e < 2; ++e) {
                const int hh = 2 * tig + e;
                if (hh < p.per_kv) {
                    float *row = dst + hh * kTxtPart;
                    if (g == 0) { row[0] = m[e]; row[1] = l[e]; }
                    #pragma unroll
                    for (int mt = 0; mt < 8; ++mt) {
                        row[2 + 16 * mt + g] = wt[mt][e];
                        row[2 + 16 * mt + g + 8] = wt[mt][2 + e];
                    }
                }
            }
        }
        __syncwarp();
        if (i_seq - c_seq < (uint32_t)kSlots) issue();
    }
    // copies still in flight (only after an abort) must land before the block exits
    while (c_seq < i_seq) {
        const int slot = c_seq % kSlots;
        const uint32_t par = (c_seq / kSlots) & 1u;
        const long long t0 = clock64();
        while (!mbar_try_wait(&sm.full[warp][slot], par) && clock64() - t0 < kWaitCycles) {}
        ++c_seq;
    }
}

}  // namespace text

// ======================================================================== visual

namespace vis {

constexpr int kWarps = 8;
constexpr int kThreads = kWarps * 32;
constexpr int kSlots = 3;
constexpr int kSlotBytes = 8192;
constexpr int kHiTok = 32;          // full-rank tokens per HI stage
constexpr int kMeta = 4;            // item metadata ring (the issue side runs up to two items ahead)

template <int NMB>
struct Cfg {
    static constexpr int kRows = 16 * NMB;                 // query-head rows (padded)
    static constexpr int kLoTok = (NMB == 1) ? 128 : 64;   // visual tokens per warp per item
    static constexpr int kItemTok = kWarps * kLoTok;       // 1024 / 512 tokens per item
    static constexpr int kHiMax = kLoTok / kHiTok;         // HI stages per warp per item, at most
    static constexpr int kUpd = kLoTok / 64 + kHiMax;      // softmax updates per warp per item, at most
};

struct Params {
    CUtensorMap tm_ck, tm_cv;   // C_lo planes: 3D {16, T, units}, box {16, 32, 1}, 32-byte swizzle
    const uint16_t *CK_lo, *CK_hi, *CV_lo, *CV_hi;
    const uint16_t *qt;         // [units][2][Hg][64] from qproj_kernel
    const uint32_t *mask;       // [units][nwords]
    float *mass;                // [units][T] or null
    float *part;                // [units][S][Hg][kVisPart]
    const float *tpart;         // [units][Sc][Hg][kTxtPart] (max and sum read) or null
    unsigned int *arrive;       // [units], zero at launch
    int n_units, T, Hg, S, tps, nwords, Sc, n_items;
};

template <int NMB>
struct Smem {
    using C = Cfg<NMB>;
    alignas(1024) unsigned char ring[kWarps][kSlots][kSlotBytes];
    alignas(128) uint16_t qt[2][C::kRows][64];              // q~ hi / lo of the current item
    float u_acc[C::kRows][64];                               // block-wide u of the item
    float wm[kWarps][C::kRows], wl[kWarps][C::kRows];
    float mcta[C::kRows], lcta[C::kRows], mfin[C::kRows], invl[C::kRows];
    float mref[2][kWarps][C::kUpd][C::kRows];               // running max at each stashed update
    uint16_t hi_list[kMeta][kWarps][C::kLoTok];             // this warp's full-rank tokens (item-relative)
    int meta[kMeta][kWarps][8];                             // lo0, n_lo, n_hi, item, 4 mask words of the LO range
    uint64_t full[kWarps][kSlots];
    uint64_t qbar;
    uint32_t tmem_base;
    int abort;
};

template <int NMB>
constexpr size_t smem_bytes() { return sizeof(Smem<NMB>) + 1024; }

// One online-softmax update of row r over NT m16n8 score tiles; returns the
// new running max.  p overwrites s.
template <int NT>
__device__ __forceinline__ float softmax_row(float (&s)[NT][4], int r, float &m, float &l, float (&u)[8][4]) {
    float mx = -INFINITY;
    #pragma unroll
    for (int nt = 0; nt < NT; ++nt) mx = fmaxf(mx, fmaxf(s[nt][2 * r], s[nt][2 * r + 1]));
    mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, 1));
    mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, 2));
    const float mn = fmaxf(m, mx);
    const bool live = mn != -INFINITY;
    const float alpha = live ? ex2(m - mn) : 1.f;
    float sum = 0.f;
    #pragma unroll
    for (int nt = 0; nt < NT; ++nt) {
        const float x0 = live ? ex2(s[nt][2 * r] - mn) : 0.f;
        const float x1 = live ? ex2(s[nt][2 * r + 1] - mn) : 0.f;
        s[nt][2 * r] = x0;
        s[nt][2 * r + 1] = x1;
        sum += x0 + x1;
    }
    l = l * alpha + sum;
    m = mn;
    #pragma unroll
    for (int nt = 0; nt < 8; ++nt) {
        u[nt][2 * r] *= alpha;
        u[nt][2 * r + 1] *= alpha;
    }
    return mn;
}

// Sum over the 8 lanes that share lane & 3 of 16 per-lane values, scattered:
// afterwards the lane holds the totals of slots 8 b4 + 4 b3 + 2 b2 + {0, 1}
// (b = bits 4, 3, 2 of the lane).
__device__ __forceinline__ void reduce_scatter16(const float (&x)[16], float (&out)[2], int lane) {
    float t8[8], t4[4];
    const bool b4 = lane & 16, b3 = lane & 8, b2 = lane & 4;
    #pragma unroll
    for (int i = 0; i < 8; ++i) {
        const float send = b4 ? x[i] : x[8 + i];
        t8[i] = (b4 ? x[8 + i] : x[i]) + __shfl_xor_sync(0xffffffffu, send, 16);
    }
    #pragma unroll
    for (int i = 0; i < 4; ++i) {
        const float send = b3 ? t8[i] : t8[4 + i];
        t4[i] = (b3 ? t8[4 + i] : t8[i]) + __shfl_xor_sync(0xffffffffu, send, 8);
    }
    #pragma unroll
    for (int i = 0; i < 2; ++i) {
        const float send = b2 ? t4[i] : t4[2 + i];
        out[i] = (b2 ? t4[2 + i] : t4[i]) + __shfl_xor_sync(0xffffffffu, send, 4);
    }
}

// 8 values -> the lane holds the total of slot 4 b4 + 2 b3 + b2
__device__ __forceinline__ float reduce_scatter8(const float (&x)[8], int lane) {
    float t4[4], t2[2];
    const bool b4 = lane & 16, b3 = lane & 8, b2 = lane & 4;
    #pragma unroll
    for (int i = 0; i < 4; ++i) {
        const float send = b4 ? x[i] : x[4 + i];
        t4[i] = (b4 ? x[4 + i] : x[i]) + __shfl_xor_sync(0xffffffffu, send, 16);
    }
    #pragma unroll
    for (int i = 0; i < 2; ++i) {
        const float send = b3 ? t4[i] : t4[2 + i];
        t2[i] = (b3 ? t4[2 + i] : t4[i]) + __shfl_xor_sync(0xffffffffu, send, 8);
    }
    const float send = b2 ? t2[0] : t2[1];
    return (b2 ? t2[1] : t2[0]) + __shfl_xor_sync(0xffffffffu, send, 4);
}

// Persistent, one 256-thread block per SM, a static round-robin over items
// (unit, split).  Each warp streams its own share of the item -- a contiguous
// range of C_lo rows (TMA) and an equal share of the item's full-rank tokens
// (C_lo + C_hi rows gathered with cp.async) -- through a private 3-slot ring,
// with heads on M and tokens on N of mma.sync m16n8k16:
//   scores  s = q~ C_K^T  (q~ as a bf16 hi + lo pair, C_K exact in bf16)
//   softmax online per head row; P stays in registers as the A operand of
//   values  u += P C_V    (rank 16 over the LO range, rank 64 for HI tokens;
//                          a token with its mask bit set gets logit -inf in LO)
// Each softmax update also stores its p (fp32) to tensor memory together with
// the running max it was taken against.  At the item's end the warps merge
// (max, sum, u) and publish the split's partial; the attention mass of the
// item is written one item later, when every split of the unit (and the text
// partials) fix the unit's max and sum: mass_t = sum_h p_ht 2^(m_ref - M_h) / L_h.
template <int NMB>
__global__ void __launch_bounds__(kThreads, 1) vis_kernel(const __grid_constant__ Params p) {
    using C = Cfg<NMB>;
    extern __shared__ __align__(1024) unsigned char smem_raw[];
    const uint32_t sbase0 = smem_u32(smem_raw);
    Smem<NMB> &sm = *reinterpret_cast<Smem<NMB> *>(smem_raw + ((1024u - (sbase0 & 1023u)) & 1023u));
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31, tid = threadIdx.x;
    const int g = lane >> 2, tig = lane & 3;
    volatile int *abort = &sm.abort;

    if (tid == 0) {
        for (int w = 0; w < kWarps; ++w)
            for (int s = 0; s < kSlots; ++s) mbar_init(&sm.full[w][s], 32);
        mbar_init(&sm.qbar, 1);
        sm.abort = 0;
        asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
    }
    for (int i = tid; i < 2 * C::kRows * 64; i += kThreads) (&sm.qt[0][0][0])[i] = 0;
    for (int i = tid; i < C::kRows * 64; i += kThreads) (&sm.u_acc[0][0])[i] = 0.f;
    if (warp == 0) tmem_alloc(&sm.tmem_base, 512);
    tmem_fence_before();
    __syncthreads();
    tmem_fence_after();
    const uint32_t tmem = sm.tmem_base + ((uint32_t)(32 * (warp & 3)) << 16) + 256u * (uint32_t)(warp >> 2);

    auto item_of = [&](int K) { return (int)blockIdx.x + K * (int)gridDim.x; };
    auto issue_q = [&](int K) {   // q~ of item K into sm.qt (one thread)
        const int unit = item_of(K) / p.S;
        const uint32_t bytes = (uint32_t)p.Hg * 128u;
        fence_proxy_async();
        mbar_arrive_tx(&sm.qbar, 2 * bytes);
        bulk_g2s(&sm.qt[0][0][0], p.qt + (size_t)unit * 2 * p.Hg * 64, bytes, &sm.qbar);
        bulk_g2s(&sm.qt[1][0][0], p.qt + (size_t)unit * 2 * p.Hg * 64 + (size_t)p.Hg * 64, bytes, &sm.qbar);
    };
    if (tid == 0) issue_q(0);

    // ------------------------------------------------------------ issue side
    auto load_words = [&](int K) -> uint32_t {   // lane i: mask word i of item K
        const int item = item_of(K);
        if (item >= p.n_items) return 0u;
        const int unit = item / p.S, t0 = (item % p.S) * p.tps;
        const int n = min(p.T, t0 + p.tps) - t0;
        const int nw = (n + 31) >> 5;
        if (lane >= nw) return 0u;
        uint32_t v = __ldg(p.mask + (size_t)unit * p.nwords + (t0 >> 5) + lane);
        if (lane == nw - 1 && (n & 31)) v &= (1u << (n & 31)) - 1u;
        return v;
    };
    int iK = 0, i_st = 0, i_nst = 0;
    bool i_done = false;
    uint32_t i_seq = 0, c_seq = 0;
    int Kc = 0;                          // item the consumer is on
    uint32_t mw = load_words(0), mw_nx = load_words(1);

    // metadata of item K for this warp (meta slot K % kMeta); false if there is no item K
    auto begin_item = [&](int K) -> bool {
        const int item = item_of(K);
        if (item >= p.n_items) return false;
        const int t0 = (item % p.S) * p.tps;
        const int n = min(p.T, t0 + p.tps) - t0;
        int wt = (n + kWarps - 1) / kWarps;
        wt = (wt + 31) & ~31;
        const int lo0 = warp * wt;
        int n_lo = max(0, min(wt, n - lo0));
        const int wl0 = lo0 >> 5;
        if (n_lo > 0) {
            // the LO range is skipped when every token in it is full-rank
            const int wln = (n_lo + 31) >> 5;
            const bool in = lane >= wl0 && lane < wl0 + wln;
            uint32_t need = 0xffffffffu;
            if (in && lane == wl0 + wln - 1 && (n_lo & 31)) need = (1u << (n_lo & 31)) - 1u;
            if (__all_sync(0xffffffffu, !in || (mw & need) == need)) n_lo = 0;
        }
        const int cnt = __popc(mw);
        int incl = cnt;
        #pragma unroll
        for (int d = 1; d < 32; d <<= 1) {
            const int v = __shfl_up_sync(0xffffffffu, incl, d);
            if (lane >= d) incl += v;
        }
        const int n_hi = __shfl_sync(0xffffffffu, incl, 31);
        const int h0 = (warp * n_hi) / kWarps, h1 = ((warp + 1) * n_hi) / kWarps;
        const int ms = K % kMeta;
        int gi = incl - cnt;
        uint32_t bits = mw;
        while (bits) {
            const int b = __ffs(bits) - 1;
            if (gi >= h0 && gi < h1) sm.hi_list[ms][warp][gi - h0] = (uint16_t)(32 * lane + b);
            ++gi;
            bits &= bits - 1u;
        }
        if (lane >= wl0 && lane < wl0 + 4) sm.meta[ms][warp][4 + lane - wl0] = (int)mw;
        if (lane == 0) {
            sm.meta[ms][warp][0] = lo0;
            sm.meta[ms][warp][1] = n_lo;
            sm.meta[ms][warp][2] = h1 - h0;
            sm.meta[ms][warp][3] = item;
        }
        __syncwarp();
        i_nst = (n_lo > 0 ? 1 : 0) + (h1 - h0 + kHiTok - 1) / kHiTok;
        i_st = 0;
        return true;
    };

    auto issue_stage = [&]() {
        const int ms = iK % kMeta;
        const int lo0 = sm.meta[ms][warp][0], n_lo = sm.meta[ms][warp][1], nh = sm.meta[ms][warp][2];
        const int item = sm.meta[ms][warp][3];
        const int unit = item / p.S, t0 = (item % p.S) * p.tps;
        const int slot = i_seq % kSlots;
        unsigned char *dst = sm.ring[warp][slot];
        uint64_t *bar = &sm.full[warp][slot];
        __syncwarp();
        if (i_st == 0 && n_lo > 0) {
            // whole 64-row halves: the value MMA reads every row of a half (masked rows get p = 0,
            // which must meet finite data -- neighbouring rows, or zeros past the unit's end)
            const int nb = 2 * ((n_lo + 63) >> 6);
            if (lane == 0) {
                fence_proxy_async();
                mbar_arrive_tx(bar, (uint32_t)nb * 2048u);
                for (int b = 0; b < nb; ++b) {
                    tma_3d(dst + 1024 * b, &p.tm_ck, 0, t0 + lo0 + 32 * b, unit, bar);
                    tma_3d(dst + 4096 + 1024 * b, &p.tm_cv, 0, t0 + lo0 + 32 * b, unit, bar);
                }
            } else {
                mbar_arrive(bar);
            }
        } else {
            const int hs = i_st - (n_lo > 0 ? 1 : 0);
            const int cnt = min(kHiTok, nh - kHiTok * hs);
            const size_t ubase = (size_t)unit * p.T + t0;
            #pragma unroll
            for (int i = 0; i < 8; ++i) {
                const int idx = lane + 32 * i;
                const int r = idx >> 3, ch = idx & 7;
                const int pos = (ch ^ (r & 7)) << 4;
                unsigned char *dk = dst + r * 128 + pos;
                unsigned char *dv = dst + 4096 + r * 128 + pos;
                if (r < cnt) {
                    const size_t row = ubase + sm.hi_list[ms][warp][kHiTok * hs + r];
                    if (ch < 2) {
                        cp_async16(dk, p.CK_lo + row * 16 + ch * 8);
                        cp_async16(dv, p.CV_lo + row * 16 + ch * 8);
                    } else {
                        cp_async16(dk, p.CK_hi + row * 48 + (ch - 2) * 8);
                        cp_async16(dv, p.CV_hi + row * 48 + (ch - 2) * 8);
                    }
                } else {
                    *reinterpret_cast<uint4 *>(dk) = make_uint4(0u, 0u, 0u, 0u);
                    *reinterpret_cast<uint4 *>(dv) = make_uint4(0u, 0u, 0u, 0u);
                }
            }
            cp_async_arrive_noinc(bar);
        }
        ++i_st;
        ++i_seq;
    };

    // issue while the ring has room; the issue side may begin items up to Kc + 2
    auto pump = [&]() {
        while (!i_done && i_seq - c_seq < (uint32_t)kSlots) {
            if (i_st == i_nst) {
                if (iK + 1 > Kc + 2) return;
                ++iK;
                mw = mw_nx;
                mw_nx = load_words(iK + 1);
                if (!begin_item(iK)) { i_done = true; return; }
                continue;
            }
            issue_stage();
        }
    };
    if (!begin_item(0)) i_done = true;
    pump();

    // ---------------------------------------------------------- consumer side
    float m[NMB][2], l[NMB][2], u[NMB][8][4];
    uint32_t qah[NMB][4], qal[NMB][4];
    const uint32_t qt0 = smem_u32(&sm.qt[0][0][0]), qt1 = smem_u32(&sm.qt[1][0][0]);

    // deferred: attention mass of item K (meta slot K % kMeta, stash buffer K & 1); block-wide
    auto mass_of = [&](int K) {
        const int item = item_of(K);
        const int unit = item / p.S;
        if (tid == 0) {
            const long long start = clock64();
            while (!*abort) {
                unsigned int v;
                asm volatile("ld.acquire.gpu.global.u32 %0, [%1];" : "=r"(v) : "l"(&p.arrive[unit]) : "memory");
                if (v >= (unsigned int)p.S) break;
                if (clock64() - start > kWaitCycles) {
                    report_error(KVPACK_ERR_TIMEOUT);
                    *abort = 1;
                    break;
                }
                __nanosleep(64);
            }
        }
        __syncthreads();
        if (*abort) return;
        // unit-wide max and 1/sum per head from the visual and text partials
        for (int h = warp; h < p.Hg; h += kWarps) {
            const float *vp = p.part + (size_t)unit * p.S * p.Hg * kVisPart + (size_t)h * kVisPart;
            const float *tp = p.tpart + (size_t)unit * p.Sc * p.Hg * kTxtPart + (size_t)h * kTxtPart;
            float mx = -INFINITY;
            for (int s = lane; s < p.S; s += 32) mx = fmaxf(mx, __ldcg(vp + (size_t)s * p.Hg * kVisPart));
            for (int c = lane; c < p.Sc; c += 32) mx = fmaxf(mx, __ldcg(tp + (size_t)c * p.Hg * kTxtPart));
            #pragma unroll
            for (int d = 16; d > 0; d >>= 1) mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, d));
            float sum = 0.f;
            for (int s = lane; s < p.S; s += 32) {
                const float ms = __ldcg(vp + (size_t)s * p.Hg * kVisPart);
                if (ms != -INFINITY) sum += __ldcg(vp + (size_t)s * p.Hg * kVisPart + 1) * ex2(ms - mx);
            }
            for (int c = lane; c < p.Sc; c += 32) {
                const float ms = __ldcg(tp + (size_t)c * p.Hg * kTxtPart);
                if (ms != -INFINITY) sum += __ldcg(tp + (size_t)c * p.Hg * kTxtPart + 1) * ex2(ms - mx);
            }
            #pragma unroll
            for (int d = 16; d > 0; d >>= 1) sum += __shfl_xor_sync(0xffffffffu, sum, d);
            if (lane == 0) {
                sm.mfin[h] = mx;
                sm.invl[h] = 1.f / sum;
            }
        }
        __syncthreads();
        const int ms = K % kMeta, b = K & 1;
        const int lo0 = sm.meta[ms][warp][0], n_lo = sm.meta[ms][warp][1], nh = sm.meta[ms][warp][2];
        const int t0 = (item % p.S) * p.tps;
        float *mrow = p.mass + (size_t)unit * p.T + t0;
        auto fac = [&](int upd, int row) -> float {
            const float mr = sm.mref[b][warp][upd][row];
            return (row < p.Hg && mr != -INFINITY) ? ex2(mr - sm.mfin[row]) * sm.invl[row] : 0.f;
        };
        tmem_fence_after();
        // LO range, 64 tokens per pass
        for (int hf = 0; hf < C::kLoTok / 64; ++hf) {
            if (64 * hf >= n_lo) break;
            float acc[16];
            #pragma unroll
            for (int i = 0; i < 16; ++i) acc[i] = 0.f;
            #pragma unroll
            for (int mb = 0; mb < NMB; ++mb) {
                float v0[16], v1[16];
                const uint32_t col = (uint32_t)(128 * b + 32 * (NMB == 1 ? hf : mb));
                tmem_ld16(tmem + col, v0);
                tmem_ld16(tmem + col + 16, v1);
                tmem_wait_ld();
                const float f0 = fac(hf, 16 * mb + g), f1 = fac(hf, 16 * mb + g + 8);
                #pragma unroll
                for (int nt = 0; nt < 4; ++nt)
                    #pragma unroll
                    for (int e = 0; e < 2; ++e) {
                        acc[2 * nt + e] += v0[4 * nt + e] * f0 + v0[4 * nt + 2 + e] * f1;
                        acc[8 + 2 * nt + e] += v1[4 * nt + e] * f0 + v1[4 * nt + 2 + e] * f1;
                    }
            }
            float out[2];
            reduce_scatter16(acc, out, lane);
            const int nt = 4 * ((lane >> 4) & 1) + 2 * ((lane >> 3) & 1) + ((lane >> 2) & 1);
            #pragma unroll
            for (int e = 0; e < 2; ++e) {
                const int r = 64 * hf + 8 * nt + 2 * tig + e;
                const bool hb = ((uint32_t)sm.meta[ms][warp][4 + (r >> 5)] >> (r & 31)) & 1u;
                if (r < n_lo && !hb) mrow[lo0 + r] = out[e];
            }
        }
        // full-rank tokens
        for (int hs = 0; hs * kHiTok < nh; ++hs) {
            const int n = min(kHiTok, nh - kHiTok * hs);
            float acc[8];
            #pragma unroll
            for (int i = 0; i < 8; ++i) acc[i] = 0.f;
            const int upd = C::kLoTok / 64 + hs;
            #pragma unroll
            for (int mb = 0; mb < NMB; ++mb) {
                float v[16];
                const uint32_t col = (uint32_t)(128 * b + 64 + (NMB == 1 ? 16 * hs : 32 * hs + 16 * mb));
                tmem_ld16(tmem + col, v);
                tmem_wait_ld();
                const float f0 = fac(upd, 16 * mb + g), f1 = fac(upd, 16 * mb + g + 8);
                #pragma unroll
                for (int nt = 0; nt < 4; ++nt)
                    #pragma unroll
                    for (int e = 0; e < 2; ++e) acc[2 * nt + e] += v[4 * nt + e] * f0 + v[4 * nt + 2 + e] * f1;
            }
            const float val = reduce_scatter8(acc, lane);
            const int j = 4 * ((lane >> 4) & 1) + 2 * ((lane >> 3) & 1) + ((lane >> 2) & 1);
            const int colt = 8 * (j >> 1) + 2 * tig + (j & 1);
            if (colt < n) mrow[sm.hi_list[ms][warp][kHiTok * hs + colt]] = val;
        }
        tmem_fence_before();
    };

    int K = 0;
    for (;; ++K) {
        const int item = item_of(K);
        if (item >= p.n_items) break;
        Kc = K;
        pump();
        const int ms = K % kMeta, b = K & 1;
        const int n_lo = sm.meta[ms][warp][1], nh = sm.meta[ms][warp][2];
        uint32_t lw[4];
        #pragma unroll
        for (int k = 0; k < 4; ++k) lw[k] = (uint32_t)sm.meta[ms][warp][4 + k];
        const int unit = item / p.S, split = item % p.S;

        bool ok = mbar_wait(&sm.qbar, (uint32_t)(K & 1), abort);
        #pragma unroll
        for (int mb = 0; mb < NMB; ++mb) {
            const int row = 16 * mb + (lane & 7) + (((lane >> 3) & 1) << 3);
            const uint32_t off = row * 128 + (((lane >> 4) ^ (row & 7)) << 4);
            ldsm_x4(qt0 + off, qah[mb][0], qah[mb][1], qah[mb][2], qah[mb][3]);
            ldsm_x4(qt1 + off, qal[mb][0], qal[mb][1], qal[mb][2], qal[mb][3]);
            m[mb][0] = m[mb][1] = -INFINITY;
            l[mb][0] = l[mb][1] = 0.f;
            #pragma unroll
            for (int a = 0; a < 8; ++a) u[mb][a][0] = u[mb][a][1] = u[mb][a][2] = u[mb][a][3] = 0.f;
        }
        const uint32_t tcol = tmem + 128u * (uint32_t)b;
        const int nst = (n_lo > 0 ? 1 : 0) + (nh + kHiTok - 1) / kHiTok;

        for (int st = 0; st < nst && ok; ++st) {
            const int slot = c_seq % kSlots;
            if (!mbar_wait(&sm.full[warp][slot], (c_seq / kSlots) & 1u, abort)) { ok = false; break; }
            const uint32_t sb = smem_u32(sm.ring[warp][slot]);
            if (st == 0 && n_lo > 0) {
                // ------------------------------------------------ LO range
                #pragma unroll
                for (int hf = 0; hf < C::kLoTok / 64; ++hf) {
                    if (64 * hf < n_lo) {
                        uint32_t kf[4][4];
                        #pragma unroll
                        for (int np = 0; np < 4; ++np) {
                            const int row = 64 * hf + 16 * np + (lane & 7) + ((lane >> 4) << 3);
                            const int ch = (lane >> 3) & 1;
                            ldsm_x4(sb + row * 32 + ((ch ^ ((row >> 2) & 1)) << 4), kf[np][0], kf[np][1], kf[np][2],
                                    kf[np][3]);
                        }
                        #pragma unroll
                        for (int mb = 0; mb < NMB; ++mb) {
                            float s[8][4];
                            #pragma unroll
                            for (int a = 0; a < 8; ++a) s[a][0] = s[a][1] = s[a][2] = s[a][3] = 0.f;
                            #pragma unroll
                            for (int np = 0; np < 4; ++np) {
                                mma_bf16(s[2 * np], qah[mb], kf[np][0], kf[np][1]);
                                mma_bf16(s[2 * np], qal[mb], kf[np][0], kf[np][1]);
                                mma_bf16(s[2 * np + 1], qah[mb], kf[np][2], kf[np][3]);
                                mma_bf16(s[2 * np + 1], qal[mb], kf[np][2], kf[np][3]);
                            }
                            #pragma unroll
                            for (int nt = 0; nt < 8; ++nt)
                                #pragma unroll
                                for (int e = 0; e < 2; ++e) {
                                    const int r = 64 * hf + 8 * nt + 2 * tig + e;
                                    const bool hb = (lw[r >> 5] >> (r & 31)) & 1u;
                                    if (r >= n_lo || hb) s[nt][e] = s[nt][2 + e] = -INFINITY;
                                }
                            const float mn0 = softmax_row<8>(s, 0, m[mb][0], l[mb][0], u[mb]);
                            const float mn1 = softmax_row<8>(s, 1, m[mb][1], l[mb][1], u[mb]);
                            if (p.mass != nullptr) {
                                if (tig == 0) {
                                    sm.mref[b][warp][hf][16 * mb + g] = mn0;
                                    sm.mref[b][warp][hf][16 * mb + g + 8] = mn1;
                                }
                                const uint32_t col = tcol + (uint32_t)(32 * (NMB == 1 ? hf : mb));
                                float v0[16], v1[16];
                                #pragma unroll
                                for (int i = 0; i < 16; ++i) {
                                    v0[i] = s[i >> 2][i & 3];
                                    v1[i] = s[4 + (i >> 2)][i & 3];
                                }
                                tmem_st16(col, v0);
                                tmem_st16(col + 16, v1);
                            }
                            #pragma unroll
                            for (int kk = 0; kk < 4; ++kk) {
                                uint32_t a[4];
                                a[0] = pack_bf16(s[2 * kk][0], s[2 * kk][1]);
                                a[1] = pack_bf16(s[2 * kk][2], s[2 * kk][3]);
                                a[2] = pack_bf16(s[2 * kk + 1][0], s[2 * kk + 1][1]);
                                a[3] = pack_bf16(s[2 * kk + 1][2], s[2 * kk + 1][3]);
                                uint32_t b0, b1, b2, b3;
                                const int row = 64 * hf + 16 * kk + (lane & 7) + (((lane >> 3) & 1) << 3);
                                const int ch = lane >> 4;
                                ldsm_x4_t(sb + 4096 + row * 32 + ((ch ^ ((row >> 2) & 1)) << 4), b0, b1, b2, b3);
                                mma_bf16(u[mb][0], a, b0, b1);
                                mma_bf16(u[mb][1], a, b2, b3);
                            }
                        }
                    }
                }
            } else {
                // ------------------------------------------------ HI stage
                const int hs = st - (n_lo > 0 ? 1 : 0);
                const int n = min(kHiTok, nh - kHiTok * hs);
                const int upd = C::kLoTok / 64 + hs;
                #pragma unroll
                for (int mb = 0; mb < NMB; ++mb) {
                    float s[4][4];
                    #pragma unroll
                    for (int a = 0; a < 4; ++a) s[a][0] = s[a][1] = s[a][2] = s[a][3] = 0.f;
                    #pragma unroll
                    for (int kb = 0; kb < 4; ++kb) {
                        uint32_t ah[4], al[4];
                        if (kb == 0) {
                            #pragma unroll
                            for (int e = 0; e < 4; ++e) { ah[e] = qah[mb][e]; al[e] = qal[mb][e]; }
                        } else {
                            const int row = 16 * mb + (lane & 7) + (((lane >> 3) & 1) << 3);
                            const int ch = 2 * kb + (lane >> 4);
                            const uint32_t off = row * 128 + ((ch ^ (row & 7)) << 4);
                            ldsm_x4(qt0 + off, ah[0], ah[1], ah[2], ah[3]);
                            ldsm_x4(qt1 + off, al[0], al[1], al[2], al[3]);
                        }
                        #pragma unroll
                        for (int np = 0; np < 2; ++np) {
                            uint32_t b0, b1, b2, b3;
                            const int row = 16 * np + (lane & 7) + ((lane >> 4) << 3);
                            const int ch = 2 * kb + ((lane >> 3) & 1);
                            ldsm_x4(sb + row * 128 + ((ch ^ (row & 7)) << 4), b0, b1, b2, b3);
                            mma_bf16(s[2 * np], ah, b0, b1);
                            mma_bf16(s[2 * np], al, b0, b1);
                            mma_bf16(s[2 * np + 1], ah, b2, b3);
                            mma_bf16(s[2 * np + 1], al, b2, b3);
                        }
                    }
                    #pragma unroll
                    for (int nt = 0; nt < 4; ++nt)
                        #pragma unroll
                        for (int e = 0; e < 2; ++e)
                            if (8 * nt + 2 * tig + e >= n) s[nt][e] = s[nt][2 + e] = -INFINITY;
                    const float mn0 = softmax_row<4>(s, 0, m[mb][0], l[mb][0], u[mb]);
                    const float mn1 = softmax_row<4>(s, 1, m[mb][1], l[mb][1], u[mb]);
                    if (p.mass != nullptr) {
                        if (tig == 0) {
                            sm.mref[b][warp][upd][16 * mb + g] = mn0;
                            sm.mref[b][warp][upd][16 * mb + g + 8] = mn1;
                        }
                        const uint32_t col = tcol + (uint32_t)(64 + (NMB == 1 ? 16 * hs : 32 * hs + 16 * mb));
                        float v0[16];
                        #pragma unroll
                        for (int i = 0; i < 16; ++i) v0[i] = s[i >> 2][i & 3];
                        tmem_st16(col, v0);
                    }
                    #pragma unroll
                    for (int kk = 0; kk < 2; ++kk) {
                        uint32_t a[4];
                        a[0] = pack_bf16(s[2 * kk][0], s[2 * kk][1]);
                        a[1] = pack_bf16(s[2 * kk][2], s[2 * kk][3]);
                        a[2] = pack_bf16(s[2 * kk + 1][0], s[2 * kk + 1][1]);
                        a[3] = pack_bf16(s[2 * kk + 1][2], s[2 * kk + 1][3]);
                        #pragma unroll
                        for (int pr = 0; pr < 4; ++pr) {
                            uint32_t b0, b1, b2, b3;
                            const int row = 16 * kk + (lane & 7) + (((lane >> 3) & 1) << 3);
                            const int ch = 2 * pr + (lane >> 4);
                            ldsm_x4_t(sb + 4096 + row * 128 + ((ch ^ (row & 7)) << 4), b0, b1, b2, b3);
                            mma_bf16(u[mb][2 * pr], a, b0, b1);
                            mma_bf16(u[mb][2 * pr + 1], a, b2, b3);
                        }
                    }
                }
            }
            ++c_seq;
            __syncwarp();
            pump();
        }
        if (!ok) *abort = 1;
        if (p.mass != nullptr) tmem_wait_st();

        // ================================================ item epilogue
        #pragma unroll
        for (int mb = 0; mb < NMB; ++mb)
            #pragma unroll
            for (int r = 0; r < 2; ++r) {
                float lt = l[mb][r];
                lt += __shfl_xor_sync(0xffffffffu, lt, 1);
                lt += __shfl_xor_sync(0xffffffffu, lt, 2);
                if (tig == 0) {
                    sm.wm[warp][16 * mb + g + 8 * r] = m[mb][r];
                    sm.wl[warp][16 * mb + g + 8 * r] = lt;
                }
            }
        tmem_fence_before();
        __syncthreads();
        if (*abort) break;
        if (tid == 0 && item_of(K + 1) < p.n_items) issue_q(K + 1);
        if (tid < C::kRows) {
            float mx = -INFINITY;
            for (int w = 0; w < kWarps; ++w) mx = fmaxf(mx, sm.wm[w][tid]);
            float sum = 0.f;
            if (mx != -INFINITY)
                for (int w = 0; w < kWarps; ++w) {
                    const float mw_ = sm.wm[w][tid];
                    if (mw_ != -INFINITY) sum += sm.wl[w][tid] * ex2(mw_ - mx);
                }
            sm.mcta[tid] = mx;
            sm.lcta[tid] = sum;
        }
        __syncthreads();
        #pragma unroll
        for (int mb = 0; mb < NMB; ++mb)
            #pragma unroll
            for (int r = 0; r < 2; ++r) {
                const int row = 16 * mb + g + 8 * r;
                const float f = (row < p.Hg && m[mb][r] != -INFINITY) ? ex2(m[mb][r] - sm.mcta[row]) : 0.f;
                if (f != 0.f) {
                    #pragma unroll
                    for (int nt = 0; nt < 8; ++nt) {
                        atomicAdd(&sm.u_acc[row][8 * nt + 2 * tig], u[mb][nt][2 * r] * f);
                        atomicAdd(&sm.u_acc[row][8 * nt + 2 * tig + 1], u[mb][nt][2 * r + 1] * f);
                    }
                }
            }
        __syncthreads();
        {
            float *dst = p.part + ((size_t)unit * p.S + split) * p.Hg * kVisPart;
            for (int i = tid; i < p.Hg * kVisPart; i += kThreads) {
                const int h = i / kVisPart, f = i % kVisPart;
                float v;
                if (f == 0) v = sm.mcta[h];
                else if (f == 1) v = sm.lcta[h];
                else { v = sm.u_acc[h][f - 2]; sm.u_acc[h][f - 2] = 0.f; }
                dst[i] = v;
            }
        }
        __threadfence();
        __syncthreads();
        if (tid == 0) asm volatile("red.release.gpu.global.add.u32 [%0], 1;" :: "l"(&p.arrive[unit]) : "memory");
        if (p.mass != nullptr && K >= 1) {
            mass_of(K - 1);
            if (*abort) break;
        }
    }
    if (p.mass != nullptr && K >= 1 && !*abort) mass_of(K - 1);

    // copies still in flight (only after an abort) must land before the block exits
    while (c_seq < i_seq) {
        const int slot = c_seq % kSlots;
        const uint32_t par = (c_seq / kSlots) & 1u;
        const long long t0 = clock64();
        while (!mbar_try_wait(&sm.full[warp][slot], par) && clock64() - t0 < kWaitCycles) {}
        ++c_seq;
    }
    cp_async_wait_all();
    tmem_fence_before();
    __syncthreads();
    if (warp == 0) {
        tmem_fence_after();
        tmem_dealloc(sm.tmem_base, 512);
    }
}

}  // namespace vis

// ======================================================================= finish

struct FinishParams {
    const uint16_t *BV;       // [units][64][512]
    const float *vpart;       // [units][S][Hg][kVisPart]
    const float *tpart;       // [units][Sc][Hg][kTxtPart] or null
    uint16_t *out;            // [(layer, batch)][n_q][128]
    int Hg, per_kv, n_q, groups, S, Sc;
};

// One block per unit: unit-wide max and sum per head, u / l and w / l from the
// partials, then o_h = (u_h / l_h) B_V[:, 128 j(h) ..] + w_h / l_h with thread
// t owning output columns 2t, 2t+1 of the unit's 512 (KV head t / 64).
__global__ void __launch_bounds__(256) finish_kernel(const FinishParams p) {
    __shared__ float mfin[kMaxHeads], invl[kMaxHeads];
    __shared__ float uf[kMaxHeads][64];
    __shared__ float wf[kMaxHeads][128];
    const int unit = blockIdx.x, tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const float *vp0 = p.vpart + (size_t)unit * p.S * p.Hg * kVisPart;
    const float *tp0 = p.tpart + (size_t)unit * p.Sc * p.Hg * kTxtPart;

    // B_V columns 2t, 2t+1 of all 64 rank rows (issued first: independent of the partials)
    const uint32_t *bv = reinterpret_cast<const uint32_t *>(p.BV + (size_t)unit * 64 * 512) + tid;
    uint32_t braw[64];
    #pragma unroll
    for (int i = 0; i < 64; ++i) braw[i] = __ldcs(bv + i * 256);

    for (int h = warp; h < p.Hg; h += 8) {
        float mx = -INFINITY;
        for (int s = lane; s < p.S; s += 32) mx = fmaxf(mx, vp0[((size_t)s * p.Hg + h) * kVisPart]);
        for (int c = lane; c < p.Sc; c += 32) mx = fmaxf(mx, tp0[((size_t)c * p.Hg + h) * kTxtPart]);
        #pragma unroll
        for (int d = 16; d > 0; d >>= 1) mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, d));
        float sum = 0.f;
        for (int s = lane; s < p.S; s += 32) {
            const float *r = vp0 + ((size_t)s * p.Hg + h) * kVisPart;
            if (r[0] != -INFINITY) sum += r[1] * ex2(r[0] - mx);
        }
        for (int c = lane; c < p.Sc; c += 32) {
            const float *r = tp0 + ((size_t)c * p.Hg + h) * kTxtPart;
            if (r[0] != -INFINITY) sum += r[1] * ex2(r[0] - mx);
        }
        #pragma unroll
        for (int d = 16; d > 0; d >>= 1) sum += __shfl_xor_sync(0xffffffffu, sum, d);
        if (lane == 0) {
            mfin[h] = mx;
            invl[h] = 1.f / sum;
        }
    }
    __syncthreads();
    for (int task = tid; task < p.Hg * 192; task += 256) {
        const int h = task / 192, f = task % 192;
        const float mh = mfin[h];
        float acc = 0.f;
        if (f < 64) {
            for (int s = 0; s < p.S; ++s) {
                const float *r = vp0 + ((size_t)s * p.Hg + h) * kVisPart;
                if (r[0] != -INFINITY) acc = fmaf(r[2 + f], ex2(r[0] - mh), acc);
            }
            uf[h][f] = acc * invl[h];
        } else {
            for (int c = 0; c < p.Sc; ++c) {
                const float *r = tp0 + ((size_t)c * p.Hg + h) * kTxtPart;
                if (r[0] != -INFINITY) acc = fmaf(r[2 + f - 64], ex2(r[0] - mh), acc);
            }
            wf[h][f - 64] = acc * invl[h];
        }
    }
    __syncthreads();
    const int j = tid >> 6, d = (2 * tid) & 127;
    const int lb = unit / p.groups, G = unit % p.groups;
    for (int hh = 0; hh < p.per_kv; ++hh) {
        const int h = j * p.per_kv + hh;
        float a0 = 0.f, a1 = 0.f;
        #pragma unroll
        for (int i = 0; i < 64; ++i) {
            const float x = uf[h][i];
            a0 = fmaf(x, __uint_as_float(braw[i] << 16), a0);
            a1 = fmaf(x, __uint_as_float(braw[i] & 0xffff0000u), a1);
        }
        a0 += wf[h][d];
        a1 += wf[h][d + 1];
        *reinterpret_cast<uint32_t *>(p.out + ((size_t)lb * p.n_q + (size_t)G * p.Hg + h) * 128 + d) = pack_bf16(a0, a1);
    }
}

}  // namespace decode
}  // namespace kvpack

namespace kvpack {
namespace decode {
// one block per SM: the opt-in shared-memory limit per block on sm_100 is 232448 bytes
static_assert(vis::smem_bytes<1>() <= 232448, "visual kernel (16 head rows) shared memory");
static_assert(vis::smem_bytes<2>() <= 232448, "visual kernel (32 head rows) shared memory");
static_assert(text::smem_bytes() <= 232448, "text kernel shared memory");
}  // namespace decode
}  // namespace kvpack
