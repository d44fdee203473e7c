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
// This file holds the decode call's first launch, the text kernel:
//   text_kernel  q~ = scale * log2(e) * B_K[:, 128 j(h) ..] q_h per (unit, KV head), split into
//                bf16 hi + lo; and the text tail (plain bf16 K/V) per (unit, KV head, chunk of
//                tokens): partial (max, sum, w = sum p V) per query head
// The visual tokens, the unit-wide softmax statistics and the final projection are
// rstream.cuh's.  Logits are kept in the log2 domain (the scale folds log2(e)).
#pragma once

#include <cuda.h>

#include <type_traits>

#include "common.cuh"

namespace kvpack {
namespace decode {

constexpr int kTxtPart = 130;   // per (unit, text chunk, head): max, sum, w[128]

// =================================================================== query block

// Per unit, the query block the visual passes copy plane by plane:
//   [2][Hg][64] bf16  q~ hi then lo (128-byte rows, 16-byte chunk c stored at c ^ (r & 7) with r the
//                     row the head lands in: h, or h + 2 for heads >= qsplit in the 28-head form)
__host__ __device__ constexpr size_t qblock_bytes(int Hg) { return (size_t)Hg * 2 * 128; }

// ========================================================================= text

namespace text {

constexpr int kWarps = 8;
constexpr int kThreads = kWarps * 32;
constexpr int kSlots = 3;
constexpr int kSlotBytes = 8192;   // 16 text tokens x (K 256 B + V 256 B) of one KV head, or 64 B_K rows x 128 B
constexpr int kTile = 16;

struct Params {
    CUtensorMap tm_k, tm_v;    // text: 4D {128, 4, L, units}, box {64, 1, 16, 1}, 128-byte swizzle
    CUtensorMap tm_bk;         // B_K: 3D {512, 64, units}, box {64, 64, 1}, 128-byte swizzle
    CUtensorMap tm_bk2;        // the text tokens' own B_K (same layout), when they are compressed too
    const uint16_t *q;
    float *part;               // [units][Sc][Hg][kTxtPart]
    unsigned char *qt;         // [units][qblock_bytes(Hg)]: q~ written here
    unsigned char *qt2;        // the same for the text tokens' basis, or null
    unsigned int *counter;     // work counter, zero at launch
    int n_units, L, Hg, per_kv, n_q, groups, Sc, ct, n_qitems, n_items;
    int qsplit;                // heads >= qsplit sit 2 rows lower in the visual passes' q~ tile (28-head form)
    float scale2;
};

struct Smem {
    alignas(1024) unsigned char ring[kWarps][kSlots][kSlotBytes];
    uint64_t full[kWarps][kSlots];
    int itemq[kWarps][8];
    int abort;
};

constexpr size_t smem_bytes() { return sizeof(Smem) + 1024; }

// Every warp streams whole work items through its own 3-slot ring, fetched from
// a global counter.  Items 0 .. n_qitems-1 project the query to rank space for
// (unit, KV head j): two stages of B_K (64 rank rows x 64 columns each), q~^T =
// B_K[:, 128 j ..] q^T on mma.sync (ranks on M, the KV head's query heads on N),
// written as the bf16 hi + lo pair of the unit's query block (items 4 units ..
// 8 units - 1, when present, do the same with the text tokens' basis).  The others are
// text items -- (unit, KV head j, chunk of ct text tokens): per 16-token tile,
// S = K q^T with tokens on M and the query heads on N, an online softmax down
// the columns, and w^T += V^T P (the transposed P from movmatrix); at the end of
// an item the partial (max, sum, w) of each query head.
__global__ void __launch_bounds__(kThreads, 1) text_kernel(const __grid_constant__ Params p) {
    extern __shared__ __align__(1024) unsigned char smem_raw[];
    const uint32_t base = smem_u32(smem_raw);
    Smem &sm = *reinterpret_cast<Smem *>(smem_raw + ((1024u - (base & 1023u)) & 1023u));
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int g = lane >> 2, tig = lane & 3;
    griddep_launch_dependents();
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
    // (unit, KV head) of an item
    auto unit_of = [&](int it) { return it < p.n_qitems ? (it % (4 * p.n_units)) >> 2 : (it - p.n_qitems) / (4 * p.Sc); };
    auto kvh_of = [&](int it) { return it < p.n_qitems ? it & 3 : ((it - p.n_qitems) / p.Sc) & 3; };
    auto n_tok = [&](int it) { const int c = (it - p.n_qitems) % p.Sc; return min(p.ct, p.L - c * p.ct); };
    auto n_tiles = [&](int it) { return it < p.n_qitems ? 2 : (n_tok(it) + kTile - 1) / kTile; };

    // ---- issue side
    int i_item = -1, i_tile = 0, i_ntiles = 0, q_push = 0;
    bool i_done = false;
    uint32_t i_seq = 0, c_seq = 0;
    auto issue = [&]() {
        if (i_done) return;
        if (i_tile == i_ntiles) {
            const int it = fetch();
            if (it >= p.n_items) { i_done = true; return; }
            i_item = it; i_tile = 0; i_ntiles = n_tiles(it);
            if (lane == 0) sm.itemq[warp][q_push & 7] = it;
            ++q_push;
        }
        const int slot = i_seq % kSlots;
        const int unit = unit_of(i_item), j = kvh_of(i_item);
        __syncwarp();
        if (lane == 0) {
            unsigned char *dst = sm.ring[warp][slot];
            uint64_t *bar = &sm.full[warp][slot];
            fence_proxy_async();
            mbar_arrive_tx(bar, kSlotBytes);
            if (i_item < p.n_qitems) {
                tma_3d(dst, i_item >= 4 * p.n_units ? &p.tm_bk2 : &p.tm_bk, 128 * j + 64 * i_tile, 0, unit, bar);
            } else {
                const int tok = ((i_item - p.n_qitems) % p.Sc) * p.ct + i_tile * kTile;
                tma_4d(dst, &p.tm_k, 0, j, tok, unit, bar);
                tma_4d(dst + 2048, &p.tm_k, 64, j, tok, unit, bar);
                tma_4d(dst + 4096, &p.tm_v, 0, j, tok, unit, bar);
                tma_4d(dst + 6144, &p.tm_v, 64, j, tok, unit, bar);
            }
        }
        ++i_tile;
        ++i_seq;
    };

    // query rows of (unit, j) as B fragments: b0 = q[g][16 kb + 2 tig ..], b1 = q[g][16 kb + 8 + 2 tig ..]
    auto load_q = [&](int it, uint32_t (&qf)[8][2]) {
        const int unit = unit_of(it), j = kvh_of(it);
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
            c_ntiles = n_tiles(c_item);
            c_n = c_item < p.n_qitems ? 0 : n_tok(c_item);
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

        if (c_item < p.n_qitems) {
            // ---------------- q~ projection: this stage holds B_K[64 ranks][64 columns] of KV head j,
            // k-steps 4 c_tile .. 4 c_tile + 3 of the 128-column product, accumulated in wt[0..3]
            auto proj = [&](auto half) {
                constexpr int H = decltype(half)::value;
                #pragma unroll
                for (int kq = 0; kq < 4; ++kq) {
                    #pragma unroll
                    for (int mt = 0; mt < 4; ++mt) {
                        uint32_t a[4];
                        const int row = 16 * mt + (lane & 7) + (((lane >> 3) & 1) << 3);
                        const int ch = 2 * kq + (lane >> 4);
                        ldsm_x4(sb + row * 128 + ((ch ^ (row & 7)) << 4), a[0], a[1], a[2], a[3]);
                        mma_bf16(wt[mt], a, qf[4 * H + kq][0], qf[4 * H + kq][1]);
                    }
                }
            };
            if (c_tile == 0) proj(std::integral_constant<int, 0>());
            else proj(std::integral_constant<int, 1>());
            ++c_tile;
            ++c_seq;
            if (c_tile == c_ntiles) {
                // wt[mt][e]: rank 16 mt + g (+8 for e >= 2), head 2 tig + (e & 1) of KV head j
                const int unit = unit_of(c_item), j = kvh_of(c_item);
                unsigned char *qb = c_item >= 4 * p.n_units ? p.qt2 : p.qt;
                uint16_t *qt = reinterpret_cast<uint16_t *>(qb + (size_t)unit * qblock_bytes(p.Hg));
                #pragma unroll
                for (int mt = 0; mt < 4; ++mt)
                    #pragma unroll
                    for (int e = 0; e < 4; ++e) {
                        const int hh = 2 * tig + (e & 1);
                        if (hh < p.per_kv) {
                            const int h = j * p.per_kv + hh, i = 16 * mt + g + 8 * (e >> 1);
                            const float v = wt[mt][e] * p.scale2;
                            const uint16_t hi = float_to_bf16_bits(v);
                            const uint16_t lo = float_to_bf16_bits(v - bf16_bits_to_float(hi));
                            const int ph = h + (h >= p.qsplit ? 2 : 0);   // the row it lands in
                            const int off = h * 64 + ((((i >> 3) ^ (ph & 7)) & 7) << 3) + (i & 7);
                            qt[off] = hi;
                            qt[p.Hg * 64 + off] = lo;
                        }
                    }
            }
            __syncwarp();
            if (i_seq - c_seq < (uint32_t)kSlots) issue();
            continue;
        }

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
            const int unit = unit_of(c_item), j = kvh_of(c_item), c = (c_item - p.n_qitems) % p.Sc;
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

static_assert(text::smem_bytes() <= 232448, "text kernel shared memory");
}  // namespace decode
}  // namespace kvpack
