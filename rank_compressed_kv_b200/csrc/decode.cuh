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
// Four of the decode call's five launches live here (the fifth, the attention
// mass of every visual token, is mass.cuh), each streaming its own bytes once:
//   text_kernel        q~ = scale * log2(e) * B_K[:, 128 j(h) ..] q_h per (unit, KV head), split
//                      into bf16 hi + lo; and the text tail (plain bf16 K/V) per (unit, KV head,
//                      chunk of tokens): partial (max, sum, w = sum p V) per query head
//   text_stats_kernel  the text tail's (max, sum) per head folded over its chunks, one warp per unit
//   vis_kernel         the compressed visual tokens per (unit, chunk of tokens), one warp per
//                      item: partial (max, sum, u = sum p C_V) per query head
//   finish_kernel      combines the partials of a unit and projects: o_h = (u B_V + w) / l, and
//                      publishes the unit's (max, 1/sum) per head for the mass pass
// Logits are kept in the log2 domain (the scale folds log2(e)).
#pragma once

#include <cuda.h>

#include <type_traits>

#include "common.cuh"

namespace kvpack {
namespace decode {

constexpr int kTxtPart = 130;   // per (unit, text chunk, head): max, sum, w[128]
constexpr int kVisPart = 66;    // per (unit, visual chunk, head): max, sum, u[64]

// =================================================================== query block

// Per unit, the query block the visual kernel copies in one piece:
//   [2][Hg][64] bf16  q~ hi then lo (128-byte rows, 16-byte chunk c stored at c ^ (h & 7))
//   [Hg][2]     f32   the text tail's (max, sum) per head, combined over its chunks
__host__ __device__ constexpr size_t qblock_bytes(int Hg) { return (size_t)Hg * (2 * 128 + 8); }

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
    const uint16_t *q;
    float *part;               // [units][Sc][Hg][kTxtPart]
    unsigned char *qt;         // [units][qblock_bytes(Hg)]: q~ written here
    unsigned int *counter;     // work counter, zero at launch
    int n_units, L, Hg, per_kv, n_q, groups, Sc, ct, n_qitems, n_items;
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
// written as the bf16 hi + lo pair of the unit's query block.  The others are
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
    auto unit_of = [&](int it) { return it < p.n_qitems ? it >> 2 : (it - p.n_qitems) / (4 * p.Sc); };
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
                tma_3d(dst, &p.tm_bk, 128 * j + 64 * i_tile, 0, unit, bar);
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
                uint16_t *qt = reinterpret_cast<uint16_t *>(p.qt + (size_t)unit * qblock_bytes(p.Hg));
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
                            const int off = h * 64 + ((((i >> 3) ^ (h & 7)) & 7) << 3) + (i & 7);
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

// The text tail's (max, sum) per head of every unit, folded over its chunks
// into the unit's query block (one warp per unit, a lane per head).
__global__ void __launch_bounds__(256) text_stats_kernel(const float *__restrict__ part, unsigned char *qt, int units,
                                                         int Hg, int Sc) {
    const int unit = blockIdx.x * 8 + (threadIdx.x >> 5), h = threadIdx.x & 31;
    if (unit >= units || h >= Hg) return;
    const float *tp = part + (size_t)unit * Sc * Hg * kTxtPart + (size_t)h * kTxtPart;
    float mx = -INFINITY;
    for (int c = 0; c < Sc; ++c) mx = fmaxf(mx, tp[(size_t)c * Hg * kTxtPart]);
    float sum = 0.f;
    for (int c = 0; c < Sc; ++c) {
        const float mc = tp[(size_t)c * Hg * kTxtPart];
        if (mc != -INFINITY) sum += tp[(size_t)c * Hg * kTxtPart + 1] * ex2(mc - mx);
    }
    float *ts = reinterpret_cast<float *>(qt + (size_t)unit * qblock_bytes(Hg) + (size_t)Hg * 256);
    ts[2 * h] = mx;
    ts[2 * h + 1] = sum;
}

}  // namespace text

// ======================================================================== visual

namespace vis {

constexpr int kWarps = 8;
constexpr int kThreads = kWarps * 32;
constexpr int kSub = 64;        // tokens per sub-chunk: one LO stage
constexpr int kMaxItemTok = 2048;               // tokens per item, at most
constexpr int kMaxItemWords = kMaxItemTok / 32;

// Geometry per head-block count.  Up to 16 query heads per unit: two blocks per
// SM.  Up to 32: one block per SM with a deeper ring.
template <int NMB>
struct Cfg {
    static constexpr int kRows = 16 * NMB;                      // query-head rows (padded)
    static constexpr int kBlocks = (NMB == 1) ? 2 : 1;          // resident blocks per SM
    static constexpr int kSlots = (NMB == 1) ? 2 : 4;           // ring slots per warp
    static constexpr int kSlotBytes = 4096;                     // K rows in the first half, V in the second
    static constexpr int kQStages = NMB;                        // ring stages of an item's q~ (hi, lo planes)
    static constexpr int kHiTok = 16;                           // full-rank tokens per HI stage
    static constexpr int kNTH = kHiTok / 8;                     // m16n8 token tiles per HI stage
    static_assert(kHiTok * 128 == kSlotBytes / 2, "HI stage rows fill half a slot");
    static_assert(kSub * 32 == kSlotBytes / 2, "LO stage rows fill half a slot");
};

struct Params {
    CUtensorMap tm_ck, tm_cv;   // C_lo planes: 3D {16, T, units}, box {16, 32, 1}, 32-byte swizzle
    const uint16_t *CK_lo, *CK_hi, *CV_lo, *CV_hi;
    const unsigned char *qt;    // [units][qblock_bytes(Hg)] from text_kernel
    const uint32_t *mask;       // [units][nwords]
    float *part;                // [units][S][Hg][kVisPart]
    unsigned int *counter;      // work counter, zero at launch
    int n_units, T, Hg, S, tps, nwords, n_items;
};

template <int NMB>
struct Smem {
    using C = Cfg<NMB>;
    alignas(1024) unsigned char ring[kWarps][C::kSlots][C::kSlotBytes];
    uint16_t hi_list[kWarps][kMaxItemTok];                   // item-relative positions of the issue side's item's
                                                             // full-rank tokens
    uint32_t mw[kWarps][kMaxItemWords];                      // that item's mask words
    int desc[kWarps][C::kSlots][6];                          // per ring slot: flags, item, n, w0, w1
    uint64_t full[kWarps][C::kSlots];
    int abort;
};

template <int NMB>
constexpr size_t smem_bytes() { return sizeof(Smem<NMB>) + 1024; }

// Reference a row starts from: any finite logit exceeds it by more than kLazy.
constexpr float kRefInit = -1e30f;
// The reference max of a row moves only when a logit exceeds it by more than
// kLazy (log2 units), so p = 2^(s - m) stays below 2^kLazy and the (rare)
// rescale of l and u is a warp-uniform branch.
constexpr float kLazy = 8.f;

// One online-softmax update of the block's rows g and g + 8 over NT m16n8
// score tiles (log2 domain, masked logits -inf).  p overwrites s.
template <int NT>
__device__ __forceinline__ void lazy_update(float (&s)[NT][4], float (&m)[2], float (&l)[2], float (&u)[8][4]) {
    float mx0 = fmaxf(s[0][0], s[0][1]), mx1 = fmaxf(s[0][2], s[0][3]);
    #pragma unroll
    for (int nt = 1; nt < NT; ++nt) {
        mx0 = fmaxf(mx0, fmaxf(s[nt][0], s[nt][1]));
        mx1 = fmaxf(mx1, fmaxf(s[nt][2], s[nt][3]));
    }
    mx0 = fmaxf(mx0, __shfl_xor_sync(0xffffffffu, mx0, 1));
    mx1 = fmaxf(mx1, __shfl_xor_sync(0xffffffffu, mx1, 1));
    mx0 = fmaxf(mx0, __shfl_xor_sync(0xffffffffu, mx0, 2));
    mx1 = fmaxf(mx1, __shfl_xor_sync(0xffffffffu, mx1, 2));
    const bool up0 = mx0 > m[0] + kLazy, up1 = mx1 > m[1] + kLazy;
    if (__any_sync(0xffffffffu, up0 || up1)) {
        const float n0 = up0 ? mx0 : m[0], n1 = up1 ? mx1 : m[1];
        const float a0 = ex2(m[0] - n0), a1 = ex2(m[1] - n1);
        l[0] *= a0;
        l[1] *= a1;
        #pragma unroll
        for (int nt = 0; nt < 8; ++nt) {
            u[nt][0] *= a0; u[nt][1] *= a0; u[nt][2] *= a1; u[nt][3] *= a1;
        }
        m[0] = n0;
        m[1] = n1;
    }
    float sum0 = 0.f, sum1 = 0.f;
    #pragma unroll
    for (int nt = 0; nt < NT; ++nt) {
        s[nt][0] = ex2(s[nt][0] - m[0]);
        s[nt][1] = ex2(s[nt][1] - m[0]);
        s[nt][2] = ex2(s[nt][2] - m[1]);
        s[nt][3] = ex2(s[nt][3] - m[1]);
        sum0 += s[nt][0] + s[nt][1];
        sum1 += s[nt][2] + s[nt][3];
    }
    l[0] += sum0;
    l[1] += sum1;
}

// Persistent, one or two 256-thread blocks per SM; every warp works alone.
// A warp fetches items (unit, chunk of tps <= 2048 tokens) from a global
// counter and streams each through a private ring: the unit's q~, then one
// TMA stage of C_lo rows of K and V per 64-token sub-chunk (skipped when every
// token of it is full-rank), then the item's full-rank tokens 16 at a time
// (C_lo + C_hi rows of K and V gathered by cp.async; the issue side lists
// them once per item, so only the item's last gathered stage is partial).
// With heads on M and tokens on N of mma.sync m16n8k16:
//   scores  s = q~ C_K^T  (q~ as a bf16 hi + lo pair, C_K exact in bf16)
//   softmax online per head row; P stays in registers as the A operand of
//   values  u += P C_V    (rank 16 over the LO tokens, rank 64 for HI tokens;
//                          a token with its mask bit set gets logit -inf in LO)
// At the item's end the warp writes the partial (max, sum, u) of each head.
// The unit's q~ (hi and lo planes) travels through the same ring: an item
// begins with kQStages bulk-copied stages that the consumer takes into
// registers.  Every ring slot carries a small descriptor of its stage.
template <int NMB>
__global__ void __launch_bounds__(kThreads, Cfg<NMB>::kBlocks) vis_kernel(const __grid_constant__ Params p) {
    using C = Cfg<NMB>;
    constexpr int kSlots = C::kSlots, kHiTok = C::kHiTok, kNTH = C::kNTH, kHalf = C::kSlotBytes / 2;
    extern __shared__ __align__(1024) unsigned char smem_raw[];
    const uint32_t sbase0 = smem_u32(smem_raw);
    Smem<NMB> &sm = *reinterpret_cast<Smem<NMB> *>(smem_raw + ((1024u - (sbase0 & 1023u)) & 1023u));
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31, tid = threadIdx.x;
    const int g = lane >> 2, tig = lane & 3;
    volatile int *abort = &sm.abort;

    if (tid == 0) {
        for (int w = 0; w < kWarps; ++w)
            for (int s = 0; s < kSlots; ++s) mbar_init(&sm.full[w][s], 32);
        sm.abort = 0;
        asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
    }
    __syncthreads();

    // ------------------------------------------------------------ issue side
    constexpr int kTypeQ = 0, kTypeLo = 1, kTypeHi = 2, kFirst = 4, kLast = 8;
    int i_item = -1, i_unit = 0, i_t0 = 0, i_n = 0;   // the item being issued
    int i_q = 0, i_sub = 0, i_lo = 0, i_hi = 0, i_nhi = 0, i_left = 0;   // i_lo: LO stages still to issue
    uint32_t i_seq = 0, c_seq = 0;
    bool i_done = false;
    auto fetch = [&]() -> int {
        int v = 0;
        if (lane == 0) v = (int)atomicAdd(p.counter, 1u);
        return __shfl_sync(0xffffffffu, v, 0);
    };
    // the next item: its mask words and the list of its full-rank tokens
    auto begin_item = [&]() -> bool {
        const int it = fetch();
        if (it >= p.n_items) return false;
        i_item = it;
        i_unit = it / p.S;
        i_t0 = (it % p.S) * p.tps;
        i_n = min(p.tps, p.T - i_t0);
        const int nw = (i_n + 31) >> 5;
        int base = 0, n_lo_st = 0;
        for (int w0 = 0; w0 < nw; w0 += 32) {
            const int wi = w0 + lane;
            uint32_t w = 0u;
            if (wi < nw) {
                w = __ldg(p.mask + (size_t)i_unit * p.nwords + (i_t0 >> 5) + wi);
                const int nb = i_n - 32 * wi;
                if (nb < 32) w &= (1u << nb) - 1u;
                sm.mw[warp][wi] = w;
            }
            const int c = __popc(w);
            int incl = c;
            #pragma unroll
            for (int d = 1; d < 32; d <<= 1) {
                const int v = __shfl_up_sync(0xffffffffu, incl, d);
                if (lane >= d) incl += v;
            }
            int r = base + incl - c;
            uint32_t bits = w;
            while (bits) {
                sm.hi_list[warp][r++] = (uint16_t)(32 * wi + __ffs(bits) - 1);
                bits &= bits - 1u;
            }
            // sub-chunks (word pairs) with a reduced-rank token need a LO stage
            const int c_pair = c + __shfl_down_sync(0xffffffffu, c, 1);
            const int nsub_tok = min(kSub, i_n - 32 * wi);
            const bool lo_st = (lane & 1) == 0 && wi < nw && c_pair < nsub_tok;
            n_lo_st += __popc(__ballot_sync(0xffffffffu, lo_st));
            base += __shfl_sync(0xffffffffu, incl, 31);
        }
        i_nhi = base;
        i_hi = 0;
        i_sub = 0;
        i_lo = n_lo_st;
        i_q = 0;
        i_left = C::kQStages + n_lo_st + (i_nhi + kHiTok - 1) / kHiTok;
        __syncwarp();
        return true;
    };
    // issue the item's next stage (the item has one)
    auto issue_stage = [&]() {
        const int slot = i_seq % kSlots;
        unsigned char *dst = sm.ring[warp][slot];
        uint64_t *bar = &sm.full[warp][slot];
        int type, n = 0;
        uint32_t w0 = 0u, w1 = 0u;
        __syncwarp();
        if (i_q < C::kQStages) {
            // q~ of the unit: the hi plane (NMB == 1: then the lo plane in the slot's second half),
            // Hg rows of 128 bytes; the consumer zeroes the rows past Hg in registers
            type = kTypeQ | (i_q == 0 ? kFirst : 0);
            n = i_q;
            if (lane == 0) {
                const unsigned char *src = p.qt + (size_t)i_unit * qblock_bytes(p.Hg);
                const uint32_t bytes = (uint32_t)p.Hg * 128u;
                fence_proxy_async();
                if (C::kQStages == 1) {
                    mbar_arrive_tx(bar, 2 * bytes);
                    bulk_g2s(dst, src, bytes, bar);
                    bulk_g2s(dst + kHalf, src + bytes, bytes, bar);
                } else {
                    mbar_arrive_tx(bar, bytes);
                    bulk_g2s(dst, src + (size_t)i_q * bytes, bytes, bar);
                }
            } else {
                mbar_arrive(bar);
            }
            ++i_q;
        } else if (i_lo > 0) {
            // the next sub-chunk with a reduced-rank token (one exists): all 64 rows of K and V (the value MMA reads
            // every row; masked rows get p = 0, which must meet finite data -- neighbouring rows, or zeros
            // past the unit's end)
            while (true) {
                n = min(kSub, i_n - kSub * i_sub);
                w0 = sm.mw[warp][2 * i_sub];
                w1 = n > 32 ? sm.mw[warp][2 * i_sub + 1] : 0u;
                if (__popc(w0) + __popc(w1) < n) break;
                ++i_sub;
            }
            type = kTypeLo;
            const int t0 = i_t0 + kSub * i_sub;
            if (lane == 0) {
                fence_proxy_async();
                mbar_arrive_tx(bar, 4u * 1024u);
                tma_3d(dst, &p.tm_ck, 0, t0, i_unit, bar);
                tma_3d(dst + 1024, &p.tm_ck, 0, t0 + 32, i_unit, bar);
                tma_3d(dst + kHalf, &p.tm_cv, 0, t0, i_unit, bar);
                tma_3d(dst + kHalf + 1024, &p.tm_cv, 0, t0 + 32, i_unit, bar);
            } else {
                mbar_arrive(bar);
            }
            ++i_sub;
            --i_lo;
        } else {
            // kHiTok full-rank tokens: C_lo + C_hi rows of K and V gathered into 128-byte rows
            // (16-byte chunk c of row r stored at c ^ (r & 7)); rows past the count are zero
            type = kTypeHi;
            n = min(kHiTok, i_nhi - i_hi);
            const size_t ubase = (size_t)i_unit * p.T + i_t0;
            #pragma unroll
            for (int i = 0; i < kHiTok / 4; ++i) {
                const int idx = lane + 32 * i;
                const int r = idx >> 3, ch = idx & 7;
                const int pos = (ch ^ (r & 7)) << 4;
                unsigned char *dk = dst + r * 128 + pos;
                unsigned char *dv = dst + kHalf + r * 128 + pos;
                if (r < n) {
                    const size_t row = ubase + sm.hi_list[warp][i_hi + r];
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
            i_hi += n;
        }
        --i_left;
        if (i_left == 0) type |= kLast;
        if (lane == 0) {
            int *d = sm.desc[warp][slot];
            d[0] = type; d[1] = i_item; d[2] = n; d[3] = (int)w0; d[4] = (int)w1;
        }
        __syncwarp();
        ++i_seq;
    };
    // issue while the ring has room
    auto pump = [&]() {
        while (!i_done && i_seq - c_seq < (uint32_t)kSlots) {
            if (i_left == 0 && !begin_item()) {
                i_done = true;
                return;
            }
            issue_stage();
        }
    };
    pump();

    // ---------------------------------------------------------- consumer side
    float m[NMB][2], l[NMB][2], u[NMB][8][4];
    uint32_t qh[NMB][4][4], ql[NMB][4][4];   // q~ hi / lo as A fragments: head block, k-step
    bool ok = true;

    // LO tokens: one softmax update over 8 NT C_lo rows of a stage (NT m16n8 tiles of tokens;
    // n of them inside the unit; mask words w0, w1 cover them)
    auto do_lo = [&](uint32_t sb, uint32_t w0, uint32_t w1, int n, auto ntc) {
        constexpr int NT = decltype(ntc)::value;
        const uint32_t x[2] = {w0 >> (2 * tig), w1 >> (2 * tig)};   // bit 8 (nt & 3) + e: token 8 nt + 2 tig + e
        const bool partial = n < 8 * NT;
        #pragma unroll
        for (int mb = 0; mb < NMB; ++mb) {
            float s[NT][4];
            #pragma unroll
            for (int a = 0; a < NT; ++a) s[a][0] = s[a][1] = s[a][2] = s[a][3] = 0.f;
            #pragma unroll
            for (int np = 0; np < NT / 2; ++np) {
                uint32_t b0, b1, b2, b3;
                const int row = 16 * np + (lane & 7) + ((lane >> 4) << 3);
                const int ch = (lane >> 3) & 1;
                ldsm_x4(sb + row * 32 + ((ch ^ ((row >> 2) & 1)) << 4), b0, b1, b2, b3);
                mma_bf16(s[2 * np], qh[mb][0], b0, b1);
                mma_bf16(s[2 * np + 1], qh[mb][0], b2, b3);
                mma_bf16(s[2 * np], ql[mb][0], b0, b1);
                mma_bf16(s[2 * np + 1], ql[mb][0], b2, b3);
            }
            #pragma unroll
            for (int nt = 0; nt < NT; ++nt)
                #pragma unroll
                for (int e = 0; e < 2; ++e) {
                    const bool hb = (x[nt >> 2] >> (8 * (nt & 3) + e)) & 1u;
                    const bool out = hb || (partial && 8 * nt + 2 * tig + e >= n);
                    if (out) s[nt][e] = s[nt][2 + e] = -INFINITY;
                }
            lazy_update<NT>(s, m[mb], l[mb], u[mb]);
            #pragma unroll
            for (int kk = 0; kk < NT / 2; ++kk) {
                uint32_t a[4];
                a[0] = pack_bf16(s[2 * kk][0], s[2 * kk][1]);
                a[1] = pack_bf16(s[2 * kk][2], s[2 * kk][3]);
                a[2] = pack_bf16(s[2 * kk + 1][0], s[2 * kk + 1][1]);
                a[3] = pack_bf16(s[2 * kk + 1][2], s[2 * kk + 1][3]);
                uint32_t b0, b1, b2, b3;
                const int row = 16 * kk + (lane & 7) + (((lane >> 3) & 1) << 3);
                const int ch = lane >> 4;
                ldsm_x4_t(sb + kHalf + row * 32 + ((ch ^ ((row >> 2) & 1)) << 4), b0, b1, b2, b3);
                mma_bf16(u[mb][0], a, b0, b1);
                mma_bf16(u[mb][1], a, b2, b3);
            }
        }
    };

    // kHiTok full-rank tokens (n of them valid)
    auto do_hi = [&](uint32_t sb, int n) {
        #pragma unroll
        for (int mb = 0; mb < NMB; ++mb) {
            float s[kNTH][4];
            #pragma unroll
            for (int a = 0; a < kNTH; ++a) s[a][0] = s[a][1] = s[a][2] = s[a][3] = 0.f;
            #pragma unroll
            for (int kb = 0; kb < 4; ++kb) {
                #pragma unroll
                for (int np = 0; np < kNTH / 2; ++np) {
                    uint32_t b0, b1, b2, b3;
                    const int row = 16 * np + (lane & 7) + ((lane >> 4) << 3);
                    const int ch = 2 * kb + ((lane >> 3) & 1);
                    ldsm_x4(sb + row * 128 + ((ch ^ (row & 7)) << 4), b0, b1, b2, b3);
                    mma_bf16(s[2 * np], qh[mb][kb], b0, b1);
                    mma_bf16(s[2 * np + 1], qh[mb][kb], b2, b3);
                    mma_bf16(s[2 * np], ql[mb][kb], b0, b1);
                    mma_bf16(s[2 * np + 1], ql[mb][kb], b2, b3);
                }
            }
            if (n < kHiTok) {
                #pragma unroll
                for (int nt = 0; nt < kNTH; ++nt)
                    #pragma unroll
                    for (int e = 0; e < 2; ++e)
                        if (8 * nt + 2 * tig + e >= n) s[nt][e] = s[nt][2 + e] = -INFINITY;
            }
            lazy_update<kNTH>(s, m[mb], l[mb], u[mb]);
            #pragma unroll
            for (int kk = 0; kk < kNTH / 2; ++kk) {
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
                    ldsm_x4_t(sb + kHalf + row * 128 + ((ch ^ (row & 7)) << 4), b0, b1, b2, b3);
                    mma_bf16(u[mb][2 * pr], a, b0, b1);
                    mma_bf16(u[mb][2 * pr + 1], a, b2, b3);
                }
            }
        }
    };

    // a q~ plane (kRows rows of 128 bytes, chunk c of row r at c ^ (r & 7)) into A fragments;
    // rows past Hg hold stale bytes and are zeroed here
    auto load_plane = [&](uint32_t base, uint32_t (&q)[NMB][4][4]) {
        #pragma unroll
        for (int mb = 0; mb < NMB; ++mb) {
            const int row = 16 * mb + (lane & 7) + (((lane >> 3) & 1) << 3);
            const bool z0 = 16 * mb + g >= p.Hg, z1 = 16 * mb + g + 8 >= p.Hg;
            #pragma unroll
            for (int kb = 0; kb < 4; ++kb) {
                const int ch = 2 * kb + (lane >> 4);
                ldsm_x4(base + row * 128 + ((ch ^ (row & 7)) << 4), q[mb][kb][0], q[mb][kb][1], q[mb][kb][2], q[mb][kb][3]);
                if (z0) q[mb][kb][0] = q[mb][kb][2] = 0u;
                if (z1) q[mb][kb][1] = q[mb][kb][3] = 0u;
            }
        }
    };

    while (ok) {
        pump();
        if (c_seq == i_seq) break;   // nothing in flight, nothing left to issue
        const int slot = c_seq % kSlots;
        if (!mbar_wait(&sm.full[warp][slot], (c_seq / kSlots) & 1u, abort)) { ok = false; break; }
        const int *dsc = sm.desc[warp][slot];
        const int type = dsc[0], item = dsc[1], n = dsc[2];
        const uint32_t sb = smem_u32(sm.ring[warp][slot]);
        if ((type & 3) == kTypeQ) {
            if (type & kFirst) {   // a new item: fresh softmax state
                #pragma unroll
                for (int mb = 0; mb < NMB; ++mb) {
                    m[mb][0] = m[mb][1] = kRefInit;
                    l[mb][0] = l[mb][1] = 0.f;
                    #pragma unroll
                    for (int a = 0; a < 8; ++a) u[mb][a][0] = u[mb][a][1] = u[mb][a][2] = u[mb][a][3] = 0.f;
                }
            }
            if (C::kQStages == 1) {
                load_plane(sb, qh);
                load_plane(sb + kHalf, ql);
            } else if (n == 0) {
                load_plane(sb, qh);
            } else {
                load_plane(sb, ql);
            }
        } else if ((type & 3) == kTypeLo) {
            const uint32_t w0 = (uint32_t)dsc[3], w1 = (uint32_t)dsc[4];
            if (NMB == 1) {   // two 32-token halves: fewer live scores
                do_lo(sb, w0, 0u, n, std::integral_constant<int, 4>{});
                if (n > 32) do_lo(sb + 1024, w1, 0u, n - 32, std::integral_constant<int, 4>{});
            } else {
                do_lo(sb, w0, w1, n, std::integral_constant<int, 8>{});
            }
        } else {
            do_hi(sb, n);
        }
        if (type & kLast) {
            // the item's partial -- per head row: max, sum, u[64]
            float *dst = p.part + (size_t)item * p.Hg * kVisPart;
            #pragma unroll
            for (int mb = 0; mb < NMB; ++mb)
                #pragma unroll
                for (int r = 0; r < 2; ++r) {
                    float lt = l[mb][r];
                    lt += __shfl_xor_sync(0xffffffffu, lt, 1);
                    lt += __shfl_xor_sync(0xffffffffu, lt, 2);
                    const int h = 16 * mb + g + 8 * r;
                    if (h < p.Hg) {
                        float *row = dst + (size_t)h * kVisPart;
                        if (tig == 0) *reinterpret_cast<float2 *>(row) = make_float2(m[mb][r], lt);
                        #pragma unroll
                        for (int nt = 0; nt < 8; ++nt)
                            *reinterpret_cast<float2 *>(row + 2 + 8 * nt + 2 * tig) =
                                make_float2(u[mb][nt][2 * r], u[mb][nt][2 * r + 1]);
                    }
                }
        }
        ++c_seq;
        __syncwarp();
    }
    if (!ok) *abort = 1;
    // copies still in flight (only after an abort) must land before the block exits
    while (c_seq < i_seq) {
        const int slot = c_seq % kSlots;
        const uint32_t par = (c_seq / kSlots) & 1u;
        const long long t0 = clock64();
        while (!mbar_try_wait(&sm.full[warp][slot], par) && clock64() - t0 < kWaitCycles) {}
        ++c_seq;
    }
    cp_async_wait_all();
}

}  // namespace vis

// ======================================================================= finish

struct FinishParams {
    const uint16_t *BV;       // [units][64][512]
    const float *vpart;       // [units][S][Hg][kVisPart]
    const float *tpart;       // [units][Sc][Hg][kTxtPart] or null
    uint16_t *out;            // [(layer, batch)][n_q][128]
    float *ustat;             // [units][Hg][2]: the unit-wide (max, 1/sum) per head, or null
    int Hg, per_kv, n_q, groups, S, Sc;
};

// dynamic shared memory of finish_kernel: the weight of every partial, then u / l and w / l
__host__ __device__ constexpr size_t finish_smem_bytes(int S, int Sc, int Hg) {
    return ((size_t)(S + Sc) * Hg + (size_t)Hg * (64 + 128)) * sizeof(float);
}
constexpr size_t kFinishSmemMax = 200 * 1024;

// One block per unit.  When the unit has many partials, thread 0 first asks
// for the unit's B_V (64 KB) to be brought into L2, so that it streams from
// DRAM while the partials are combined.  Per head, the unit-wide max M and sum L over every visual and text
// partial give each partial the weight 2^(m - M) / L; u / l and w / l are
// weighted sums with the feature index across threads (coalesced).  Then
// o_h = (u_h / l_h) B_V[:, 128 j(h) ..] + w_h / l_h, thread t owning output
// columns 2t, 2t+1 of the unit's 512 (KV head t / 64).
// PK = query heads per KV head (the projection's inner loop is unrolled over exactly PK heads).
template <int PK>
__global__ void __launch_bounds__(256) finish_kernel(const FinishParams p) {
    extern __shared__ float fsm[];
    float *wv = fsm;                              // [S][Hg]
    float *wt = wv + (size_t)p.S * p.Hg;          // [Sc][Hg]
    float *uf = wt + (size_t)p.Sc * p.Hg;         // [Hg][64]
    float *wf = uf + (size_t)p.Hg * 64;           // [Hg][128]
    const int unit = blockIdx.x, tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const float *vp0 = p.vpart + (size_t)unit * p.S * p.Hg * kVisPart;
    const float *tp0 = p.tpart + (size_t)unit * p.Sc * p.Hg * kTxtPart;
    const uint16_t *bvg = p.BV + (size_t)unit * 64 * 512;
    if (tid == 0 && p.S + p.Sc > 8) bulk_prefetch_l2(bvg, 64 * 512 * 2);   // long combine: overlap B_V

    for (int h = warp; h < p.Hg; h += 8) {
        float mx = -INFINITY;
        for (int s = lane; s < p.S; s += 32) mx = fmaxf(mx, __ldcg(vp0 + ((size_t)s * p.Hg + h) * kVisPart));
        for (int c = lane; c < p.Sc; c += 32) mx = fmaxf(mx, __ldcg(tp0 + ((size_t)c * p.Hg + h) * kTxtPart));
        #pragma unroll
        for (int d = 16; d > 0; d >>= 1) mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, d));
        float sum = 0.f;
        for (int s = lane; s < p.S; s += 32) {
            const float *r = vp0 + ((size_t)s * p.Hg + h) * kVisPart;
            const float e = ex2(__ldcg(r) - mx);
            wv[s * p.Hg + h] = e;
            sum += __ldcg(r + 1) * e;
        }
        for (int c = lane; c < p.Sc; c += 32) {
            const float *r = tp0 + ((size_t)c * p.Hg + h) * kTxtPart;
            const float m = __ldcg(r);
            const float e = (m != -INFINITY) ? ex2(m - mx) : 0.f;
            wt[c * p.Hg + h] = e;
            sum += (m != -INFINITY) ? __ldcg(r + 1) * e : 0.f;
        }
        #pragma unroll
        for (int d = 16; d > 0; d >>= 1) sum += __shfl_xor_sync(0xffffffffu, sum, d);
        const float inv = 1.f / sum;
        if (lane == 0 && p.ustat != nullptr)
            *reinterpret_cast<float2 *>(p.ustat + ((size_t)unit * p.Hg + h) * 2) = make_float2(mx, inv);
        __syncwarp();
        for (int s = lane; s < p.S; s += 32) wv[s * p.Hg + h] *= inv;
        for (int c = lane; c < p.Sc; c += 32) wt[c * p.Hg + h] *= inv;
    }
    __syncthreads();
    // weighted sums: thread tid takes the tasks tid, tid + 256, ... K at a time (K = the tasks per
    // thread, up to 4), so that the partial loads of K sums are in flight together
    auto combine_k = [&](auto kc, const float *base, int row, int n_task, int npart, const float *wgt, float *dst,
                         int shift) {
        constexpr int K = decltype(kc)::value;
        const size_t st = (size_t)p.Hg * row;
        for (int t0 = tid; t0 < n_task; t0 += K * 256) {
            const float *r[K];
            int hk[K];
            bool ok[K];
            #pragma unroll
            for (int k = 0; k < K; ++k) {
                const int task = t0 + 256 * k;
                ok[k] = task < n_task;
                hk[k] = ok[k] ? task >> shift : 0;
                r[k] = base + (size_t)hk[k] * row + 2 + (ok[k] ? (task & ((1 << shift) - 1)) : 0);
            }
            float acc[K];
            #pragma unroll
            for (int k = 0; k < K; ++k) acc[k] = 0.f;
            for (int s2 = 0; s2 < npart; ++s2) {
                #pragma unroll
                for (int k = 0; k < K; ++k)
                    if (ok[k]) acc[k] = fmaf(__ldcg(r[k] + s2 * st), wgt[s2 * p.Hg + hk[k]], acc[k]);
            }
            #pragma unroll
            for (int k = 0; k < K; ++k)
                if (ok[k]) dst[t0 + 256 * k] = acc[k];
        }
    };
    auto combine = [&](const float *base, int row, int n_task, int npart, const float *wgt, float *dst, int shift) {
        const int per = (n_task + 255) / 256;
        if (per <= 1) combine_k(std::integral_constant<int, 1>(), base, row, n_task, npart, wgt, dst, shift);
        else if (per == 2) combine_k(std::integral_constant<int, 2>(), base, row, n_task, npart, wgt, dst, shift);
        else combine_k(std::integral_constant<int, 4>(), base, row, n_task, npart, wgt, dst, shift);
    };
    combine(vp0, kVisPart, p.Hg * 64, p.S, wv, uf, 6);
    combine(tp0, kTxtPart, p.Hg * 128, p.Sc, wt, wf, 7);
    __syncthreads();
    const int j = tid >> 6, d = (2 * tid) & 127;
    const int lb = unit / p.groups, G = unit % p.groups;
    const uint32_t *bv = reinterpret_cast<const uint32_t *>(bvg) + tid;
    float acc[PK][2];
    #pragma unroll
    for (int hh = 0; hh < PK; ++hh) acc[hh][0] = acc[hh][1] = 0.f;
    const int h0 = j * PK;
    #pragma unroll 4
    for (int i0 = 0; i0 < 64; i0 += 16) {
        uint32_t braw[16];
        #pragma unroll
        for (int i = 0; i < 16; ++i) braw[i] = __ldcs(bv + (i0 + i) * 256);
        #pragma unroll
        for (int i = 0; i < 16; ++i) {
            const float b0 = __uint_as_float(braw[i] << 16), b1 = __uint_as_float(braw[i] & 0xffff0000u);
            #pragma unroll
            for (int hh = 0; hh < PK; ++hh) {
                const float x = uf[(h0 + hh) * 64 + i0 + i];
                acc[hh][0] = fmaf(x, b0, acc[hh][0]);
                acc[hh][1] = fmaf(x, b1, acc[hh][1]);
            }
        }
    }
    #pragma unroll
    for (int hh = 0; hh < PK; ++hh) {
        const int h = h0 + hh;
        *reinterpret_cast<uint32_t *>(p.out + ((size_t)lb * p.n_q + (size_t)G * p.Hg + h) * 128 + d) =
            pack_bf16(acc[hh][0] + wf[h * 128 + d], acc[hh][1] + wf[h * 128 + d + 1]);
    }
}

static_assert(2 * (vis::smem_bytes<1>() + 1024) <= 233472, "visual kernel (16 head rows): two blocks per SM");
static_assert(vis::smem_bytes<2>() <= 232448, "visual kernel (32 head rows) shared memory");
static_assert(text::smem_bytes() <= 232448, "text kernel shared memory");
}  // namespace decode
}  // namespace kvpack
