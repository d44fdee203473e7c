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
//   text_kernel    q~ = scale * log2(e) * B_K[:, 128 j(h) ..] q_h per (unit, KV head), split into
//                  bf16 hi + lo; and the text tail (plain bf16 K/V) per (unit, KV head, chunk of
//                  tokens): partial (max, sum, w = sum p V) per query head
//   text_stats     the text tail's (max, sum) per head folded over its chunks, one warp per unit
//   vis_kernel     the compressed visual tokens per (unit, split of tokens): partial
//                  (max, sum, u = sum p C_V) per query head, then -- once every split
//                  of the unit has published -- the attention mass of each token
//   finish_kernel  combines the partials of a unit and projects: o_h = (u B_V + w) / l
// Logits are kept in the log2 domain (the scale folds log2(e)).
#pragma once

#include <cuda.h>

#include <type_traits>

#include "common.cuh"

namespace kvpack {
namespace decode {

constexpr int kMaxHeads = 32;
constexpr int kTxtPart = 130;   // per (unit, text chunk, head): max, sum, w[128]
constexpr int kVisPart = 66;    // per (unit, visual split, head): max, sum, u[64]

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
constexpr int kMeta = 4;            // item metadata ring (the issue side runs up to two items ahead)

// Geometry per head-block count.  Up to 16 query heads per unit: two blocks per
// SM (their serial phases overlap), 4 KB ring slots.  Up to 32: one block per SM.
template <int NMB>
struct Cfg {
    static constexpr int kRows = 16 * NMB;                      // query-head rows (padded)
    static constexpr int kBlocks = (NMB == 1) ? 2 : 1;          // resident blocks per SM
    static constexpr int kSlots = 2;                            // ring slots per warp
    static constexpr int kSlotBytes = (NMB == 1) ? 4096 : 8192; // K rows in the first half, V in the second
    static constexpr int kHiTok = (NMB == 1) ? 16 : 32;         // full-rank tokens per HI stage
    static constexpr int kNTH = kHiTok / 8;                     // m16n8 token tiles per HI stage
    static constexpr int kLoTok = 64;                           // visual tokens per warp per item
    static constexpr int kItemTok = kWarps * kLoTok;            // tokens per item
    static constexpr int kHiMax = kLoTok / kHiTok;              // HI stages per warp per item, at most
    static constexpr int kUpd = 1 + kHiMax;                     // softmax updates per warp per item, at most
    // tensor-memory columns of one warp's stash of one item: LO p (32 per head block), then HI p
    static constexpr int kBufCols = 32 * NMB + 4 * kNTH * NMB * kHiMax;
    static constexpr int kTmemCols = 4 * kBufCols;              // two warps per lane quarter, two items each
    static_assert(kHiTok * 128 == kSlotBytes / 2, "HI stage rows fill half a slot");
    static_assert(kLoTok * 32 <= kSlotBytes / 2, "LO stage rows fit half a slot");
};

struct Params {
    CUtensorMap tm_ck, tm_cv;   // C_lo planes: 3D {16, T, units}, box {16, 32, 1}, 32-byte swizzle
    const uint16_t *CK_lo, *CK_hi, *CV_lo, *CV_hi;
    const unsigned char *qt;    // [units][qblock_bytes(Hg)] from text_kernel and text_stats_kernel
    const uint32_t *mask;       // [units][nwords]
    float *mass;                // [units][T] or null
    float *part;                // [units][S][Hg][kVisPart]
    float *ustat;               // [units][Hg][2]: unit-wide (max, 1/sum); NaN at launch (S > 1)
    unsigned int *arrive;       // [units], zero at launch
    int n_units, T, Hg, S, tps, nwords, n_items;
};

template <int NMB>
struct Smem {
    using C = Cfg<NMB>;
    alignas(1024) unsigned char ring[kWarps][C::kSlots][C::kSlotBytes];
    alignas(128) uint16_t qt[2][C::kRows][64];              // q~ hi / lo of the current item
    alignas(16) float tst[C::kRows][2];                      // text (max, sum) of the current item's unit
    float tcur[C::kRows][2];                                 // the same, kept through the epilogue
    float ubuf[4][16][64];                                   // merge staging: 4 warps x one 16-row block of u
    float wm[kWarps][C::kRows], wl[kWarps][C::kRows];
    float mcta[C::kRows], lcta[C::kRows], mfin[C::kRows], invl[C::kRows];
    float mref[2][kWarps][C::kUpd][C::kRows];               // reference max of each stashed update
    float upf[C::kRows][2];                                  // prefetched unit (max, 1/sum) of the previous item
    uint16_t hi_list[kMeta][kWarps][C::kLoTok];             // this warp's full-rank tokens (item-relative)
    int meta[kMeta][kWarps][12];                            // lo0, n_lo, n_hi, item, 4 mask words of the LO range, unit, t0
    uint64_t full[kWarps][C::kSlots];
    uint64_t qbar;
    uint32_t tmem_base;
    int abort;
    int last;
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

// 4 values -> lanes with bit 2 clear hold the total of slot 2 b4 + b3 (the
// lanes with bit 2 set hold the same totals)
__device__ __forceinline__ float reduce_scatter4(const float (&x)[4], int lane) {
    float t2[2];
    const bool b4 = lane & 16, b3 = lane & 8;
    #pragma unroll
    for (int i = 0; i < 2; ++i) {
        const float send = b4 ? x[i] : x[2 + i];
        t2[i] = (b4 ? x[2 + i] : x[i]) + __shfl_xor_sync(0xffffffffu, send, 16);
    }
    const float send = b3 ? t2[0] : t2[1];
    const float t = (b3 ? t2[1] : t2[0]) + __shfl_xor_sync(0xffffffffu, send, 8);
    return t + __shfl_xor_sync(0xffffffffu, t, 4);
}

// Persistent, one or two 256-thread blocks per SM, a static round-robin over items
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
        mbar_init(&sm.qbar, 1);
        sm.abort = 0;
        asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
    }
    for (int i = tid; i < 2 * C::kRows * 64; i += kThreads) (&sm.qt[0][0][0])[i] = 0;
    if (warp == 0) tmem_alloc(&sm.tmem_base, C::kTmemCols);
    tmem_fence_before();
    __syncthreads();
    tmem_fence_after();
    const uint32_t tmem = sm.tmem_base + ((uint32_t)(32 * (warp & 3)) << 16) + (uint32_t)(2 * C::kBufCols * (warp >> 2));

    auto item_of = [&](int K) { return (int)blockIdx.x + K * (int)gridDim.x; };
    auto issue_q = [&](int K) {   // query block of item K's unit into sm.qt / sm.tst (one thread)
        const unsigned char *src = p.qt + (size_t)(item_of(K) / p.S) * qblock_bytes(p.Hg);
        const uint32_t bytes = (uint32_t)p.Hg * 128u;
        fence_proxy_async();
        mbar_arrive_tx(&sm.qbar, (uint32_t)qblock_bytes(p.Hg));
        bulk_g2s(&sm.qt[0][0][0], src, bytes, &sm.qbar);
        bulk_g2s(&sm.qt[1][0][0], src + bytes, bytes, &sm.qbar);
        bulk_g2s(&sm.tst[0][0], src + 2 * bytes, (uint32_t)p.Hg * 8u, &sm.qbar);
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
            sm.meta[ms][warp][8] = item / p.S;
            sm.meta[ms][warp][9] = t0;
        }
        __syncwarp();
        i_nst = (n_lo > 0 ? 1 : 0) + (h1 - h0 + kHiTok - 1) / kHiTok;
        i_st = 0;
        return true;
    };

    auto issue_stage = [&]() {
        const int ms = iK % kMeta;
        const int lo0 = sm.meta[ms][warp][0], n_lo = sm.meta[ms][warp][1], nh = sm.meta[ms][warp][2];
        const int unit = sm.meta[ms][warp][8], t0 = sm.meta[ms][warp][9];
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
                    tma_3d(dst + kHalf + 1024 * b, &p.tm_cv, 0, t0 + lo0 + 32 * b, unit, bar);
                }
            } else {
                mbar_arrive(bar);
            }
        } else {
            // 32 full-rank tokens: C_lo + C_hi rows of K and V gathered into 128-byte rows
            // (16-byte chunk c of row r stored at c ^ (r & 7)); rows past the count are zero
            const int hs = i_st - (n_lo > 0 ? 1 : 0);
            const int cnt = min(kHiTok, nh - kHiTok * hs);
            const size_t ubase = (size_t)unit * p.T + t0;
            #pragma unroll
            for (int i = 0; i < kHiTok / 4; ++i) {
                const int idx = lane + 32 * i;
                const int r = idx >> 3, ch = idx & 7;
                const int pos = (ch ^ (r & 7)) << 4;
                unsigned char *dk = dst + r * 128 + pos;
                unsigned char *dv = dst + kHalf + r * 128 + pos;
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

    // Attention mass of this warp's tokens of item K (meta slot K % kMeta, stash
    // buffer K & 1), one warp alone.  The unit's (max, 1/sum) per head come from
    // shared memory (single-split units) or from ustat, polled until the unit's
    // last split has written them.
    auto mass_warp = [&](int K, int src) {
        const int item = item_of(K);
        const int unit = item / p.S;
        float Mr[NMB][2], IL[NMB][2];
        bool ready = true;
        #pragma unroll
        for (int mb = 0; mb < NMB; ++mb)
            #pragma unroll
            for (int r = 0; r < 2; ++r) {
                const int row = 16 * mb + g + 8 * r;
                const bool ok = row < p.Hg;
                Mr[mb][r] = ok ? (src == 0 ? sm.mfin[row] : sm.upf[row][0]) : 0.f;
                IL[mb][r] = ok ? (src == 0 ? sm.invl[row] : sm.upf[row][1]) : 0.f;
                ready = ready && !(Mr[mb][r] != Mr[mb][r]) && !(IL[mb][r] != IL[mb][r]);
            }
        if (src == 1 || (src == 2 && !__all_sync(0xffffffffu, ready))) {
            const long long start = clock64();
            while (true) {
                ready = true;
                #pragma unroll
                for (int mb = 0; mb < NMB; ++mb)
                    #pragma unroll
                    for (int r = 0; r < 2; ++r) {
                        const int row = 16 * mb + g + 8 * r;
                        float a = 0.f, b2 = 0.f;
                        if (row < p.Hg) {
                            const float *us = p.ustat + ((size_t)unit * p.Hg + row) * 2;
                            asm volatile("ld.relaxed.gpu.global.v2.f32 {%0, %1}, [%2];" : "=f"(a), "=f"(b2) : "l"(us) : "memory");
                        }
                        Mr[mb][r] = a;
                        IL[mb][r] = b2;
                        ready = ready && !(a != a) && !(b2 != b2);
                    }
                if (__all_sync(0xffffffffu, ready)) break;
                if (*abort) return;
                if (clock64() - start > kWaitCycles) {
                    report_error(KVPACK_ERR_TIMEOUT);
                    *abort = 1;
                    return;
                }
                __nanosleep(100);
            }
        }
        const int ms = K % kMeta, b = K & 1;
        const int lo0 = sm.meta[ms][warp][0], n_lo = sm.meta[ms][warp][1], nh = sm.meta[ms][warp][2];
        const int t0 = (item % p.S) * p.tps;
        float *mrow = p.mass + (size_t)unit * p.T + t0;
        auto fac = [&](int upd, int mb, int r) -> float {
            const int row = 16 * mb + g + 8 * r;
            return row < p.Hg ? ex2(sm.mref[b][warp][upd][row] - Mr[mb][r]) * IL[mb][r] : 0.f;
        };
        tmem_fence_after();
        // LO range (64 tokens)
        const uint32_t bcol = (uint32_t)(C::kBufCols * b);
        if (n_lo > 0) {
            float acc[16];
            #pragma unroll
            for (int i = 0; i < 16; ++i) acc[i] = 0.f;
            #pragma unroll
            for (int mb = 0; mb < NMB; ++mb) {
                float v0[16], v1[16];
                const uint32_t col = bcol + (uint32_t)(32 * mb);
                tmem_ld16(tmem + col, v0);
                tmem_ld16(tmem + col + 16, v1);
                tmem_wait_ld();
                const float f0 = fac(0, mb, 0), f1 = fac(0, mb, 1);
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
                const int r = 8 * nt + 2 * tig + e;
                const bool hb = ((uint32_t)sm.meta[ms][warp][4 + (r >> 5)] >> (r & 31)) & 1u;
                if (r < n_lo && !hb) mrow[lo0 + r] = out[e];
            }
        }
        // full-rank tokens
        for (int hs = 0; hs * kHiTok < nh; ++hs) {
            const int n = min(kHiTok, nh - kHiTok * hs);
            float acc[2 * kNTH];
            #pragma unroll
            for (int i = 0; i < 2 * kNTH; ++i) acc[i] = 0.f;
            const int upd = 1 + hs;
            #pragma unroll
            for (int mb = 0; mb < NMB; ++mb) {
                float v[16];
                const uint32_t col = bcol + (uint32_t)(32 * NMB + (hs * NMB + mb) * 4 * kNTH);
                if (kNTH == 4) {
                    tmem_ld16(tmem + col, v);
                } else {
                    float v8[8];
                    tmem_ld8(tmem + col, v8);
                    #pragma unroll
                    for (int i = 0; i < 8; ++i) v[i] = v8[i];
                }
                tmem_wait_ld();
                const float f0 = fac(upd, mb, 0), f1 = fac(upd, mb, 1);
                #pragma unroll
                for (int nt = 0; nt < kNTH; ++nt)
                    #pragma unroll
                    for (int e = 0; e < 2; ++e) acc[2 * nt + e] += v[4 * nt + e] * f0 + v[4 * nt + 2 + e] * f1;
            }
            int j;
            float val;
            if (kNTH == 4) {
                float a8[8];
                #pragma unroll
                for (int i = 0; i < 8; ++i) a8[i] = acc[i];
                val = reduce_scatter8(a8, lane);
                j = 4 * ((lane >> 4) & 1) + 2 * ((lane >> 3) & 1) + ((lane >> 2) & 1);
            } else {
                float a4[4];
                #pragma unroll
                for (int i = 0; i < 4; ++i) a4[i] = acc[i];
                val = reduce_scatter4(a4, lane);
                j = ((lane >> 4) & 1) * 2 + ((lane >> 3) & 1);
            }
            const int colt = 8 * (j >> 1) + 2 * tig + (j & 1);
            const bool writer = kNTH == 4 || ((lane >> 2) & 1) == 0;
            if (writer && colt < n) mrow[sm.hi_list[ms][warp][kHiTok * hs + colt]] = val;
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
            m[mb][0] = m[mb][1] = kRefInit;
            l[mb][0] = l[mb][1] = 0.f;
            #pragma unroll
            for (int a = 0; a < 8; ++a) u[mb][a][0] = u[mb][a][1] = u[mb][a][2] = u[mb][a][3] = 0.f;
        }
        const uint32_t tcol = tmem + (uint32_t)(C::kBufCols * b);
        const int nst = (n_lo > 0 ? 1 : 0) + (nh + kHiTok - 1) / kHiTok;

        // LO range: one softmax update over all of this warp's C_lo rows (NT m16n8 tiles of tokens)
        auto do_lo = [&](uint32_t sb, auto ntc) {
            constexpr int NT = decltype(ntc)::value;
            uint32_t x[NT / 4];   // mask words shifted so that bit 8 (nt & 3) + e is token 8 nt + 2 tig + e
            #pragma unroll
            for (int w4 = 0; w4 < NT / 4; ++w4) x[w4] = lw[w4] >> (2 * tig);
            const bool partial = n_lo < 8 * NT;
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
                    mma_bf16(s[2 * np], qah[mb], b0, b1);
                    mma_bf16(s[2 * np + 1], qah[mb], b2, b3);
                    mma_bf16(s[2 * np], qal[mb], b0, b1);
                    mma_bf16(s[2 * np + 1], qal[mb], b2, b3);
                }
                #pragma unroll
                for (int nt = 0; nt < NT; ++nt)
                    #pragma unroll
                    for (int e = 0; e < 2; ++e) {
                        const bool hb = (x[nt >> 2] >> (8 * (nt & 3) + e)) & 1u;
                        const bool out = hb || (partial && 8 * nt + 2 * tig + e >= n_lo);
                        if (out) s[nt][e] = s[nt][2 + e] = -INFINITY;
                    }
                lazy_update<NT>(s, m[mb], l[mb], u[mb]);
                if (p.mass != nullptr) {
                    if (tig == 0) {
                        sm.mref[b][warp][0][16 * mb + g] = m[mb][0];
                        sm.mref[b][warp][0][16 * mb + g + 8] = m[mb][1];
                    }
                    #pragma unroll
                    for (int c4 = 0; c4 < NT / 4; ++c4) {
                        float v[16];
                        #pragma unroll
                        for (int i = 0; i < 16; ++i) v[i] = s[4 * c4 + (i >> 2)][i & 3];
                        tmem_st16(tcol + (uint32_t)(32 * mb + 16 * c4), v);
                    }
                }
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

        for (int st = 0; st < nst && ok; ++st) {
            const int slot = c_seq % kSlots;
            if (!mbar_wait(&sm.full[warp][slot], (c_seq / kSlots) & 1u, abort)) { ok = false; break; }
            const uint32_t sb = smem_u32(sm.ring[warp][slot]);
            if (st == 0 && n_lo > 0) {
                do_lo(sb, std::integral_constant<int, 8>{});
            } else {
                // ------------------------------------------------ HI stage: kHiTok full-rank tokens
                const int hs = st - (n_lo > 0 ? 1 : 0);
                const int n = min(kHiTok, nh - kHiTok * hs);
                const int upd = 1 + hs;
                #pragma unroll
                for (int mb = 0; mb < NMB; ++mb) {
                    float s[kNTH][4];
                    #pragma unroll
                    for (int a = 0; a < kNTH; ++a) s[a][0] = s[a][1] = s[a][2] = s[a][3] = 0.f;
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
                        for (int np = 0; np < kNTH / 2; ++np) {
                            uint32_t b0, b1, b2, b3;
                            const int row = 16 * np + (lane & 7) + ((lane >> 4) << 3);
                            const int ch = 2 * kb + ((lane >> 3) & 1);
                            ldsm_x4(sb + row * 128 + ((ch ^ (row & 7)) << 4), b0, b1, b2, b3);
                            mma_bf16(s[2 * np], ah, b0, b1);
                            mma_bf16(s[2 * np + 1], ah, b2, b3);
                            mma_bf16(s[2 * np], al, b0, b1);
                            mma_bf16(s[2 * np + 1], al, b2, b3);
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
                    if (p.mass != nullptr) {
                        if (tig == 0) {
                            sm.mref[b][warp][upd][16 * mb + g] = m[mb][0];
                            sm.mref[b][warp][upd][16 * mb + g + 8] = m[mb][1];
                        }
                        const uint32_t col = tcol + (uint32_t)(32 * NMB + (hs * NMB + mb) * 4 * kNTH);
                        if (kNTH == 4) {
                            float v0[16];
                            #pragma unroll
                            for (int i = 0; i < 16; ++i) v0[i] = s[(i >> 2) % kNTH][i & 3];
                            tmem_st16(col, v0);
                        } else {
                            float v0[8];
                            #pragma unroll
                            for (int i = 0; i < 8; ++i) v0[i] = s[(i >> 2) % kNTH][i & 3];
                            tmem_st8(col, v0);
                        }
                    }
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
        if (tid < C::kRows) {   // the next item's query block lands in sm.tst after the barrier
            sm.tcur[tid][0] = tid < p.Hg ? sm.tst[tid][0] : -INFINITY;
            sm.tcur[tid][1] = tid < p.Hg ? sm.tst[tid][1] : 0.f;
        }
        // the previous item's unit (max, 1/sum), read now and stored after the merge
        float pf0 = 0.f, pf1 = 0.f;
        const bool prefetch = p.mass != nullptr && p.S > 1 && K >= 1 && tid < p.Hg;
        if (prefetch) {
            const float *us = p.ustat + ((size_t)(item_of(K - 1) / p.S) * p.Hg + tid) * 2;
            asm volatile("ld.relaxed.gpu.global.v2.f32 {%0, %1}, [%2];" : "=f"(pf0), "=f"(pf1) : "l"(us) : "memory");
        }
        tmem_fence_before();
        __syncthreads();
        if (*abort) break;
        if (tid == 0 && item_of(K + 1) < p.n_items) issue_q(K + 1);
        if (tid < C::kRows) {
            float mx = sm.wm[0][tid];
            #pragma unroll
            for (int w = 1; w < kWarps; ++w) mx = fmaxf(mx, sm.wm[w][tid]);
            float sum = 0.f;
            #pragma unroll
            for (int w = 0; w < kWarps; ++w) sum += sm.wl[w][tid] * ex2(sm.wm[w][tid] - mx);
            sm.mcta[tid] = mx;
            sm.lcta[tid] = sum;
            if (p.S == 1) {   // the unit's max and sum: this block's visual part and the text tail
                const float t0m = sm.tcur[tid][0];
                const float M = fmaxf(mx, t0m);
                float L = sum * ex2(mx - M);
                if (t0m != -INFINITY) L += sm.tcur[tid][1] * ex2(t0m - M);
                sm.mfin[tid] = M;
                sm.invl[tid] = 1.f / L;
            }
        }
        // every thread rescales its u rows to the block reference (the max of the warps' references)
        #pragma unroll
        for (int mb = 0; mb < NMB; ++mb)
            #pragma unroll
            for (int r = 0; r < 2; ++r) {
                const int row = 16 * mb + g + 8 * r;
                float mc = sm.wm[0][row];
                #pragma unroll
                for (int w = 1; w < kWarps; ++w) mc = fmaxf(mc, sm.wm[w][row]);
                const float f = row < p.Hg ? ex2(m[mb][r] - mc) : 0.f;
                #pragma unroll
                for (int nt = 0; nt < 8; ++nt) {
                    u[mb][nt][2 * r] *= f;
                    u[mb][nt][2 * r + 1] *= f;
                }
            }
        // sum over the 8 warps, one 16-row block at a time: warps 4-7 hand their u to warps
        // 0-3, which hand the pair sums on; every thread then adds the four for 4 outputs
        {
            float *dst = p.part + ((size_t)unit * p.S + split) * p.Hg * kVisPart;
            #pragma unroll
            for (int mb = 0; mb < NMB; ++mb) {
                float *ub = &sm.ubuf[warp & 3][0][0];
                if (mb > 0) __syncthreads();   // the previous block's sums have been read
                if (warp >= 4) {
                    #pragma unroll
                    for (int nt = 0; nt < 8; ++nt)
                        *reinterpret_cast<float4 *>(ub + 4 * (32 * nt + lane)) =
                            make_float4(u[mb][nt][0], u[mb][nt][1], u[mb][nt][2], u[mb][nt][3]);
                }
                __syncthreads();
                if (warp < 4) {
                    #pragma unroll
                    for (int nt = 0; nt < 8; ++nt) {
                        const float4 v = *reinterpret_cast<const float4 *>(ub + 4 * (32 * nt + lane));
                        *reinterpret_cast<float4 *>(ub + 4 * (32 * nt + lane)) =
                            make_float4(u[mb][nt][0] + v.x, u[mb][nt][1] + v.y, u[mb][nt][2] + v.z, u[mb][nt][3] + v.w);
                    }
                }
                __syncthreads();
                // output (row, col) of the block: fragment (nt = col / 8, lane = 4 (row % 8) + (col % 8) / 2,
                // element 2 (row / 8) + col % 2)
                for (int o = tid; o < 16 * 64; o += kThreads) {
                    const int row = o >> 6, col = o & 63;
                    const int h = 16 * mb + row;
                    if (h < p.Hg) {
                        const int off = 4 * (32 * (col >> 3) + 4 * (row & 7) + ((col & 7) >> 1)) + 2 * (row >> 3) + (col & 1);
                        const float v = sm.ubuf[0][0][off] + sm.ubuf[1][0][off] + sm.ubuf[2][0][off] + sm.ubuf[3][0][off];
                        dst[(size_t)h * kVisPart + 2 + col] = v;
                    }
                }
            }
            if (tid < p.Hg) {
                dst[(size_t)tid * kVisPart] = sm.mcta[tid];
                dst[(size_t)tid * kVisPart + 1] = sm.lcta[tid];
            }
        }
        if (prefetch) { sm.upf[tid][0] = pf0; sm.upf[tid][1] = pf1; }
        if (p.mass == nullptr) continue;
        if (p.S == 1) {
            mass_warp(K, 0);
            continue;
        }
        // several splits: the last one to publish fixes the unit's (max, 1/sum).  Only warp 0
        // takes the arrival count (lanes over splits); the other warps go on to the mass.
        __syncthreads();
        if (warp == 0) {
            unsigned int old = 0;
            if (lane == 0) {
                __threadfence();
                asm volatile("atom.acq_rel.gpu.global.add.u32 %0, [%1], 1;" : "=r"(old) : "l"(&p.arrive[unit]) : "memory");
            }
            old = __shfl_sync(0xffffffffu, old, 0);
            if (old == (unsigned int)(p.S - 1)) {
                // lanes over the splits, four heads at a time with all their loads in flight
                const float *vu = p.part + (size_t)unit * p.S * p.Hg * kVisPart;
                for (int h0 = 0; h0 < p.Hg; h0 += 4) {
                    float ml[4][4], ll[4][4];
                    #pragma unroll
                    for (int hh = 0; hh < 4; ++hh)
                        #pragma unroll
                        for (int k = 0; k < 4; ++k) {
                            const int sp = lane + 32 * k;
                            const float *r2 = vu + ((size_t)sp * p.Hg + h0 + hh) * kVisPart;
                            ml[hh][k] = sp < p.S ? __ldcg(r2) : kRefInit;
                            ll[hh][k] = sp < p.S ? __ldcg(r2 + 1) : 0.f;
                        }
                    #pragma unroll
                    for (int hh = 0; hh < 4; ++hh) {
                        const int h = h0 + hh;
                        float mx = sm.tcur[h][0];
                        #pragma unroll
                        for (int k = 0; k < 4; ++k) mx = fmaxf(mx, ml[hh][k]);
                        for (int sp = lane + 128; sp < p.S; sp += 32)
                            mx = fmaxf(mx, __ldcg(vu + ((size_t)sp * p.Hg + h) * kVisPart));
                        #pragma unroll
                        for (int d = 16; d > 0; d >>= 1) mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, d));
                        float sum = 0.f;
                        #pragma unroll
                        for (int k = 0; k < 4; ++k) sum += ll[hh][k] * ex2(ml[hh][k] - mx);
                        for (int sp = lane + 128; sp < p.S; sp += 32) {
                            const float *r2 = vu + ((size_t)sp * p.Hg + h) * kVisPart;
                            sum += __ldcg(r2 + 1) * ex2(__ldcg(r2) - mx);
                        }
                        #pragma unroll
                        for (int d = 16; d > 0; d >>= 1) sum += __shfl_xor_sync(0xffffffffu, sum, d);
                        if (lane == 0) {
                            if (sm.tcur[h][0] != -INFINITY) sum += sm.tcur[h][1] * ex2(sm.tcur[h][0] - mx);
                            float *us = p.ustat + ((size_t)unit * p.Hg + h) * 2;
                            const float inv = 1.f / sum;
                            asm volatile("st.relaxed.gpu.global.v2.f32 [%0], {%1, %2};" :: "l"(us), "f"(mx), "f"(inv) : "memory");
                        }
                    }
                }
            }
            __syncwarp();
        }
        if (K >= 1) mass_warp(K - 1, 2);
    }
    if (p.mass != nullptr && p.S > 1 && K >= 1 && !*abort) mass_warp(K - 1, 1);

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
        tmem_dealloc(sm.tmem_base, C::kTmemCols);
    }
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

// dynamic shared memory of finish_kernel: weights of every partial, then u / l and w / l
__host__ __device__ constexpr size_t finish_smem_bytes(int S, int Sc) {
    return (size_t)(S + Sc) * kMaxHeads * sizeof(float) + (size_t)kMaxHeads * (64 + 128) * sizeof(float);
}

// One block per unit.  Per head, the unit-wide max M and sum L over every
// visual and text partial give each partial the weight 2^(m - M) / L; u / l and
// w / l are weighted sums with the feature index across threads (coalesced).
// Then o_h = (u_h / l_h) B_V[:, 128 j(h) ..] + w_h / l_h, thread t owning output
// columns 2t, 2t+1 of the unit's 512 (KV head t / 64).
__global__ void __launch_bounds__(256) finish_kernel(const FinishParams p) {
    extern __shared__ float fsm[];
    float *wv = fsm;                                  // [S][kMaxHeads]
    float *wt = wv + p.S * kMaxHeads;                 // [Sc][kMaxHeads]
    float (*uf)[64] = reinterpret_cast<float (*)[64]>(wt + p.Sc * kMaxHeads);
    float (*wf)[128] = reinterpret_cast<float (*)[128]>(&uf[kMaxHeads][0]);
    const int unit = blockIdx.x, tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const float *vp0 = p.vpart + (size_t)unit * p.S * p.Hg * kVisPart;
    const float *tp0 = p.tpart + (size_t)unit * p.Sc * p.Hg * kTxtPart;

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
            wv[s * kMaxHeads + h] = e;
            sum += __ldcg(r + 1) * e;
        }
        for (int c = lane; c < p.Sc; c += 32) {
            const float *r = tp0 + ((size_t)c * p.Hg + h) * kTxtPart;
            const float m = __ldcg(r);
            const float e = (m != -INFINITY) ? ex2(m - mx) : 0.f;
            wt[c * kMaxHeads + h] = e;
            sum += (m != -INFINITY) ? __ldcg(r + 1) * e : 0.f;
        }
        #pragma unroll
        for (int d = 16; d > 0; d >>= 1) sum += __shfl_xor_sync(0xffffffffu, sum, d);
        const float inv = 1.f / sum;
        if (lane == 0 && p.ustat != nullptr)
            *reinterpret_cast<float2 *>(p.ustat + ((size_t)unit * p.Hg + h) * 2) = make_float2(mx, inv);
        __syncwarp();
        for (int s = lane; s < p.S; s += 32) wv[s * kMaxHeads + h] *= inv;
        for (int c = lane; c < p.Sc; c += 32) wt[c * kMaxHeads + h] *= inv;
    }
    __syncthreads();
    for (int task = tid; task < p.Hg * 64; task += 256) {
        const int h = task >> 6, f = task & 63;
        const float *r = vp0 + (size_t)h * kVisPart + 2 + f;
        float a0 = 0.f, a1 = 0.f;
        int s = 0;
        for (; s + 2 <= p.S; s += 2) {
            a0 = fmaf(__ldcg(r + (size_t)s * p.Hg * kVisPart), wv[s * kMaxHeads + h], a0);
            a1 = fmaf(__ldcg(r + (size_t)(s + 1) * p.Hg * kVisPart), wv[(s + 1) * kMaxHeads + h], a1);
        }
        if (s < p.S) a0 = fmaf(__ldcg(r + (size_t)s * p.Hg * kVisPart), wv[s * kMaxHeads + h], a0);
        uf[h][f] = a0 + a1;
    }
    for (int task = tid; task < p.Hg * 128; task += 256) {
        const int h = task >> 7, f = task & 127;
        const float *r = tp0 + (size_t)h * kTxtPart + 2 + f;
        float a0 = 0.f, a1 = 0.f;
        int c = 0;
        for (; c + 2 <= p.Sc; c += 2) {
            a0 = fmaf(__ldcg(r + (size_t)c * p.Hg * kTxtPart), wt[c * kMaxHeads + h], a0);
            a1 = fmaf(__ldcg(r + (size_t)(c + 1) * p.Hg * kTxtPart), wt[(c + 1) * kMaxHeads + h], a1);
        }
        if (c < p.Sc) a0 = fmaf(__ldcg(r + (size_t)c * p.Hg * kTxtPart), wt[c * kMaxHeads + h], a0);
        wf[h][f] = a0 + a1;
    }
    __syncthreads();
    const int j = tid >> 6, d = (2 * tid) & 127;
    const int lb = unit / p.groups, G = unit % p.groups;
    const uint32_t *bv = reinterpret_cast<const uint32_t *>(p.BV + (size_t)unit * 64 * 512) + tid;
    float acc[8][2];
    #pragma unroll
    for (int hh = 0; hh < 8; ++hh) acc[hh][0] = acc[hh][1] = 0.f;
    const int h0 = j * p.per_kv;
    #pragma unroll 4
    for (int i0 = 0; i0 < 64; i0 += 16) {
        uint32_t braw[16];
        #pragma unroll
        for (int i = 0; i < 16; ++i) braw[i] = __ldcs(bv + (i0 + i) * 256);
        #pragma unroll
        for (int i = 0; i < 16; ++i) {
            const float b0 = __uint_as_float(braw[i] << 16), b1 = __uint_as_float(braw[i] & 0xffff0000u);
            #pragma unroll
            for (int hh = 0; hh < 8; ++hh) {
                if (hh < p.per_kv) {
                    const float x = uf[h0 + hh][i0 + i];
                    acc[hh][0] = fmaf(x, b0, acc[hh][0]);
                    acc[hh][1] = fmaf(x, b1, acc[hh][1]);
                }
            }
        }
    }
    #pragma unroll
    for (int hh = 0; hh < 8; ++hh) {
        if (hh < p.per_kv) {
            const int h = h0 + hh;
            *reinterpret_cast<uint32_t *>(p.out + ((size_t)lb * p.n_q + (size_t)G * p.Hg + h) * 128 + d) =
                pack_bf16(acc[hh][0] + wf[h][d], acc[hh][1] + wf[h][d + 1]);
        }
    }
}

}  // namespace decode
}  // namespace kvpack

namespace kvpack {
namespace decode {
// one block per SM: the opt-in shared-memory limit per block on sm_100 is 232448 bytes
static_assert(2 * (vis::smem_bytes<1>() + 1024) <= 233472, "visual kernel (16 head rows): two blocks per SM");
static_assert(vis::smem_bytes<2>() <= 232448, "visual kernel (32 head rows) shared memory");
static_assert(text::smem_bytes() <= 232448, "text kernel shared memory");
}  // namespace decode
}  // namespace kvpack
