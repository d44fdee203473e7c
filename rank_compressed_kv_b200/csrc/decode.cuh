// decode.cuh -- fused split-T decode attention over the rank-compressed visual
// cache plus the uncompressed text tail (AttentionPack decode step).
//
// Method ("Attention-aware Inference Optimizations for Large Vision-Language
// Models with Memory-efficient Decoding", technical summaries 2.B, fr/es/de
// pages): tokens whose importance is high are decompressed at the full rank,
// the others at a quarter of it.  Here decompression is folded into the
// attention by associativity: the query goes to rank space once
// (q~ = B_K[:, slice] q), a token's logit is C_K[t, :rho_t] . q~[:rho_t], the
// softmax-weighted V coefficients are summed in rank space and projected back
// through B_V once per head.  K and V are never materialised.
//
// Kernels
//   qproj_kernel  one block per unit: q~ for the unit's Hg heads, stored as a
//                 bf16 pair (hi + lo) so that the score MMA keeps ~16
//                 significant bits of q~; also clears the unit's arrival count.
//   attn_kernel   persistent; work item = (unit, split of the visual tokens and
//                 of the text tail).  Warp 8 is the producer: it walks the
//                 item's tokens and stages them into a 6-slot ring with
//                 cp.async (16-byte copies), one mbarrier pair per slot:
//                   LO   128 (or 64) tokens' 32-byte C_lo rows of K and V
//                   HI   32 full-rank tokens: C_lo + C_hi rows (128 B) of K and V
//                   TEXT 16 text tokens of one KV head: 256-byte K and V rows
//                 Warps 0-7 consume: mma.sync m16n8k16 bf16 with heads on M,
//                 tokens on N; online softmax in registers; P re-used from the
//                 score accumulators as the A operand of the value MMA.  A
//                 token with its mask bit set is scored in the HI stream at
//                 rank 64 and excluded (logit -inf) from the LO stream.
//                 Logits are kept on chip (fp32) for the attention mass.
//                 When a unit has S > 1 splits, the splits publish
//                 (max, sum, u, w) per head, count arrivals on a per-unit
//                 counter and wait (bounded) for their siblings; then each
//                 split writes the mass of its own tokens and the outputs of
//                 the heads h with h % S == split.
#pragma once

#include "common.cuh"

namespace kvpack {
namespace decode {

constexpr int kConsumerWarps = 8;
constexpr int kConsumers = kConsumerWarps * 32;
constexpr int kThreads = kConsumers + 32;
constexpr int kStages = 6;
constexpr int kStageBytes = 8192;
constexpr int kHiTokens = 32;
constexpr int kTextTokens = 16;
constexpr int kMaxHeads = 32;
constexpr int kPartFloats = 196;     // per (unit, split, head): m, l, pad2, u[64], w[128]

enum : int { ST_QT = 0, ST_Q = 1, ST_LO = 2, ST_HI = 3, ST_TEXT = 4, ST_END = 5, ST_STOP = 6 };

template <int NMB>
struct Cfg {
    static constexpr int kMRows = 16 * NMB;          // head rows (padded)
    static constexpr int kWPM = kConsumerWarps / NMB; // consumer warps per 16-head block
    static constexpr int kLoT = 16 * kWPM;            // tokens per LO stage
    static constexpr int kLS = kMRows + 4;            // logits row stride (floats), bank-conflict free
    static constexpr int kTPS = (NMB == 1) ? 1536 : 832;  // max visual tokens per split
};

struct StageHdr {
    int type, item, base, n, aux, aux2;
    uint32_t mask[4];
    uint16_t tok[kHiTokens];
    int pad[6];
};
static_assert(sizeof(StageHdr) == 128, "stage header size");

template <int NMB>
struct Smem {
    alignas(128) unsigned char ring[kStages][kStageBytes];
    StageHdr hdr[kStages];
    uint64_t full[kStages];
    uint64_t empty[kStages];
    uint64_t cbar;                                  // consumer-wide barrier (bounded waits)
    alignas(128) uint16_t qa[2][kMaxHeads][64];     // q~ hi / lo, 128-byte rows, 16-B chunks XOR-swizzled
    alignas(128) uint16_t qtxt[4][16][128];         // q rows of each KV head, 256-byte rows, swizzled
    float acc_u[kMaxHeads][64];
    float acc_w[kMaxHeads][128];
    float acc_l[kMaxHeads];
    float mcta[kMaxHeads];
    float mfin[kMaxHeads];
    float invl[kMaxHeads];
    float wmax_v[kConsumerWarps][16];
    float wmax_t[kConsumerWarps][16];
    float ucomb[2][64];
    uint16_t hi_pend[kHiTokens + 128];
    int abort;
    alignas(16) float logits[Cfg<NMB>::kTPS * Cfg<NMB>::kLS];
};

struct Params {
    const uint16_t *q, *CK_lo, *CK_hi, *BK, *CV_lo, *CV_hi, *BV, *Kt, *Vt;
    const uint32_t *mask;
    uint16_t *out;
    float *mass;
    uint16_t *qt;            // workspace: [units][2][Hg][64] bf16 q~ (hi, lo)
    float *part;             // workspace: [units][S][Hg][kPartFloats]
    unsigned int *arrive;    // workspace: [units]
    int n_units, T, L, Lcap, Hg, per_kv, n_q, groups, S, tps, txs, n_items, nwords;
    float scale2;            // softmax scale * log2(e)
};

__device__ __forceinline__ float ex2(float x) {
    float y;
    asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
    return y;
}

// ------------------------------------------------------------------ qproj

__global__ void __launch_bounds__(256) qproj_kernel(Params p) {
    __shared__ float qs[kMaxHeads][128];
    const int unit = blockIdx.x;
    const int lb = unit / p.groups, G = unit % p.groups;
    const uint16_t *qsrc = p.q + ((size_t)lb * p.n_q + (size_t)G * p.Hg) * 128;
    for (int i = threadIdx.x; i < p.Hg * 128; i += blockDim.x) qs[i >> 7][i & 127] = bf16_bits_to_float(qsrc[i]);
    if (threadIdx.x == 0) p.arrive[unit] = 0u;
    __syncthreads();
    const uint16_t *bk = p.BK + (size_t)unit * 64 * 512;
    uint16_t *dst = p.qt + (size_t)unit * 2 * p.Hg * 64;
    for (int o = threadIdx.x; o < p.Hg * 64; o += blockDim.x) {
        const int h = o >> 6, i = o & 63;
        float acc = 0.f;
        {
            const int j = h / p.per_kv;
            const uint4 *row = reinterpret_cast<const uint4 *>(bk + (size_t)i * 512 + j * 128);
            #pragma unroll 4
            for (int c = 0; c < 16; ++c) {
                uint4 v = __ldg(row + c);
                const uint32_t w[4] = {v.x, v.y, v.z, v.w};
                #pragma unroll
                for (int e = 0; e < 4; ++e) {
                    acc = fmaf(__uint_as_float(w[e] << 16), qs[h][8 * c + 2 * e], acc);
                    acc = fmaf(__uint_as_float(w[e] & 0xffff0000u), qs[h][8 * c + 2 * e + 1], acc);
                }
            }
        }
        const uint16_t hi = float_to_bf16_bits(acc);
        const uint16_t lo = float_to_bf16_bits(acc - bf16_bits_to_float(hi));
        dst[o] = hi;
        dst[p.Hg * 64 + o] = lo;
    }
}

// -------------------------------------------------------------- helpers

// Consumer-wide barrier on an mbarrier (count = kConsumers) with a bounded wait.
__device__ __forceinline__ void csync(uint64_t *bar, uint32_t &phase, volatile int *abort) {
    mbar_arrive(bar);
    mbar_wait(bar, phase, abort);
    phase ^= 1u;
}

// One online-softmax update of a 16-row x 16-token score block held as two
// m16n8 accumulators s[nb][0..3]; rescales NB accumulator tiles, returns P as
// the bf16 A fragment of the value MMA.
template <int NB>
__device__ __forceinline__ void softmax_step(float (&s)[2][4], float (&m)[2], float (&l)[2], float (&acc)[NB][4],
                                             uint32_t (&pa)[4]) {
    #pragma unroll
    for (int r = 0; r < 2; ++r) {
        float mx = fmaxf(fmaxf(s[0][2 * r], s[0][2 * r + 1]), fmaxf(s[1][2 * r], s[1][2 * r + 1]));
        mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, 1));
        mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, 2));
        const float mn = fmaxf(m[r], mx);
        float alpha;
        if (mn == -INFINITY) {
            alpha = 1.f;
            s[0][2 * r] = s[0][2 * r + 1] = s[1][2 * r] = s[1][2 * r + 1] = 0.f;
        } else {
            alpha = ex2(m[r] - mn);
            s[0][2 * r] = ex2(s[0][2 * r] - mn);
            s[0][2 * r + 1] = ex2(s[0][2 * r + 1] - mn);
            s[1][2 * r] = ex2(s[1][2 * r] - mn);
            s[1][2 * r + 1] = ex2(s[1][2 * r + 1] - mn);
        }
        l[r] = l[r] * alpha + (s[0][2 * r] + s[0][2 * r + 1]) + (s[1][2 * r] + s[1][2 * r + 1]);
        m[r] = mn;
        #pragma unroll
        for (int nb = 0; nb < NB; ++nb) {
            acc[nb][2 * r] *= alpha;
            acc[nb][2 * r + 1] *= alpha;
        }
    }
    pa[0] = pack_bf16(s[0][0], s[0][1]);
    pa[1] = pack_bf16(s[0][2], s[0][3]);
    pa[2] = pack_bf16(s[1][0], s[1][1]);
    pa[3] = pack_bf16(s[1][2], s[1][3]);
}

__device__ __forceinline__ void zero16(void *dst) {
    *reinterpret_cast<uint4 *>(dst) = make_uint4(0u, 0u, 0u, 0u);
}

// ---------------------------------------------------------------- producer

template <int NMB>
__device__ void producer(const Params &p, Smem<NMB> &sm, int lane) {
    using C = Cfg<NMB>;
    uint32_t seq = 0;
    auto acquire = [&]() -> int {
        const int slot = seq % kStages;
        const uint32_t k = seq / kStages;
        if (!mbar_wait(&sm.empty[slot], (k & 1u) ^ 1u, &sm.abort)) return -1;
        return slot;
    };
    auto commit = [&](int slot) {
        cp_async_arrive(&sm.full[slot]);
        mbar_arrive(&sm.full[slot]);
        ++seq;
    };
    auto header = [&](int slot, int type, int item, int base, int n, int aux, int aux2) {
        if (lane == 0) {
            StageHdr &h = sm.hdr[slot];
            h.type = type; h.item = item; h.base = base; h.n = n; h.aux = aux; h.aux2 = aux2;
        }
    };

    for (int item = blockIdx.x; item < p.n_items; item += gridDim.x) {
        const int unit = item / p.S, split = item % p.S;
        const int t0 = split * p.tps, t1 = min(p.T, t0 + p.tps);
        const int c0 = min(p.L, split * p.txs), c1 = min(p.L, c0 + p.txs);
        const size_t ubase = (size_t)unit * p.T;
        int slot;

        // q~ (bf16 hi and lo parts, 2 x Hg x 128 B)
        if ((slot = acquire()) < 0) break;
        header(slot, ST_QT, item, 0, 0, 0, 0);
        {
            const unsigned char *src = reinterpret_cast<const unsigned char *>(p.qt + (size_t)unit * 2 * p.Hg * 64);
            for (int c = lane; c < p.Hg * 16; c += 32) cp_async16(sm.ring[slot] + 16 * c, src + 16 * c);
        }
        commit(slot);

        // q rows of the unit's heads (Hg x 256 B)
        if ((slot = acquire()) < 0) break;
        header(slot, ST_Q, item, 0, 0, 0, 0);
        {
            const uint16_t *src = p.q + ((size_t)(unit / p.groups) * p.n_q + (size_t)(unit % p.groups) * p.Hg) * 128;
            for (int c = lane; c < p.Hg * 16; c += 32) cp_async16(sm.ring[slot] + 16 * c, src + 8 * c);
        }
        commit(slot);

        // visual tokens: LO tiles, HI stages of 32 pending full-rank tokens
        int npend = 0, hi_count = 0, lo_count = 0;
        bool ok = true;
        auto emit_hi = [&](int cnt) -> bool {
            int s2 = acquire();
            if (s2 < 0) return false;
            header(s2, ST_HI, item, t0, cnt, hi_count, 0);
            for (int i = lane; i < cnt; i += 32) sm.hdr[s2].tok[i] = sm.hi_pend[i];
            unsigned char *dk = sm.ring[s2];
            unsigned char *dv = sm.ring[s2] + 4096;
            for (int idx = lane; idx < kHiTokens * 8; idx += 32) {
                const int r = idx >> 3, ch = idx & 7;
                const int pos = (ch ^ (r & 7)) * 16;
                if (r < cnt) {
                    const size_t row = ubase + t0 + sm.hi_pend[r];
                    if (ch < 2) {
                        cp_async16(dk + r * 128 + pos, p.CK_lo + row * 16 + ch * 8);
                        cp_async16(dv + r * 128 + pos, p.CV_lo + row * 16 + ch * 8);
                    } else {
                        cp_async16(dk + r * 128 + pos, p.CK_hi + row * 48 + (ch - 2) * 8);
                        cp_async16(dv + r * 128 + pos, p.CV_hi + row * 48 + (ch - 2) * 8);
                    }
                } else {
                    zero16(dk + r * 128 + pos);
                    zero16(dv + r * 128 + pos);
                }
            }
            commit(s2);
            ++hi_count;
            return true;
        };

        for (int tb = t0; tb < t1 && ok; tb += C::kLoT) {
            const int n = min(C::kLoT, t1 - tb);
            if ((slot = acquire()) < 0) { ok = false; break; }
            header(slot, ST_LO, item, tb, n, lo_count, 0);
            // mask words of this tile (bits of tokens past n cleared)
            uint32_t word = 0u;
            const int nw = C::kLoT / 32;
            if (lane < nw) {
                const int widx = tb / 32 + lane;
                word = (widx < p.nwords) ? p.mask[(size_t)unit * p.nwords + widx] : 0u;
                const int lo_tok = 32 * lane;
                if (lo_tok >= n) word = 0u;
                else if (n - lo_tok < 32) word &= (1u << (n - lo_tok)) - 1u;
                sm.hdr[slot].mask[lane] = word;
            }
            unsigned char *dk = sm.ring[slot];
            unsigned char *dv = sm.ring[slot] + 4096;
            for (int idx = lane; idx < C::kLoT * 2; idx += 32) {
                const int r = idx >> 1, ch = idx & 1;
                const int pos = (ch ^ ((r >> 2) & 1)) * 16;
                if (r < n) {
                    const size_t row = ubase + tb + r;
                    cp_async16(dk + r * 32 + pos, p.CK_lo + row * 16 + ch * 8);
                    cp_async16(dv + r * 32 + pos, p.CV_lo + row * 16 + ch * 8);
                } else {
                    zero16(dk + r * 32 + pos);
                    zero16(dv + r * 32 + pos);
                }
            }
            commit(slot);
            ++lo_count;

            // append the tile's full-rank tokens (split-relative) to the pending list
            const int cnt = __popc(word);
            int incl = cnt;
            #pragma unroll
            for (int d = 1; d < 32; d <<= 1) {
                const int v = __shfl_up_sync(0xffffffffu, incl, d);
                if (lane >= d) incl += v;
            }
            const int total = __shfl_sync(0xffffffffu, incl, 31);
            int off = npend + incl - cnt;
            while (word) {
                const int b = __ffs(word) - 1;
                sm.hi_pend[off++] = (uint16_t)(tb - t0 + 32 * lane + b);
                word &= word - 1u;
            }
            npend += total;
            __syncwarp();
            while (npend >= kHiTokens) {
                if (!emit_hi(kHiTokens)) { ok = false; break; }
                __syncwarp();
                uint16_t mv[5];
                const int rest = npend - kHiTokens;
                #pragma unroll
                for (int k = 0; k < 5; ++k) {
                    const int i = lane + 32 * k;
                    mv[k] = (i < rest) ? sm.hi_pend[kHiTokens + i] : 0;
                }
                __syncwarp();
                #pragma unroll
                for (int k = 0; k < 5; ++k) {
                    const int i = lane + 32 * k;
                    if (i < rest) sm.hi_pend[i] = mv[k];
                }
                __syncwarp();
                npend = rest;
            }
        }
        if (!ok) break;
        if (npend > 0) {
            if (!emit_hi(npend)) break;
        }

        // text tail: 16 tokens x one KV head per stage
        for (int ct = c0, tt = 0; ct < c1 && ok; ct += kTextTokens, ++tt) {
            const int n = min(kTextTokens, c1 - ct);
            for (int j = 0; j < 4; ++j) {
                if ((slot = acquire()) < 0) { ok = false; break; }
                header(slot, ST_TEXT, item, ct, n, j, tt);
                unsigned char *dk = sm.ring[slot];
                unsigned char *dv = sm.ring[slot] + 4096;
                for (int idx = lane; idx < kTextTokens * 16; idx += 32) {
                    const int r = idx >> 4, ch = idx & 15;
                    const int pos = (ch ^ (r & 7)) * 16;
                    if (r < n) {
                        const size_t row = (((size_t)unit * p.Lcap + ct + r) * 4 + j) * 128;
                        cp_async16(dk + r * 256 + pos, p.Kt + row + ch * 8);
                        cp_async16(dv + r * 256 + pos, p.Vt + row + ch * 8);
                    } else {
                        zero16(dk + r * 256 + pos);
                        zero16(dv + r * 256 + pos);
                    }
                }
                commit(slot);
            }
        }
        if (!ok) break;

        if ((slot = acquire()) < 0) break;
        header(slot, ST_END, item, 0, 0, 0, 0);
        commit(slot);
    }
    int slot = acquire();
    if (slot >= 0) {
        header(slot, ST_STOP, -1, 0, 0, 0, 0);
        commit(slot);
    }
    cp_async_wait_all();
}

// ---------------------------------------------------------------- consumers

template <int NMB>
__device__ void consumers(const Params &p, Smem<NMB> &sm, int warp, int lane) {
    using C = Cfg<NMB>;
    const int g = lane >> 2, tig = lane & 3;
    const int ctid = warp * 32 + lane;
    const int mb = warp / C::kWPM;        // this warp's 16-head block (visual)
    const int win = warp % C::kWPM;
    const int jt = warp & 3;              // this warp's KV head (text)
    volatile int *abort = &sm.abort;
    uint32_t cphase = 0;

    // visual softmax state (rows g, g+8 of block mb) and rank-space accumulator u^T
    float vm[2], vl[2], u[8][4];
    // text softmax state (rows g, g+8 of KV head jt) and head-space accumulator w^T
    float tm[2], tl[2], w[16][4];
    uint32_t qah[4], qal[4];              // q~ A fragments, rank 0..15 (hi / lo)

    auto reset_state = [&]() {
        vm[0] = vm[1] = tm[0] = tm[1] = -INFINITY;
        vl[0] = vl[1] = tl[0] = tl[1] = 0.f;
        #pragma unroll
        for (int a = 0; a < 8; ++a) u[a][0] = u[a][1] = u[a][2] = u[a][3] = 0.f;
        #pragma unroll
        for (int a = 0; a < 16; ++a) w[a][0] = w[a][1] = w[a][2] = w[a][3] = 0.f;
    };
    reset_state();
    for (int i = ctid; i < kMaxHeads * 64; i += kConsumers) (&sm.acc_u[0][0])[i] = 0.f;
    for (int i = ctid; i < kMaxHeads * 128; i += kConsumers) (&sm.acc_w[0][0])[i] = 0.f;
    if (ctid < kMaxHeads) sm.acc_l[ctid] = 0.f;
    csync(&sm.cbar, cphase, abort);

    const uint32_t qa_base[2] = {smem_u32(&sm.qa[0][0][0]), smem_u32(&sm.qa[1][0][0])};
    int item = -1, unit = 0, split = 0, t0 = 0, t1 = 0;

    for (uint32_t seq = 0;; ++seq) {
        const int slot = seq % kStages;
        const uint32_t k = seq / kStages;
        const bool ok = mbar_wait(&sm.full[slot], k & 1u, abort);
        const StageHdr &hd = sm.hdr[slot];
        const int type = ok ? hd.type : ST_STOP;
        const unsigned char *st = sm.ring[slot];
        const uint32_t sbase = smem_u32(st);

        if (type == ST_QT) {
            item = hd.item;
            unit = item / p.S; split = item % p.S;
            t0 = split * p.tps; t1 = min(p.T, t0 + p.tps);
            for (int c = ctid; c < 512; c += kConsumers) {
                const int part = c >> 8, row = (c >> 3) & 31, ch = c & 7;
                uint4 v = make_uint4(0u, 0u, 0u, 0u);
                if (row < p.Hg) v = *reinterpret_cast<const uint4 *>(st + (part * p.Hg + row) * 128 + 16 * ch);
                *reinterpret_cast<uint4 *>(reinterpret_cast<unsigned char *>(&sm.qa[part][row][0]) + ((ch ^ (row & 7)) << 4)) = v;
            }
            csync(&sm.cbar, cphase, abort);
            const int row = 16 * mb + (lane & 7) + (((lane >> 3) & 1) << 3);
            const int ch = lane >> 4;
            const uint32_t off = row * 128 + ((ch ^ (row & 7)) << 4);
            ldsm_x4(qa_base[0] + off, qah[0], qah[1], qah[2], qah[3]);
            ldsm_x4(qa_base[1] + off, qal[0], qal[1], qal[2], qal[3]);
        } else if (type == ST_Q) {
            for (int c = ctid; c < 4 * 16 * 16; c += kConsumers) {
                const int j = c >> 8, rr = (c >> 4) & 15, ch = c & 15;
                uint4 v = make_uint4(0u, 0u, 0u, 0u);
                if (rr < p.per_kv) v = *reinterpret_cast<const uint4 *>(st + (j * p.per_kv + rr) * 256 + 16 * ch);
                *reinterpret_cast<uint4 *>(reinterpret_cast<unsigned char *>(&sm.qtxt[j][rr][0]) + ((ch ^ (rr & 7)) << 4)) = v;
            }
            csync(&sm.cbar, cphase, abort);
        } else if (type == ST_LO) {
            const int base = hd.base, n = hd.n;
            // scores S^T[h, t] for 16 heads x 16 tokens at rank 0..15
            uint32_t b0, b1, b2, b3;
            {
                const int row = win * 16 + (lane & 7) + ((lane >> 4) << 3);
                const int ch = (lane >> 3) & 1;
                ldsm_x4(sbase + row * 32 + ((ch ^ ((row >> 2) & 1)) << 4), b0, b1, b2, b3);
            }
            float s[2][4] = {{0.f, 0.f, 0.f, 0.f}, {0.f, 0.f, 0.f, 0.f}};
            mma_bf16(s[0], qah, b0, b1);
            mma_bf16(s[0], qal, b0, b1);
            mma_bf16(s[1], qah, b2, b3);
            mma_bf16(s[1], qal, b2, b3);
            #pragma unroll
            for (int nb = 0; nb < 2; ++nb) {
                #pragma unroll
                for (int e = 0; e < 2; ++e) {
                    const int tl_ = win * 16 + nb * 8 + 2 * tig + e;
                    const bool hi = (hd.mask[tl_ >> 5] >> (tl_ & 31)) & 1u;
                    const bool use = (tl_ < n) && !hi;
                    const float x0 = use ? s[nb][e] * p.scale2 : -INFINITY;
                    const float x1 = use ? s[nb][2 + e] * p.scale2 : -INFINITY;
                    s[nb][e] = x0;
                    s[nb][2 + e] = x1;
                    if (use) {
                        const int rel = base + tl_ - t0;
                        if (rel >= 0 && rel < C::kTPS) {
                            sm.logits[rel * C::kLS + 16 * mb + g] = x0;
                            sm.logits[rel * C::kLS + 16 * mb + g + 8] = x1;
                        }
                    }
                }
            }
            uint32_t pa[4];
            softmax_step<8>(s, vm, vl, u, pa);
            {
                const int row = win * 16 + (lane & 7) + (((lane >> 3) & 1) << 3);
                const int ch = lane >> 4;
                ldsm_x4_t(sbase + 4096 + row * 32 + ((ch ^ ((row >> 2) & 1)) << 4), b0, b1, b2, b3);
            }
            mma_bf16(u[0], pa, b0, b1);
            mma_bf16(u[1], pa, b2, b3);
        } else if (type == ST_HI) {
            const int n = hd.n, hc = hd.aux;
            const int sub = ((win - 2 * hc) % C::kWPM + C::kWPM) % C::kWPM;
            if (sub < 2) {
                float s[2][4] = {{0.f, 0.f, 0.f, 0.f}, {0.f, 0.f, 0.f, 0.f}};
                #pragma unroll
                for (int kb = 0; kb < 4; ++kb) {
                    uint32_t ah[4], al[4];
                    if (kb == 0) {
                        #pragma unroll
                        for (int e = 0; e < 4; ++e) { ah[e] = qah[e]; al[e] = qal[e]; }
                    } else {
                        const int row = 16 * mb + (lane & 7) + (((lane >> 3) & 1) << 3);
                        const int ch = 2 * kb + (lane >> 4);
                        const uint32_t off = row * 128 + ((ch ^ (row & 7)) << 4);
                        ldsm_x4(qa_base[0] + off, ah[0], ah[1], ah[2], ah[3]);
                        ldsm_x4(qa_base[1] + off, al[0], al[1], al[2], al[3]);
                    }
                    uint32_t b0, b1, b2, b3;
                    const int row = 16 * sub + (lane & 7) + ((lane >> 4) << 3);
                    const int ch = 2 * kb + ((lane >> 3) & 1);
                    ldsm_x4(sbase + row * 128 + ((ch ^ (row & 7)) << 4), b0, b1, b2, b3);
                    mma_bf16(s[0], ah, b0, b1);
                    mma_bf16(s[0], al, b0, b1);
                    mma_bf16(s[1], ah, b2, b3);
                    mma_bf16(s[1], al, b2, b3);
                }
                #pragma unroll
                for (int nb = 0; nb < 2; ++nb) {
                    #pragma unroll
                    for (int e = 0; e < 2; ++e) {
                        const int cl = 16 * sub + nb * 8 + 2 * tig + e;
                        const bool use = cl < n;
                        const float x0 = use ? s[nb][e] * p.scale2 : -INFINITY;
                        const float x1 = use ? s[nb][2 + e] * p.scale2 : -INFINITY;
                        s[nb][e] = x0;
                        s[nb][2 + e] = x1;
                        if (use) {
                            const int rel = hd.tok[cl];
                            if (rel < C::kTPS) {
                                sm.logits[rel * C::kLS + 16 * mb + g] = x0;
                                sm.logits[rel * C::kLS + 16 * mb + g + 8] = x1;
                            }
                        }
                    }
                }
                uint32_t pa[4];
                softmax_step<8>(s, vm, vl, u, pa);
                #pragma unroll
                for (int pr = 0; pr < 4; ++pr) {
                    uint32_t b0, b1, b2, b3;
                    const int row = 16 * sub + (lane & 7) + (((lane >> 3) & 1) << 3);
                    const int ch = 2 * pr + (lane >> 4);
                    ldsm_x4_t(sbase + 4096 + row * 128 + ((ch ^ (row & 7)) << 4), b0, b1, b2, b3);
                    mma_bf16(u[2 * pr], pa, b0, b1);
                    mma_bf16(u[2 * pr + 1], pa, b2, b3);
                }
            }
        } else if (type == ST_TEXT) {
            const int j = hd.aux, tt = hd.aux2, n = hd.n;
            if (warp == 4 * (tt & 1) + j) {
                const uint32_t qb = smem_u32(&sm.qtxt[j][0][0]);
                float s[2][4] = {{0.f, 0.f, 0.f, 0.f}, {0.f, 0.f, 0.f, 0.f}};
                #pragma unroll
                for (int kb = 0; kb < 8; ++kb) {
                    uint32_t a[4], b0, b1, b2, b3;
                    {
                        const int row = (lane & 7) + (((lane >> 3) & 1) << 3);
                        const int ch = 2 * kb + (lane >> 4);
                        ldsm_x4(qb + row * 256 + ((ch ^ (row & 7)) << 4), a[0], a[1], a[2], a[3]);
                    }
                    {
                        const int row = (lane & 7) + ((lane >> 4) << 3);
                        const int ch = 2 * kb + ((lane >> 3) & 1);
                        ldsm_x4(sbase + row * 256 + ((ch ^ (row & 7)) << 4), b0, b1, b2, b3);
                    }
                    mma_bf16(s[0], a, b0, b1);
                    mma_bf16(s[1], a, b2, b3);
                }
                #pragma unroll
                for (int nb = 0; nb < 2; ++nb) {
                    #pragma unroll
                    for (int e = 0; e < 2; ++e) {
                        const bool use = (nb * 8 + 2 * tig + e) < n;
                        s[nb][e] = use ? s[nb][e] * p.scale2 : -INFINITY;
                        s[nb][2 + e] = use ? s[nb][2 + e] * p.scale2 : -INFINITY;
                    }
                }
                uint32_t pa[4];
                softmax_step<16>(s, tm, tl, w, pa);
                #pragma unroll
                for (int pr = 0; pr < 8; ++pr) {
                    uint32_t b0, b1, b2, b3;
                    const int row = (lane & 7) + (((lane >> 3) & 1) << 3);
                    const int ch = 2 * pr + (lane >> 4);
                    ldsm_x4_t(sbase + 4096 + row * 256 + ((ch ^ (row & 7)) << 4), b0, b1, b2, b3);
                    mma_bf16(w[2 * pr], pa, b0, b1);
                    mma_bf16(w[2 * pr + 1], pa, b2, b3);
                }
            }
        }

        __syncwarp();
        if (lane == 0) mbar_arrive(&sm.empty[slot]);
        if (type == ST_STOP) break;
        if (type != ST_END) continue;

        // ============================ epilogue of one work item
        const int Hg = p.Hg;
        #pragma unroll
        for (int r = 0; r < 2; ++r) {
            vl[r] += __shfl_xor_sync(0xffffffffu, vl[r], 1);
            vl[r] += __shfl_xor_sync(0xffffffffu, vl[r], 2);
            tl[r] += __shfl_xor_sync(0xffffffffu, tl[r], 1);
            tl[r] += __shfl_xor_sync(0xffffffffu, tl[r], 2);
        }
        if (tig == 0) {
            sm.wmax_v[warp][g] = vm[0];
            sm.wmax_v[warp][g + 8] = vm[1];
            sm.wmax_t[warp][g] = tm[0];
            sm.wmax_t[warp][g + 8] = tm[1];
        }
        csync(&sm.cbar, cphase, abort);
        if (ctid < Hg) {
            const int h = ctid;
            float mx = -INFINITY;
            for (int w2 = 0; w2 < kConsumerWarps; ++w2) {
                if (w2 / C::kWPM == h / 16) mx = fmaxf(mx, sm.wmax_v[w2][h % 16]);
                const int j = h / p.per_kv, rr = h % p.per_kv;
                if ((w2 & 3) == j) mx = fmaxf(mx, sm.wmax_t[w2][rr]);
            }
            sm.mcta[h] = mx;
        }
        csync(&sm.cbar, cphase, abort);
        // rescale this warp's partials to the block maximum and add them up
        #pragma unroll
        for (int r = 0; r < 2; ++r) {
            const int h = 16 * mb + g + 8 * r;
            if (h < Hg) {
                const float mc = sm.mcta[h];
                const float f = (vm[r] == -INFINITY) ? 0.f : ex2(vm[r] - mc);
                #pragma unroll
                for (int nb = 0; nb < 8; ++nb) {
                    atomicAdd(&sm.acc_u[h][8 * nb + 2 * tig], u[nb][2 * r] * f);
                    atomicAdd(&sm.acc_u[h][8 * nb + 2 * tig + 1], u[nb][2 * r + 1] * f);
                }
                if (tig == 0) atomicAdd(&sm.acc_l[h], vl[r] * f);
            }
            const int rr = g + 8 * r;
            if (rr < p.per_kv) {
                const int ht = jt * p.per_kv + rr;
                const float mc = sm.mcta[ht];
                const float f = (tm[r] == -INFINITY) ? 0.f : ex2(tm[r] - mc);
                if (f != 0.f) {
                    #pragma unroll
                    for (int nb = 0; nb < 16; ++nb) {
                        atomicAdd(&sm.acc_w[ht][8 * nb + 2 * tig], w[nb][2 * r] * f);
                        atomicAdd(&sm.acc_w[ht][8 * nb + 2 * tig + 1], w[nb][2 * r + 1] * f);
                    }
                    if (tig == 0) atomicAdd(&sm.acc_l[ht], tl[r] * f);
                }
            }
        }
        csync(&sm.cbar, cphase, abort);

        if (p.S > 1) {
            float *mine = p.part + ((size_t)unit * p.S + split) * Hg * kPartFloats;
            for (int i = ctid; i < Hg * kPartFloats; i += kConsumers) {
                const int h = i / kPartFloats, f = i % kPartFloats;
                float v;
                if (f == 0) v = sm.mcta[h];
                else if (f == 1) v = sm.acc_l[h];
                else if (f < 4) v = 0.f;
                else if (f < 68) v = sm.acc_u[h][f - 4];
                else v = sm.acc_w[h][f - 68];
                mine[i] = v;
            }
            __threadfence();
            csync(&sm.cbar, cphase, abort);
            if (ctid == 0) {
                atomicAdd(&p.arrive[unit], 1u);
                const long long start = clock64();
                while (true) {
                    unsigned int v;
                    asm volatile("ld.acquire.gpu.global.u32 %0, [%1];" : "=r"(v) : "l"(&p.arrive[unit]) : "memory");
                    if (v >= (unsigned int)p.S) break;
                    if (*abort) break;
                    if (clock64() - start > kWaitCycles) {
                        report_error(KVPACK_ERR_TIMEOUT);
                        *abort = 1;
                        break;
                    }
                    __nanosleep(256);
                }
            }
            csync(&sm.cbar, cphase, abort);
            if (ctid < Hg) {
                const int h = ctid;
                const float *ph = p.part + (size_t)unit * p.S * Hg * kPartFloats + (size_t)h * kPartFloats;
                float M = -INFINITY;
                for (int s2 = 0; s2 < p.S; ++s2) M = fmaxf(M, __ldcg(ph + (size_t)s2 * Hg * kPartFloats));
                float Lsum = 0.f;
                for (int s2 = 0; s2 < p.S; ++s2) {
                    const float ms = __ldcg(ph + (size_t)s2 * Hg * kPartFloats);
                    if (ms != -INFINITY) Lsum += __ldcg(ph + (size_t)s2 * Hg * kPartFloats + 1) * ex2(ms - M);
                }
                sm.mfin[h] = M;
                sm.invl[h] = 1.f / Lsum;
            }
        } else {
            if (ctid < Hg) {
                sm.mfin[ctid] = sm.mcta[ctid];
                sm.invl[ctid] = 1.f / sm.acc_l[ctid];
            }
        }
        csync(&sm.cbar, cphase, abort);

        // attention mass of this split's visual tokens
        if (p.mass != nullptr) {
            for (int t = t0 + ctid; t < t1; t += kConsumers) {
                const float *lg = sm.logits + (size_t)(t - t0) * C::kLS;
                float acc = 0.f;
                for (int h = 0; h < Hg; ++h) acc = fmaf(ex2(lg[h] - sm.mfin[h]), sm.invl[h], acc);
                p.mass[(size_t)unit * p.T + t] = acc;
            }
        }

        // outputs of the heads assigned to this split, two heads at a time
        {
            const int lb = unit / p.groups, G = unit % p.groups;
            const int half = ctid >> 7, d = ctid & 127;
            const float *pu = p.part + (size_t)unit * p.S * Hg * kPartFloats;
            for (int h0 = split; h0 < Hg; h0 += 2 * p.S) {
                const int h = h0 + half * p.S;
                const bool act = h < Hg;
                // combined u (rank space) of head h into ucomb[half]
                if (act && d < 64) {
                    float uv;
                    if (p.S == 1) {
                        uv = sm.acc_u[h][d];
                    } else {
                        uv = 0.f;
                        for (int s2 = 0; s2 < p.S; ++s2) {
                            const float *ps = pu + ((size_t)s2 * Hg + h) * kPartFloats;
                            const float ms = __ldcg(ps);
                            if (ms != -INFINITY) uv += __ldcg(ps + 4 + d) * ex2(ms - sm.mfin[h]);
                        }
                    }
                    sm.ucomb[half][d] = uv;
                }
                csync(&sm.cbar, cphase, abort);
                if (act) {
                    const int j = h / p.per_kv;
                    float wv;
                    if (p.S == 1) {
                        wv = sm.acc_w[h][d];
                    } else {
                        wv = 0.f;
                        for (int s2 = 0; s2 < p.S; ++s2) {
                            const float *ps = pu + ((size_t)s2 * Hg + h) * kPartFloats;
                            const float ms = __ldcg(ps);
                            if (ms != -INFINITY) wv += __ldcg(ps + 68 + d) * ex2(ms - sm.mfin[h]);
                        }
                    }
                    const uint16_t *bv = p.BV + (size_t)unit * 64 * 512 + j * 128 + d;
                    float o = wv;
                    #pragma unroll 8
                    for (int i = 0; i < 64; ++i) o = fmaf(sm.ucomb[half][i], bf16_bits_to_float(__ldg(bv + (size_t)i * 512)), o);
                    p.out[((size_t)lb * p.n_q + (size_t)G * Hg + h) * 128 + d] = float_to_bf16_bits(o * sm.invl[h]);
                }
                csync(&sm.cbar, cphase, abort);
            }
        }

        // clear the block accumulators and the warp state for the next item
        for (int i = ctid; i < kMaxHeads * 64; i += kConsumers) (&sm.acc_u[0][0])[i] = 0.f;
        for (int i = ctid; i < kMaxHeads * 128; i += kConsumers) (&sm.acc_w[0][0])[i] = 0.f;
        if (ctid < kMaxHeads) sm.acc_l[ctid] = 0.f;
        reset_state();
        csync(&sm.cbar, cphase, abort);
    }
}

template <int NMB>
__global__ void __launch_bounds__(kThreads, 1) attn_kernel(Params p) {
    extern __shared__ __align__(128) unsigned char smem_raw[];
    Smem<NMB> &sm = *reinterpret_cast<Smem<NMB> *>(smem_raw);
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    if (threadIdx.x == 0) {
        for (int s = 0; s < kStages; ++s) {
            mbar_init(&sm.full[s], 32);
            mbar_init(&sm.empty[s], kConsumerWarps);
        }
        mbar_init(&sm.cbar, kConsumers);
        sm.abort = 0;
        asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
    }
    __syncthreads();
    if (warp == kConsumerWarps) producer<NMB>(p, sm, lane);
    else consumers<NMB>(p, sm, warp, lane);
}

}  // namespace decode
}  // namespace kvpack
