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
// attn_kernel is persistent (one 288-thread block per SM).  A work item is a
// unit's split of the visual tokens and of the text tail.  Warp 8 produces:
// it stages the item into a 6-slot shared-memory ring (8 KB per slot, a
// full / empty mbarrier pair per slot):
//   Q     the unit's query rows (cp.async)
//   BK    32 rows of B_K for one KV head (TMA, 128-byte swizzle)
//   QDONE barrier: q~ complete
//   LO    128 (Hg <= 16) or 64 tokens' 32-byte C_lo rows of K and V (TMA, 32-byte swizzle)
//   HI    32 full-rank tokens: C_lo + C_hi rows of K and V gathered with cp.async
//   TEXT  16 text tokens of one KV head, K and V (TMA, 128-byte swizzle)
//   END   the item's tokens are done
//   BV    32 rows of B_V for one KV head (TMA)
//   FIN   outputs complete
// Warps 0-7 consume.  q~ = q B_K^T by mma.sync from the BK stages, kept as a
// bf16 hi + lo pair (~16 significant bits).  Scores and values run on
// mma.sync m16n8k16 (bf16 in, fp32 accumulate) with heads on M and tokens on
// N; the online softmax stays in registers and P is reused from the score
// accumulators as the A operand of the value MMA.  A token with its mask bit
// set is scored at rank 64 in the HI stream and gets logit -inf in the LO
// stream (rank 16).  Logits stay in shared memory for the attention mass.
// When a unit has S > 1 splits, each split publishes (max, sum) and (u, w)
// per head, counts itself on a per-unit counter and waits (bounded) for its
// siblings; a static round-robin schedule on a cooperative launch keeps the
// wait deadlock-free.  Split s then writes the mass of its own tokens and the
// outputs of heads h with h % S == s, projecting u through B_V.
#pragma once

#include <cuda.h>

#include "common.cuh"

namespace kvpack {
namespace decode {

constexpr int kConsumerWarps = 8;
constexpr int kConsumers = kConsumerWarps * 32;
constexpr int kThreads = kConsumers + 32;
constexpr int kStages = 11;
constexpr int kStageBytes = 8192;
constexpr int kHiTokens = 32;
constexpr int kTextTokens = 16;
constexpr int kMaxHeads = 32;
constexpr int kUW = 192;              // per (unit, split, head): u[64] then w[128]

enum : int {
    ST_Q = 0, ST_BK = 1, ST_QDONE = 2, ST_LO = 3, ST_HI = 4, ST_TEXT = 5, ST_END = 6, ST_BV = 7, ST_FIN = 8,
    ST_STOP = 9
};

template <int NMB>
struct Cfg {
    static constexpr int kMRows = 16 * NMB;          // head rows (padded)
    static constexpr int kWPM = kConsumerWarps / NMB; // consumer warps per 16-head block
    static constexpr int kLoT = 16 * kWPM;            // tokens per LO stage
    static constexpr int kLS = kMRows + 4;            // logits row stride (floats), bank-conflict free
    static constexpr int kTPS = (NMB == 1) ? 1024 : 512;  // max visual tokens per split
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
    alignas(1024) unsigned char ring[kStages][kStageBytes];
    StageHdr hdr[kStages];
    uint64_t hbar[kStages];     // header published (1 arrival): warps that skip a stage need only this
    uint64_t full[kStages];     // header and data landed
    uint64_t empty[kStages];    // every consumer warp is done with the slot
    uint64_t cbar;                                  // consumer-wide barrier (bounded waits)
    union {
        struct {   // while an item's tokens stream
            alignas(128) uint16_t qa[2][kMaxHeads][64];   // q~ hi / lo, 128-byte rows, 16-B chunks XOR-swizzled
            alignas(128) uint16_t qtxt[4][16][128];       // q rows of each KV head, 256-byte rows, swizzled
        };
        struct {   // in the item's epilogue: block-wide sums in register order (bank-conflict-free atomics)
            float frag_u[2][32][32];                      // [head block][register][lane]
            float frag_w[4][32][32];                      // [KV head][register][lane]
        };
    };
    float acc_u[kMaxHeads][64];                     // u / l of the unit (rank space)
    float acc_w[kMaxHeads][128];                    // w / l of the unit (text part)
    float acc_l[kMaxHeads];
    float mcta[kMaxHeads];
    float mfin[kMaxHeads];
    float invl[kMaxHeads];
    float wmax_v[kConsumerWarps][16];
    float wmax_t[kConsumerWarps][16];
    uint16_t hi_pend[kHiTokens + 128];
    uint32_t mask_words[Cfg<NMB>::kTPS / 32];    // producer's copy of the item's rank-mask words
    int abort;
    alignas(16) float logits[Cfg<NMB>::kTPS * Cfg<NMB>::kLS];
};

struct Params {
    CUtensorMap tm_ck, tm_cv;    // C_lo planes of K and V: 2D [units*T][16], box {16, LoT}, 32-byte swizzle
    CUtensorMap tm_kt, tm_vt;    // text tails: 3D [units*Lcap][4][128], box {64, 1, 16}, 128-byte swizzle
    CUtensorMap tm_bk, tm_bv;    // bases: 2D [units*64][512], box {64, 32}, 128-byte swizzle
    const uint16_t *q, *CK_lo, *CK_hi, *CV_lo, *CV_hi;
    const uint32_t *mask;
    uint16_t *out;
    float *mass;
    float *ml;               // workspace: [units][S][Hg][2]  (max, sum) of each split
    float *uw;               // workspace: [units][S][Hg][kUW] (u, w) of each split
    unsigned int *arrive;    // workspace: [units]
    int n_units, T, L, Lcap, Hg, per_kv, n_q, groups, S, tps, txs, n_items, nwords;
    float scale2;            // softmax scale * log2(e)
};

__device__ __forceinline__ float ex2(float x) {
    float y;
    asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
    return y;
}

// -------------------------------------------------------------- TMA helpers

__device__ __forceinline__ void mbar_arrive_tx(uint64_t *bar, uint32_t bytes) {
    asm volatile("mbarrier.arrive.expect_tx.shared::cta.b64 _, [%0], %1;" :: "r"(smem_u32(bar)), "r"(bytes) : "memory");
}

__device__ __forceinline__ void tma_2d(void *dst, const CUtensorMap *tm, int c0, int c1, uint64_t *bar) {
    asm volatile(
        "cp.async.bulk.tensor.2d.shared::cluster.global.tile.mbarrier::complete_tx::bytes [%0], [%1, {%2, %3}], [%4];"
        :: "r"(smem_u32(dst)), "l"(reinterpret_cast<uint64_t>(tm)), "r"(c0), "r"(c1), "r"(smem_u32(bar)) : "memory");
}

__device__ __forceinline__ void tma_3d(void *dst, const CUtensorMap *tm, int c0, int c1, int c2, uint64_t *bar) {
    asm volatile(
        "cp.async.bulk.tensor.3d.shared::cluster.global.tile.mbarrier::complete_tx::bytes [%0], [%1, {%2, %3, %4}], [%5];"
        :: "r"(smem_u32(dst)), "l"(reinterpret_cast<uint64_t>(tm)), "r"(c0), "r"(c1), "r"(c2), "r"(smem_u32(bar))
        : "memory");
}

// byte offset of element (row, col) of a 128-byte-swizzled box of 64 bf16 per row
__device__ __forceinline__ uint32_t sw128(int row, int col) {
    return row * 128 + ((((col >> 3) ^ (row & 7)) & 7) << 4) + (col & 7) * 2;
}

// -------------------------------------------------------------- helpers

// Consumer-wide barrier on an mbarrier (one arrival per consumer warp, after a
// warp-level sync that orders the warp's earlier shared-memory writes) with a
// bounded wait.
__device__ __forceinline__ void csync(uint64_t *bar, uint32_t &phase, volatile int *abort) {
    __syncwarp();
    if ((threadIdx.x & 31) == 0) mbar_arrive(bar);
    __syncwarp();   // no lane polls before lane 0 has arrived
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

// Heads of this split's output: h % S == split.  Bit j of the result is set if
// a head of KV head j is among them.
__device__ __forceinline__ int output_kv_heads(const Params &p, int split) {
    int m = 0;
    for (int h = split; h < p.Hg; h += p.S) m |= 1 << (h / p.per_kv);
    return m;
}

// ---------------------------------------------------------------- producer

template <int NMB>
__device__ void producer(const Params &p, Smem<NMB> &sm, int lane) {
    using C = Cfg<NMB>;
    uint32_t seq = 0;
    auto acquire = [&]() -> int {
        __syncwarp();   // lane 0's arrivals and copy issues of the previous stage are done
        const int slot = seq % kStages;
        const uint32_t k = seq / kStages;
        if (!mbar_wait(&sm.empty[slot], (k & 1u) ^ 1u, &sm.abort)) return -1;
        return slot;
    };
    // arrivals: lane 0 announces the TMA bytes (0 for none); lanes that issued cp.async
    // copies arrive again when those land
    auto commit = [&](int slot, uint32_t tma_bytes, bool used_cp_async) {
        if (used_cp_async) cp_async_arrive(&sm.full[slot]);
        if (lane == 0 && tma_bytes) mbar_arrive_tx(&sm.full[slot], tma_bytes);
        else mbar_arrive(&sm.full[slot]);
        ++seq;
    };
    auto header = [&](int slot, int type, int item, int base, int n, int aux, int aux2) {
        if (lane == 0) {
            StageHdr &h = sm.hdr[slot];
            h.type = type; h.item = item; h.base = base; h.n = n; h.aux = aux; h.aux2 = aux2;
        }
    };
    auto bar_of = [&](int slot) { return &sm.full[slot]; };
    // the header (and any per-stage fields the lanes wrote) becomes visible to the consumers
    auto publish = [&](int slot) {
        __syncwarp();
        if (lane == 0) mbar_arrive(&sm.hbar[slot]);
        __syncwarp();
    };

    for (int item = blockIdx.x; item < p.n_items; item += gridDim.x) {
        const int unit = item / p.S, split = item % p.S;
        const int t0 = split * p.tps, t1 = min(p.T, t0 + p.tps);
        const int c0 = min(p.L, split * p.txs), c1 = min(p.L, c0 + p.txs);
        const size_t ubase = (size_t)unit * p.T;
        int slot;

        // rank-mask words of this split, once per item
        for (int i = lane; i < (t1 - t0 + 31) / 32; i += 32) {
            const int widx = t0 / 32 + i;
            sm.mask_words[i] = (widx < p.nwords) ? p.mask[(size_t)unit * p.nwords + widx] : 0u;
        }
        __syncwarp();

        // query rows of the unit's heads (Hg x 256 B)
        if ((slot = acquire()) < 0) break;
        header(slot, ST_Q, item, 0, 0, 0, 0);
        publish(slot);
        {
            const uint16_t *src = p.q + ((size_t)(unit / p.groups) * p.n_q + (size_t)(unit % p.groups) * p.Hg) * 128;
            for (int c = lane; c < p.Hg * 16; c += 32) cp_async16(sm.ring[slot] + 16 * c, src + 8 * c);
        }
        commit(slot, 0, true);

        // B_K, 32 rank rows of one KV head per stage
        bool ok = true;
        for (int j = 0; j < 4 && ok; ++j)
            for (int sub = 0; sub < 2; ++sub) {
                if ((slot = acquire()) < 0) { ok = false; break; }
                header(slot, ST_BK, item, 0, 0, j, sub);
                publish(slot);
                if (lane == 0) {
                    mbar_arrive_tx(bar_of(slot), kStageBytes);
                    tma_2d(sm.ring[slot], &p.tm_bk, j * 128, unit * 64 + 32 * sub, bar_of(slot));
                    tma_2d(sm.ring[slot] + 4096, &p.tm_bk, j * 128 + 64, unit * 64 + 32 * sub, bar_of(slot));
                } else {
                    mbar_arrive(bar_of(slot));
                }
                ++seq;
            }
        if (!ok) break;
        if ((slot = acquire()) < 0) break;
        header(slot, ST_QDONE, item, 0, 0, 0, 0);
        publish(slot);
        commit(slot, 0, false);

        // visual tokens: LO tiles, HI stages of 32 pending full-rank tokens
        int npend = 0, hi_count = 0;
        auto emit_hi = [&](int cnt) -> bool {
            int s2 = acquire();
            if (s2 < 0) return false;
            header(s2, ST_HI, item, t0, cnt, hi_count, 0);
            for (int i = lane; i < cnt; i += 32) sm.hdr[s2].tok[i] = sm.hi_pend[i];
            publish(s2);
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
            commit(s2, 0, true);
            ++hi_count;
            return true;
        };

        for (int tb = t0; tb < t1 && ok; tb += C::kLoT) {
            const int n = min(C::kLoT, t1 - tb);
            if ((slot = acquire()) < 0) { ok = false; break; }
            header(slot, ST_LO, item, tb, n, 0, 0);
            uint32_t word = 0u;
            const int nw = C::kLoT / 32;
            if (lane < nw) {
                const int widx = tb / 32 + lane;
                word = (widx < p.nwords) ? sm.mask_words[widx - t0 / 32] : 0u;
                const int lo_tok = 32 * lane;
                if (lo_tok >= n) word = 0u;
                else if (n - lo_tok < 32) word &= (1u << (n - lo_tok)) - 1u;
                sm.hdr[slot].mask[lane] = word;
            }
            publish(slot);
            if (lane == 0) {
                mbar_arrive_tx(bar_of(slot), C::kLoT * 64);
                tma_2d(sm.ring[slot], &p.tm_ck, 0, (int)(ubase + tb), bar_of(slot));
                tma_2d(sm.ring[slot] + 4096, &p.tm_cv, 0, (int)(ubase + tb), bar_of(slot));
            } else {
                mbar_arrive(bar_of(slot));
            }
            ++seq;

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
                publish(slot);
                if (lane == 0) {
                    const int row = unit * p.Lcap + ct;
                    mbar_arrive_tx(bar_of(slot), kStageBytes);
                    tma_3d(sm.ring[slot], &p.tm_kt, 0, j, row, bar_of(slot));
                    tma_3d(sm.ring[slot] + 2048, &p.tm_kt, 64, j, row, bar_of(slot));
                    tma_3d(sm.ring[slot] + 4096, &p.tm_vt, 0, j, row, bar_of(slot));
                    tma_3d(sm.ring[slot] + 6144, &p.tm_vt, 64, j, row, bar_of(slot));
                } else {
                    mbar_arrive(bar_of(slot));
                }
                ++seq;
            }
        }
        if (!ok) break;

        if ((slot = acquire()) < 0) break;
        header(slot, ST_END, item, 0, 0, 0, 0);
        publish(slot);
        commit(slot, 0, false);

        // B_V rows of the KV heads this split writes outputs for
        const int jm = output_kv_heads(p, split);
        for (int j = 0; j < 4 && ok; ++j) {
            if (!((jm >> j) & 1)) continue;
            for (int sub = 0; sub < 2; ++sub) {
                if ((slot = acquire()) < 0) { ok = false; break; }
                header(slot, ST_BV, item, 0, 0, j, sub);
                publish(slot);
                if (lane == 0) {
                    mbar_arrive_tx(bar_of(slot), kStageBytes);
                    tma_2d(sm.ring[slot], &p.tm_bv, j * 128, unit * 64 + 32 * sub, bar_of(slot));
                    tma_2d(sm.ring[slot] + 4096, &p.tm_bv, j * 128 + 64, unit * 64 + 32 * sub, bar_of(slot));
                } else {
                    mbar_arrive(bar_of(slot));
                }
                ++seq;
            }
        }
        if (!ok) break;
        if ((slot = acquire()) < 0) break;
        header(slot, ST_FIN, item, 0, 0, 0, 0);
        publish(slot);
        commit(slot, 0, false);
    }
    int slot = acquire();
    if (slot >= 0) {
        header(slot, ST_STOP, -1, 0, 0, 0, 0);
        publish(slot);
        commit(slot, 0, false);
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

    float vm[2], vl[2], u[8][4];          // visual softmax state, u^T accumulator (rank space)
    float tm[2], tl[2], w[16][4];         // text softmax state, w^T accumulator (head space)
    uint32_t qah[4], qal[4];              // q~ A fragments, rank 0..15 (hi / lo)

    auto reset_state = [&]() {
        vm[0] = vm[1] = tm[0] = tm[1] = -INFINITY;
        vl[0] = vl[1] = tl[0] = tl[1] = 0.f;
        #pragma unroll
        for (int a = 0; a < 8; ++a) u[a][0] = u[a][1] = u[a][2] = u[a][3] = 0.f;
        #pragma unroll
        for (int a = 0; a < 16; ++a) w[a][0] = w[a][1] = w[a][2] = w[a][3] = 0.f;
    };
    auto clear_acc = [&]() {
        if (ctid < kMaxHeads) sm.acc_l[ctid] = 0.f;
    };
    reset_state();
    clear_acc();
    csync(&sm.cbar, cphase, abort);

    const uint32_t qa_base[2] = {smem_u32(&sm.qa[0][0][0]), smem_u32(&sm.qa[1][0][0])};
    int item = -1, unit = 0, split = 0, t0 = 0, t1 = 0;
    int held_slot = -1;       // first B_V stage of a pair, kept until the second arrives

    for (uint32_t seq = 0;; ++seq) {
        const int slot = seq % kStages;
        const uint32_t k = seq / kStages;
        __syncwarp();   // every lane is past the previous stage's release
        const bool hok = mbar_wait(&sm.hbar[slot], k & 1u, abort);
        const StageHdr &hd = sm.hdr[slot];
        int type = hok ? hd.type : ST_STOP;
        // does this warp read the stage's data?  Stages it skips are released without
        // waiting for their data to land.
        bool mine = true;
        if (type == ST_BK) mine = warp == ((2 * hd.aux + hd.aux2) & 7);
        else if (type == ST_BV) mine = (warp >> 1) == hd.aux;
        else if (type == ST_TEXT) mine = warp == 4 * (hd.aux2 & 1) + hd.aux;
        else if (type == ST_HI) mine = ((win - 2 * hd.aux) % C::kWPM + C::kWPM) % C::kWPM < 2;
        if (type != ST_STOP && mine && !mbar_wait(&sm.full[slot], k & 1u, abort)) type = ST_STOP;
        const unsigned char *st = sm.ring[slot];
        const uint32_t sbase = smem_u32(st);

        if (type == ST_Q) {
            item = hd.item;
            unit = item / p.S; split = item % p.S;
            t0 = split * p.tps; t1 = min(p.T, t0 + p.tps);
            for (int c = ctid; c < 4 * 16 * 16; c += kConsumers) {
                const int j = c >> 8, rr = (c >> 4) & 15, ch = c & 15;
                uint4 v = make_uint4(0u, 0u, 0u, 0u);
                if (rr < p.per_kv) v = *reinterpret_cast<const uint4 *>(st + (j * p.per_kv + rr) * 256 + 16 * ch);
                *reinterpret_cast<uint4 *>(reinterpret_cast<unsigned char *>(&sm.qtxt[j][rr][0]) + ((ch ^ (rr & 7)) << 4)) = v;
            }
            for (int i = ctid; i < 2 * kMaxHeads * 64 / 8; i += kConsumers) zero16(reinterpret_cast<uint4 *>(&sm.qa[0][0][0]) + i);
            csync(&sm.cbar, cphase, abort);
        } else if (type == ST_BK) {
            // q~[h][32 sub + n] = sum_d q_h[d] B_K[32 sub + n][128 j + d] for the heads of KV head j
            const int j = hd.aux, sub = hd.aux2;
            if (warp == ((2 * j + sub) & 7)) {
                const uint32_t qb = smem_u32(&sm.qtxt[j][0][0]);
                float acc[4][4];
                #pragma unroll
                for (int a = 0; a < 4; ++a) acc[a][0] = acc[a][1] = acc[a][2] = acc[a][3] = 0.f;
                #pragma unroll
                for (int kb = 0; kb < 8; ++kb) {
                    uint32_t a[4];
                    {
                        const int row = (lane & 7) + (((lane >> 3) & 1) << 3);
                        const int ch = 2 * kb + (lane >> 4);
                        ldsm_x4(qb + row * 256 + ((ch ^ (row & 7)) << 4), a[0], a[1], a[2], a[3]);
                    }
                    #pragma unroll
                    for (int np = 0; np < 2; ++np) {
                        uint32_t b0, b1, b2, b3;
                        const int row = 16 * np + (lane & 7) + ((lane >> 4) << 3);
                        const int c = 2 * kb + ((lane >> 3) & 1);
                        ldsm_x4(sbase + (c >> 3) * 4096 + row * 128 + ((((c & 7) ^ (row & 7))) << 4), b0, b1, b2, b3);
                        mma_bf16(acc[2 * np], a, b0, b1);
                        mma_bf16(acc[2 * np + 1], a, b2, b3);
                    }
                }
                #pragma unroll
                for (int nb = 0; nb < 4; ++nb)
                    #pragma unroll
                    for (int e = 0; e < 4; ++e) {
                        const int rr = g + 8 * (e >> 1);
                        if (rr < p.per_kv) {
                            const int h = j * p.per_kv + rr;
                            const int i = 32 * sub + 8 * nb + 2 * tig + (e & 1);
                            const float v = acc[nb][e];
                            const uint16_t hi = float_to_bf16_bits(v);
                            const uint16_t lo = float_to_bf16_bits(v - bf16_bits_to_float(hi));
                            const uint32_t off = ((((i >> 3) ^ (h & 7)) & 7) << 4) + (i & 7) * 2;
                            *reinterpret_cast<uint16_t *>(reinterpret_cast<unsigned char *>(&sm.qa[0][h][0]) + off) = hi;
                            *reinterpret_cast<uint16_t *>(reinterpret_cast<unsigned char *>(&sm.qa[1][h][0]) + off) = lo;
                        }
                    }
            }
        } else if (type == ST_QDONE) {
            csync(&sm.cbar, cphase, abort);
            const int row = 16 * mb + (lane & 7) + (((lane >> 3) & 1) << 3);
            const int ch = lane >> 4;
            const uint32_t off = row * 128 + ((ch ^ (row & 7)) << 4);
            ldsm_x4(qa_base[0] + off, qah[0], qah[1], qah[2], qah[3]);
            ldsm_x4(qa_base[1] + off, qal[0], qal[1], qal[2], qal[3]);
        } else if (type == ST_LO) {
            const int base = hd.base, n = hd.n;
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
                        const int c = 2 * kb + ((lane >> 3) & 1);
                        ldsm_x4(sbase + (c >> 3) * 2048 + row * 128 + ((((c & 7) ^ (row & 7))) << 4), b0, b1, b2, b3);
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
                    const int c = 2 * pr + (lane >> 4);
                    ldsm_x4_t(sbase + 4096 + (c >> 3) * 2048 + row * 128 + ((((c & 7) ^ (row & 7))) << 4), b0, b1, b2, b3);
                    mma_bf16(w[2 * pr], pa, b0, b1);
                    mma_bf16(w[2 * pr + 1], pa, b2, b3);
                }
            }
        } else if (type == ST_BV) {
            // o_h = (u_h / l_h) B_V[:, 128 j + d] + w_h / l_h for the output heads of KV head j:
            // warps 2j and 2j+1 take output columns [0, 64) and [64, 128); they keep the first of
            // the two 32-row stages until the second arrives and run both through mma.sync
            const int j = hd.aux, sub = hd.aux2;
            if ((warp >> 1) == j) {
                if (sub == 0) {
                    held_slot = slot;
                } else if (held_slot >= 0) {
                    const int dh = warp & 1;
                    const int h = j * p.per_kv + g;
                    const bool valid = (g < p.per_kv) && (h % p.S == split);
                    float o[8][4];
                    #pragma unroll
                    for (int a2 = 0; a2 < 8; ++a2) o[a2][0] = o[a2][1] = o[a2][2] = o[a2][3] = 0.f;
                    #pragma unroll
                    for (int half = 0; half < 2; ++half) {
                        const uint32_t bbase = smem_u32(sm.ring[half == 0 ? held_slot : slot]) + dh * 4096;
                        #pragma unroll
                        for (int kb = 0; kb < 2; ++kb) {
                            const int i0 = 32 * half + 16 * kb + 2 * tig;
                            float a0 = 0.f, a1 = 0.f, a2 = 0.f, a3 = 0.f;
                            if (valid) {
                                a0 = sm.acc_u[h][i0]; a1 = sm.acc_u[h][i0 + 1];
                                a2 = sm.acc_u[h][i0 + 8]; a3 = sm.acc_u[h][i0 + 9];
                            }
                            uint32_t ah[4], al[4];
                            split2(a0, a1, ah[0], al[0]);
                            split2(a2, a3, ah[2], al[2]);
                            ah[1] = ah[3] = al[1] = al[3] = 0u;
                            #pragma unroll
                            for (int np = 0; np < 4; ++np) {
                                uint32_t b0, b1, b2, b3;
                                const int row = 16 * kb + (lane & 7) + (((lane >> 3) & 1) << 3);
                                const int ch = 2 * np + (lane >> 4);
                                ldsm_x4_t(bbase + row * 128 + ((((ch ^ (row & 7))) & 7) << 4), b0, b1, b2, b3);
                                mma_bf16(o[2 * np], ah, b0, b1);
                                mma_bf16(o[2 * np], al, b0, b1);
                                mma_bf16(o[2 * np + 1], ah, b2, b3);
                                mma_bf16(o[2 * np + 1], al, b2, b3);
                            }
                        }
                    }
                    if (valid) {
                        const int lb = unit / p.groups, G = unit % p.groups;
                        uint16_t *orow = p.out + ((size_t)lb * p.n_q + (size_t)G * p.Hg + h) * 128;
                        #pragma unroll
                        for (int nb = 0; nb < 8; ++nb) {
                            const int d = 64 * dh + 8 * nb + 2 * tig;
                            const uint32_t v = pack_bf16(o[nb][0] + sm.acc_w[h][d], o[nb][1] + sm.acc_w[h][d + 1]);
                            *reinterpret_cast<uint32_t *>(orow + d) = v;
                        }
                    }
                }
            }
        }

        __syncwarp();
        if (lane == 0) {
            if (type == ST_BV && held_slot == slot) {
                // released together with the second stage of the pair
            } else {
                mbar_arrive(&sm.empty[slot]);
                if (type == ST_BV && held_slot >= 0 && held_slot != slot) mbar_arrive(&sm.empty[held_slot]);
            }
        }
        if (type == ST_BV && held_slot >= 0 && held_slot != slot) held_slot = -1;
        if (type == ST_STOP) break;

        if (type == ST_FIN) {
            csync(&sm.cbar, cphase, abort);
            clear_acc();
            reset_state();
            continue;
        }
        if (type != ST_END) continue;

        // ============================ epilogue of the item's tokens
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
        // every warp is past its token stages: the q staging area is dead and becomes the merge buffer
        for (int i = ctid; i < 6 * 32 * 32; i += kConsumers) (&sm.frag_u[0][0][0])[i] = 0.f;
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
        // rescale this warp's partials to the block maximum and add them up in register order:
        // one warp-wide atomic touches 32 consecutive words (no bank conflicts)
        #pragma unroll
        for (int r = 0; r < 2; ++r) {
            const int h = 16 * mb + g + 8 * r;
            const float f = (h < Hg && vm[r] != -INFINITY) ? ex2(vm[r] - sm.mcta[h]) : 0.f;
            #pragma unroll
            for (int nb = 0; nb < 8; ++nb) {
                atomicAdd(&sm.frag_u[mb][4 * nb + 2 * r][lane], u[nb][2 * r] * f);
                atomicAdd(&sm.frag_u[mb][4 * nb + 2 * r + 1][lane], u[nb][2 * r + 1] * f);
            }
            if (tig == 0 && f != 0.f) atomicAdd(&sm.acc_l[h], vl[r] * f);
        }
        {
            // text rows: KV head jt has per_kv <= 8 query heads, all in row g (r = 0)
            const bool row_ok = g < p.per_kv;
            const int ht = jt * p.per_kv + g;
            const float f = (row_ok && tm[0] != -INFINITY) ? ex2(tm[0] - sm.mcta[ht]) : 0.f;
            #pragma unroll
            for (int nb = 0; nb < 16; ++nb) {
                atomicAdd(&sm.frag_w[jt][2 * nb][lane], w[nb][0] * f);
                atomicAdd(&sm.frag_w[jt][2 * nb + 1][lane], w[nb][1] * f);
            }
            if (tig == 0 && f != 0.f) atomicAdd(&sm.acc_l[ht], tl[0] * f);
        }
        csync(&sm.cbar, cphase, abort);
        // register order -> [head][column]
        for (int i = ctid; i < Hg * 64; i += kConsumers) {
            const int h = i >> 6, c = i & 63, hh = h & 15;
            sm.acc_u[h][c] = sm.frag_u[h >> 4][4 * (c >> 3) + 2 * (hh >> 3) + (c & 1)][4 * (hh & 7) + ((c & 7) >> 1)];
        }
        for (int i = ctid; i < Hg * 128; i += kConsumers) {
            const int h = i >> 7, d = i & 127;
            const int j = h / p.per_kv, rr = h % p.per_kv;
            sm.acc_w[h][d] = sm.frag_w[j][2 * (d >> 3) + (d & 1)][4 * rr + ((d & 7) >> 1)];
        }
        csync(&sm.cbar, cphase, abort);

        if (p.S > 1) {
            // publish this split's (max, sum) and (u, w), then wait for the unit's other splits
            float *mlu = p.ml + (size_t)unit * p.S * Hg * 2;
            float *uwu = p.uw + (size_t)unit * p.S * Hg * kUW;
            if (ctid < Hg) {
                mlu[((size_t)split * Hg + ctid) * 2] = sm.mcta[ctid];
                mlu[((size_t)split * Hg + ctid) * 2 + 1] = sm.acc_l[ctid];
            }
            for (int i = ctid; i < Hg * kUW; i += kConsumers) {
                const int h = i / kUW, f = i % kUW;
                uwu[(size_t)split * Hg * kUW + i] = (f < 64) ? sm.acc_u[h][f] : sm.acc_w[h][f - 64];
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
                    __nanosleep(128);
                }
            }
            csync(&sm.cbar, cphase, abort);
            // unit-wide max and sum per head: one warp per head, lanes over splits
            for (int h = warp; h < Hg; h += kConsumerWarps) {
                float mloc = -INFINITY;
                for (int s2 = lane; s2 < p.S; s2 += 32) mloc = fmaxf(mloc, __ldcg(mlu + ((size_t)s2 * Hg + h) * 2));
                #pragma unroll
                for (int d = 16; d > 0; d >>= 1) mloc = fmaxf(mloc, __shfl_xor_sync(0xffffffffu, mloc, d));
                float lsum = 0.f;
                for (int s2 = lane; s2 < p.S; s2 += 32) {
                    const float ms = __ldcg(mlu + ((size_t)s2 * Hg + h) * 2);
                    if (ms != -INFINITY) lsum += __ldcg(mlu + ((size_t)s2 * Hg + h) * 2 + 1) * ex2(ms - mloc);
                }
                #pragma unroll
                for (int d = 16; d > 0; d >>= 1) lsum += __shfl_xor_sync(0xffffffffu, lsum, d);
                if (lane == 0) {
                    sm.mfin[h] = mloc;
                    sm.invl[h] = 1.f / lsum;
                }
            }
            csync(&sm.cbar, cphase, abort);
            // combined u / l and w / l of this split's output heads, all (head, feature) pairs in parallel
            const int n_out = (split < Hg) ? (Hg - split + p.S - 1) / p.S : 0;
            for (int task = ctid; task < n_out * kUW; task += kConsumers) {
                const int h = split + (task / kUW) * p.S, f = task % kUW;
                const float mh = sm.mfin[h];
                float a0 = 0.f, a1 = 0.f, a2 = 0.f, a3 = 0.f;
                int s2 = 0;
                for (; s2 + 4 <= p.S; s2 += 4) {
                    const float m0 = __ldcg(mlu + ((size_t)(s2 + 0) * Hg + h) * 2);
                    const float m1 = __ldcg(mlu + ((size_t)(s2 + 1) * Hg + h) * 2);
                    const float m2 = __ldcg(mlu + ((size_t)(s2 + 2) * Hg + h) * 2);
                    const float m3 = __ldcg(mlu + ((size_t)(s2 + 3) * Hg + h) * 2);
                    const float x0 = __ldcg(uwu + ((size_t)(s2 + 0) * Hg + h) * kUW + f);
                    const float x1 = __ldcg(uwu + ((size_t)(s2 + 1) * Hg + h) * kUW + f);
                    const float x2 = __ldcg(uwu + ((size_t)(s2 + 2) * Hg + h) * kUW + f);
                    const float x3 = __ldcg(uwu + ((size_t)(s2 + 3) * Hg + h) * kUW + f);
                    if (m0 != -INFINITY) a0 = fmaf(x0, ex2(m0 - mh), a0);
                    if (m1 != -INFINITY) a1 = fmaf(x1, ex2(m1 - mh), a1);
                    if (m2 != -INFINITY) a2 = fmaf(x2, ex2(m2 - mh), a2);
                    if (m3 != -INFINITY) a3 = fmaf(x3, ex2(m3 - mh), a3);
                }
                for (; s2 < p.S; ++s2) {
                    const float m0 = __ldcg(mlu + ((size_t)s2 * Hg + h) * 2);
                    const float x0 = __ldcg(uwu + ((size_t)s2 * Hg + h) * kUW + f);
                    if (m0 != -INFINITY) a0 = fmaf(x0, ex2(m0 - mh), a0);
                }
                const float v = ((a0 + a1) + (a2 + a3)) * sm.invl[h];
                if (f < 64) sm.acc_u[h][f] = v;
                else sm.acc_w[h][f - 64] = v;
            }
        } else {
            if (ctid < Hg) {
                sm.mfin[ctid] = sm.mcta[ctid];
                sm.invl[ctid] = 1.f / sm.acc_l[ctid];
            }
            csync(&sm.cbar, cphase, abort);
            for (int i = ctid; i < Hg * kUW; i += kConsumers) {
                const int h = i / kUW, f = i % kUW;
                if (f < 64) sm.acc_u[h][f] *= sm.invl[h];
                else sm.acc_w[h][f - 64] *= sm.invl[h];
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
        // the BV stages that follow add u B_V into acc_w; FIN writes the outputs
    }
}

template <int NMB>
__global__ void __launch_bounds__(kThreads, 1) attn_kernel(const __grid_constant__ Params p) {
    extern __shared__ __align__(1024) unsigned char smem_raw[];
    // the ring must start on a 1024-byte boundary (128-byte swizzle pattern)
    const uint32_t base = smem_u32(smem_raw);
    unsigned char *aligned = smem_raw + ((1024u - (base & 1023u)) & 1023u);
    Smem<NMB> &sm = *reinterpret_cast<Smem<NMB> *>(aligned);
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    if (threadIdx.x == 0) {
        for (int s = 0; s < kStages; ++s) {
            mbar_init(&sm.hbar[s], 1);
            mbar_init(&sm.full[s], 32);
            mbar_init(&sm.empty[s], kConsumerWarps);
        }
        mbar_init(&sm.cbar, kConsumerWarps);
        sm.abort = 0;
        asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
    }
    __syncthreads();
    if (warp == kConsumerWarps) producer<NMB>(p, sm, lane);
    else consumers<NMB>(p, sm, warp, lane);
}

template <int NMB>
constexpr size_t smem_bytes() { return sizeof(Smem<NMB>) + 1024; }

}  // namespace decode
}  // namespace kvpack
