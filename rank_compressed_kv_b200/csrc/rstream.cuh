// rstream.cuh -- the visual half of an AttentionPack decode step as two streaming
// passes over the rank-compressed cache, with the scores on the 5th-generation
// tensor cores.
//
// Method ("Attention-aware Inference Optimizations for Large Vision-Language
// Models with Memory-efficient Decoding", technical summaries 2.B on the
// es / fr / de pages): a token with a high importance score is decompressed at
// the full rank, the others at a quarter of it (or, in the de summary's
// variant, not at all).  Decompression is folded into the attention by
// associativity: with q~ = B_K[:, slice] q in rank space, a token's logit is
// C_K[t, :rho_t] . q~[:rho_t]; the softmax-weighted V coefficients are summed
// in rank space and projected through B_V once per head (finish kernel).
//
//   stats pass  per segment of a unit's tokens: max and sum of 2^s per query
//               head (s = the logit in the log2 domain), from C_K only
//   value pass  with the unit's final (M, 1/L) per head known (combine
//               kernel): p' = 2^(s - M); the attention mass of every token,
//               sum_h p'_h / L_h; and u_h = sum_t p'_t C_V[t, :rho_t]
//
// Work split: the units' tokens, flattened in 128-token tiles, are cut into
// one contiguous range per CTA; a CTA walks its range unit by unit
// ("segments") and writes one partial per segment, so a unit has at most a
// few partials whatever its length.
//
// A CTA has eight warps:
//   warp 0     producer: per 512-token block of the segment, one TMA tile of
//              the C_lo rows (K, and V in the value pass; 32-byte rows,
//              32-byte swizzle) unless every token of the block is full-rank;
//              the block's full-rank tokens are counted, and every 128 of them
//              (and the rest at the segment's end) make a HI tile: a run of the
//              unit's list of full-rank positions (hipos_kernel, ahead of the
//              passes) lands in the tile's descriptor by bulk copy; the unit's
//              q~ (bf16 hi and lo planes) by bulk copy per segment
//   warp 1     tensor memory owner and MMA issuer: per tile, S = C q~^T with
//              tokens on M = 128 (the tensor-memory lanes) and the query heads
//              on N, as two bf16 products (q~ hi, q~ lo) accumulated in fp32:
//              K = 16 (one k-step) for a LO sub-tile, 64 (four) for a HI tile
//   warps 2-5  consumers: thread = token.  Each reads its token's logits for
//              every head from tensor memory (tcgen05.ld) and does the
//              per-token work; in the value pass it writes its row of p' to
//              shared memory, and the warp adds u^T += C_V^T P for its 32 tokens
//              with mma.sync (ranks on M, heads on N).
//   warps 6-7  gather: a HI tile's rows, 128 bytes each (C_lo + C_hi, 128-byte
//              swizzle), by cp.async from the positions in its descriptor
// Every ring slot carries a descriptor of its tile; one barrier triple per slot
// (data landed / scores ready / slot free) orders the roles, and a slot's
// tensor-memory score buffer is reused with the slot.
#pragma once

#include <cuda.h>

#include "common.cuh"
#include "decode.cuh"
#include "quant.cuh"

namespace kvpack {
namespace decode {
namespace rs {

constexpr int kGatherWarp = 6;              // warps 6 and 7 gather the full-rank tokens' rows
constexpr int kConsumer2 = 8;               // warps 8-11: the second consumer group (kSplit = 2)
constexpr int kGatherThreads = 64;
constexpr int kND = 12;                     // descriptor ring (written by the producer, freed by the consumers)
constexpr int kNQ = 4;                      // queue of full-rank tiles handed to the gather warp
constexpr int kTile = 128;          // tokens per tensor-memory tile (M of the score MMA)
constexpr int kDescInts = 8 + 68;   // header + up to 16 mask words (LO) or 8 + 128 uint16 positions (HI)
constexpr int kTypeLo = 0, kTypeHi = 1, kTypeEnd = 2;
constexpr int kFlagFirst = 1 << 8, kFlagLast = 1 << 9;
constexpr float kRefInit = -1e30f;
constexpr float kLazy = 8.f;        // a per-thread reference sits 2^8 above the largest logit at its last move

// Geometry per (query heads NH, pass).  NH is the unit's Hg rounded up to 4, 8, 16, 28 or 32.  In the
// 28-head form the two consumer groups' 14 heads sit at tensor-memory columns 0-13 and 16-29 (the
// q~ rows of heads 14-27 two rows lower), so each group's loads start on a 16-column boundary.
// Three rings per CTA, released independently:
//   K slots   the C_K part of a tile: a LO tile of 512 tokens of 32-byte rows or a HI tile of 128
//             tokens of 128-byte rows, 16 KB, freed by the score MMA's completion
//             (tcgen05.commit) -- the consumers never read them
//   V slots   the C_V part of a value-pass tile (the same geometry, 16 KB), freed by the consumers
//             after their V sums
//   S buffers tensor-memory scores of a tile (kSub x kNHP columns), freed by the consumers
template <int NH, bool VALUE>
struct Cfg {
    static constexpr int kNHP = NH < 16 ? 16 : (NH + 15) / 16 * 16;  // N of the score MMA
    // consumer warp groups: each has four warps (one per tensor-memory lane quarter) and NH / kSplit heads
    // (measured: two groups pay off at 32 heads; at 16 they run no faster than one group of two CTAs per SM)
    static constexpr int kSplit = NH >= 28 ? 2 : 1;
    static constexpr int kHS = NH / kSplit;
    static constexpr int kPHS = kHS <= 8 ? 8 : kHS <= 16 ? 16 : 32;   // heads per row of a group's P (mma.sync n8 tiles)
    static constexpr int kGCol = kNHP / kSplit;                      // tensor-memory columns of a group
    static constexpr int kThreads = (8 + 4 * (kSplit - 1)) * 32;
    static constexpr int kBlocks = NH <= 16 ? 2 : 1;                 // resident CTAs per SM
    static constexpr int kLoTok = 512;                               // tokens per LO tile
    static constexpr int kHiTok = 128;                               // tokens per HI tile
    static constexpr int kSub = kLoTok / kTile;                      // 128-token sub-tiles per LO tile
    static constexpr int kKBytes = 16384;
    static constexpr int kVBytes = 16384;
    // the V slots stay with a tile until its consumers are done, the K slots only until its score
    // MMA is (which runs up to kNS tiles ahead of them): the value pass holds more V than K slots
    static constexpr int kNK = VALUE ? (NH <= 16 ? 2 : 5) : (NH <= 16 ? 5 : 10);
    static constexpr int kNV = VALUE ? (NH <= 16 ? 3 : 5) : 1;
    static constexpr int kMaskWin = VALUE && NH <= 16 ? 512 : 1024;   // producer's window of mask words
    static constexpr int kNS = 4;
    static constexpr int kSCols = kSub * kNHP;                       // tensor-memory columns of one S buffer
    static constexpr int kTmemCols = kNS * kSCols;                   // 128, 256 or 512
    static_assert(kTmemCols == 128 || kTmemCols == 256 || kTmemCols == 512, "power-of-two allocation");
    static_assert(kLoTok / 32 <= 16 && kHiTok <= 128, "descriptor capacity");
};

struct Params {
    CUtensorMap tm_ck, tm_cv;       // C_lo planes: 3D {16, T, units}, box {16, 256, 1}, 32-byte swizzle
    const uint16_t *CK_lo, *CK_hi, *CV_lo, *CV_hi;
    const uint8_t *QK_lo, *QK_hi, *QV_lo, *QV_hi;   // 4-bit planes (quant.cuh), when the kernel is Q4
    const int8_t *EK, *EV;                           // their exponents [units][T][2]
    const unsigned char *qt;        // [units][qblock_bytes(Hg)]: q~ hi, lo planes (from text_kernel)
    const uint32_t *mask;           // [units][nwords]
    const uint16_t *hipos;          // [units][Tp]: each unit's full-rank token positions, ascending (hipos_kernel)
    const int *hicnt;               // [units][tpu]: full-rank tokens of the unit before each tile
    const float *ustat;             // value pass: [units][Hg][2] = (M, 1/L)
    float *part;                    // stats: [units][nslot][Hg][2] = (m, l); value: [units][nslot][Hg][64] = u
    float *mass;                    // value pass: [units][T] or null
    int units, T, Hg, nwords, tpu, nslot, rank0, Tp;
    long long ntiles;               // units * tpu
};

// Flattened 128-token tiles [x0, x1) of CTA c among C: x0 = floor(c NT / C).  The CTA that
// holds tile x is floor(((x + 1) C - 1) / NT); a unit's partial slot is its CTA's offset
// from the CTA holding the unit's first tile.
__host__ __device__ inline long long tile_begin(long long c, long long C, long long NT) { return c * NT / C; }
__host__ __device__ inline long long cta_of_tile(long long x, long long C, long long NT) { return ((x + 1) * C - 1) / NT; }

template <int NH, bool VALUE>
struct Smem {
    using C = Cfg<NH, VALUE>;
    alignas(1024) unsigned char kslot[C::kNK][C::kKBytes];
    alignas(1024) unsigned char vslot[C::kNV][VALUE ? C::kVBytes : 16];
    alignas(1024) unsigned char qbuf[2][2][C::kNHP * 128];          // [q slot][hi, lo][rows of 128 B]
    int kdesc[kND][kDescInts];                                      // tile descriptors, written once by the producer
    int hiq[kNQ][8];                                                // full-rank tiles for the gather warp
    uint32_t mwin[C::kMaskWin];                                     // producer's window of the CTA's mask words
    unsigned char pbuf[VALUE ? 4 * C::kSplit : 1][VALUE ? 32 * C::kPHS * 2 : 16];   // value pass: P rows per consumer warp
    float merge[VALUE ? 3 : 4][VALUE ? NH * 64 : NH * 2];           // partial merge across the consumer warps
    uint64_t kfull[C::kNK], kempty[C::kNK], vfull[C::kNV], vempty[C::kNV], sfull[C::kNS], sfree[C::kNS];
    uint64_t dfree[kND], gready[kNQ], gfree[kNQ];
    uint64_t qfull[2], qempty[2], mdone;
    uint32_t tmem_base;
    int abort;
};

template <int NH, bool VALUE>
constexpr size_t smem_bytes() { return sizeof(Smem<NH, VALUE>) + 1024; }

// resident CTAs per SM as planned: 228 KB of shared memory per SM, 1 KB of it reserved per CTA
template <int NH, bool VALUE>
constexpr bool smem_fits() { return Cfg<NH, VALUE>::kBlocks * (smem_bytes<NH, VALUE>() + 1024) <= 233472; }
static_assert(smem_fits<4, false>() && smem_fits<4, true>() && smem_fits<8, false>() && smem_fits<8, true>(), "smem");
static_assert(smem_fits<16, false>() && smem_fits<16, true>(), "shared memory of two CTAs per SM");
static_assert(smem_fits<28, false>() && smem_fits<28, true>() && smem_fits<32, false>() && smem_fits<32, true>(),
              "shared memory of one CTA per SM");
static_assert(kGatherThreads == 64, "the 4-bit gather assumes 64 threads");

// ------------------------------------------------------------------ tcgen05 helpers

// Shared-memory descriptor of a K-major operand in swizzled 8-row atoms: SBO = byte
// stride between 8-row groups; the leading offset is unused for swizzled K-major tiles.
// swz: 6 = 32-byte swizzle, 2 = 128-byte swizzle.
__device__ __forceinline__ uint64_t desc_kmajor(uint32_t saddr, uint32_t sbo, uint32_t swz) {
    uint64_t d = 0;
    d |= (uint64_t)((saddr >> 4) & 0x3FFFu);
    d |= (uint64_t)1 << 16;
    d |= (uint64_t)((sbo >> 4) & 0x3FFFu) << 32;
    d |= (uint64_t)1 << 46;
    d |= (uint64_t)swz << 61;
    return d;
}

// Instruction descriptor: bf16 x bf16 -> fp32, both operands K-major, M x N.
__host__ __device__ constexpr uint32_t idesc_bf16_kk(int M, int N) {
    return (1u << 4) | (1u << 7) | (1u << 10) | ((uint32_t)(N >> 3) << 17) | ((uint32_t)(M >> 4) << 24);
}

template <int N>
__device__ __forceinline__ void tmem_ld(uint32_t taddr, float (&v)[N]);

template <>
__device__ __forceinline__ void tmem_ld<4>(uint32_t taddr, float (&v)[4]) {
    asm volatile("tcgen05.ld.sync.aligned.32x32b.x4.b32 {%0,%1,%2,%3}, [%4];"
                 : "=f"(v[0]), "=f"(v[1]), "=f"(v[2]), "=f"(v[3]) : "r"(taddr) : "memory");
}
template <>
__device__ __forceinline__ void tmem_ld<8>(uint32_t taddr, float (&v)[8]) {
    asm volatile("tcgen05.ld.sync.aligned.32x32b.x8.b32 {%0,%1,%2,%3,%4,%5,%6,%7}, [%8];"
                 : "=f"(v[0]), "=f"(v[1]), "=f"(v[2]), "=f"(v[3]), "=f"(v[4]), "=f"(v[5]), "=f"(v[6]), "=f"(v[7])
                 : "r"(taddr) : "memory");
}
template <>
__device__ __forceinline__ void tmem_ld<16>(uint32_t taddr, float (&v)[16]) {
    asm volatile(
        "tcgen05.ld.sync.aligned.32x32b.x16.b32 {%0,%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15}, [%16];"
        : "=f"(v[0]), "=f"(v[1]), "=f"(v[2]), "=f"(v[3]), "=f"(v[4]), "=f"(v[5]), "=f"(v[6]), "=f"(v[7]),
          "=f"(v[8]), "=f"(v[9]), "=f"(v[10]), "=f"(v[11]), "=f"(v[12]), "=f"(v[13]), "=f"(v[14]), "=f"(v[15])
        : "r"(taddr) : "memory");
}
template <>
__device__ __forceinline__ void tmem_ld<32>(uint32_t taddr, float (&v)[32]) {
    tmem_ld32(taddr, v);
}

// ------------------------------------------------------------------ the kernel

// Q4: the coefficients are 4-bit (quant.cuh); the gather warps then dequantize every tile, LO and
// HI, into the same shared-memory layouts the TMA and cp.async copies produce, so the score MMA
// and the consumers are unchanged.
template <int NH, bool VALUE, bool Q4>
__global__ void __launch_bounds__(Cfg<NH, VALUE>::kThreads, Cfg<NH, VALUE>::kBlocks) rs_kernel(const __grid_constant__ Params p) {
    using C = Cfg<NH, VALUE>;
    constexpr int kNK = C::kNK, kNV = C::kNV, kNS = C::kNS, kNHP = C::kNHP;
    extern __shared__ __align__(1024) unsigned char smem_raw[];
    const uint32_t base0 = smem_u32(smem_raw);
    Smem<NH, VALUE> &sm = *reinterpret_cast<Smem<NH, VALUE> *>(smem_raw + ((1024u - (base0 & 1023u)) & 1023u));
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    volatile int *abort = &sm.abort;

    const long long NT = p.ntiles, CT = gridDim.x;
    const long long x0 = tile_begin(blockIdx.x, CT, NT), x1 = tile_begin(blockIdx.x + 1, CT, NT);

    if (threadIdx.x == 0) {
        // data slots complete with the producer's 32 lanes and the gather warps' 64 threads
        for (int s = 0; s < kNK; ++s) {
            mbar_init(&sm.kfull[s], 32 + kGatherThreads);
            mbar_init(&sm.kempty[s], 1);
        }
        for (int s = 0; s < kNV; ++s) {
            mbar_init(&sm.vfull[s], 32 + kGatherThreads);
            mbar_init(&sm.vempty[s], 4 * C::kSplit);
        }
        for (int s = 0; s < kND; ++s) mbar_init(&sm.dfree[s], 4 * C::kSplit);
        for (int s = 0; s < kNQ; ++s) {
            mbar_init(&sm.gready[s], 1);
            mbar_init(&sm.gfree[s], kGatherThreads);
        }
        for (int s = 0; s < kNS; ++s) {
            mbar_init(&sm.sfull[s], 1);
            mbar_init(&sm.sfree[s], 4 * C::kSplit);
        }
        for (int s = 0; s < 2; ++s) {
            mbar_init(&sm.qfull[s], 1);
            mbar_init(&sm.qempty[s], 1);
        }
        mbar_init(&sm.mdone, 1);
        sm.abort = 0;
        asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
    }
    // q~ rows past Hg stay zero for the whole kernel (the bulk copies write Hg rows), so the
    // scores of padding heads are exactly zero
    for (int i = threadIdx.x; i < 2 * 2 * kNHP * 128 / 16; i += C::kThreads)
        reinterpret_cast<uint4 *>(&sm.qbuf[0][0][0])[i] = make_uint4(0u, 0u, 0u, 0u);
    fence_proxy_async();
    if (warp == 1) tmem_alloc(&sm.tmem_base, C::kTmemCols);
    tmem_fence_before();
    __syncthreads();
    tmem_fence_after();
    const uint32_t tmem = sm.tmem_base;
    // everything above overlaps the previous kernel's tail; its outputs (q~, the unit
    // statistics) are read only from here on
    griddep_launch_dependents();
    griddep_wait();

    if (warp == 0) {
        // =============================================================== producer
        uint32_t seq = 0, qseq = 0;
        bool ok = true;
        // wait until the K slot (and, in the value pass, the V slot) of tile `seq` may be refilled
        auto acquire_k = [&](int ks) -> bool {
            return seq < (uint32_t)kNK || mbar_wait(&sm.kempty[ks], ((seq / kNK) - 1) & 1u, abort);
        };
        auto acquire_v = [&](int vs) -> bool {
            return seq < (uint32_t)kNV || mbar_wait(&sm.vempty[vs], ((seq / kNV) - 1) & 1u, abort);
        };
        // The CTA's mask words are one contiguous run (its tiles are consecutive 128-token tiles
        // and a unit's words follow the previous unit's), read into shared memory a window at a
        // time so that no tile waits on a global load of its mask.
        const long long gw_end = (x1 - 1) / p.tpu * p.nwords +
                                 (min(p.T, (int)((x1 - 1) % p.tpu + 1) * kTile) + 31) / 32;
        long long wbase = -1;
        auto mask_words = [&](long long gw, int nw) -> const uint32_t * {
            if (wbase < 0 || gw < wbase || gw + nw > wbase + C::kMaskWin) {
                wbase = gw;
                const int cnt = (int)min((long long)C::kMaskWin, gw_end - gw);
                __syncwarp();
                for (int i = lane; i < cnt; i += 32) sm.mwin[i] = __ldg(p.mask + gw + i);
                __syncwarp();
            }
            return sm.mwin + (gw - wbase);
        };
        // wait until descriptor ds of tile `seq` may be rewritten (the consumers are done with it)
        auto acquire_d = [&](int ds) -> bool {
            return seq < (uint32_t)kND || mbar_wait(&sm.dfree[ds], ((seq / kND) - 1) & 1u, abort);
        };
        // hand a full-rank tile (K slot ks, V slot vs, descriptor ds) to the gather warps; ks < 0 ends
        // them.  A tile's token positions (pos_bytes from src) land in its descriptor by a bulk copy
        // that completes on the queue entry's barrier, so the gather warps start once they are there.
        uint32_t hseq = 0;
        auto push_gather = [&](int ks, int vs, int ds, int n, int unit, int skew, const uint16_t *src,
                               uint32_t pos_bytes, int type = kTypeHi, int tok = 0) -> bool {
            const int hq = hseq % kNQ;
            if (hseq >= (uint32_t)kNQ && !mbar_wait(&sm.gfree[hq], ((hseq / kNQ) - 1) & 1u, abort)) return false;
            if (lane == 0) {
                int *e = sm.hiq[hq];
                e[0] = ks; e[1] = vs; e[2] = ds; e[3] = n; e[4] = unit; e[5] = skew; e[6] = type; e[7] = tok;
                if (pos_bytes > 0) {
                    fence_proxy_async();   // the descriptor's earlier readers went through the generic proxy
                    mbar_arrive_tx(&sm.gready[hq], pos_bytes);
                    bulk_g2s(sm.kdesc[ds] + 8, src, pos_bytes, &sm.gready[hq]);
                } else {
                    mbar_arrive(&sm.gready[hq]);
                }
            }
            ++hseq;
            return true;
        };
        // full-rank tokens of the CTA's first unit before its first tile: a unit's list of full-rank
        // positions starts at its first token, and only the CTA's first segment can start inside a unit
        int hi_first = 0;
        if (lane == 0 && x0 < x1 && x0 % p.tpu != 0) hi_first = __ldg(p.hicnt + x0);
        hi_first = __shfl_sync(0xffffffffu, hi_first, 0);
        long long x = x0;
        while (ok && x < x1) {
            const int unit = (int)(x / p.tpu);
            const long long ue = (long long)(unit + 1) * p.tpu;
            const long long xe = x1 < ue ? x1 : ue;
            const int tok0 = (int)(x - (long long)unit * p.tpu) * kTile;
            const int tok1 = min(p.T, (int)(xe - (long long)unit * p.tpu) * kTile);
            const int pslot = (int)(blockIdx.x - cta_of_tile((long long)unit * p.tpu, CT, NT));
            const size_t hi_base = (size_t)unit * p.Tp + (x == x0 ? hi_first : 0);
            x = xe;
            // the unit's q~ into the next q slot
            const int qs = qseq & 1;
            if (qseq >= 2 && !mbar_wait(&sm.qempty[qs], ((qseq >> 1) - 1) & 1u, abort)) { ok = false; break; }
            if (lane == 0) {
                const unsigned char *src = p.qt + (size_t)unit * qblock_bytes(p.Hg);
                const uint32_t bytes = (uint32_t)p.Hg * 128u;
                fence_proxy_async();
                mbar_arrive_tx(&sm.qfull[qs], 2 * bytes);
                if (NH == 28 && p.Hg > 14) {
                    // heads 14 .. Hg-1 two rows lower (columns 16 on of the scores)
                    const uint32_t b0 = 14u * 128u, b1 = bytes - b0;
                    for (int pl = 0; pl < 2; ++pl) {
                        bulk_g2s(&sm.qbuf[qs][pl][0], src + pl * bytes, b0, &sm.qfull[qs]);
                        bulk_g2s(&sm.qbuf[qs][pl][16 * 128], src + pl * bytes + b0, b1, &sm.qfull[qs]);
                    }
                } else {
                    bulk_g2s(&sm.qbuf[qs][0][0], src, bytes, &sm.qfull[qs]);
                    bulk_g2s(&sm.qbuf[qs][1][0], src + bytes, bytes, &sm.qfull[qs]);
                }
            }
            ++qseq;
            bool first = true;
            unsigned hi_head = 0, hi_tail = 0;   // the segment's full-rank tokens: emitted, passed
            for (int tok = tok0; tok < tok1 && ok; tok += C::kLoTok) {
                const int n = min(C::kLoTok, tok1 - tok);
                // the block's mask words (bits past n cleared) and its count of full-rank tokens
                const uint32_t *mw = mask_words((long long)unit * p.nwords + (tok >> 5), (n + 31) >> 5);
                uint32_t wd = 0u;
                if (lane < C::kLoTok / 32 && 32 * lane < n) {
                    wd = mw[lane];
                    const int nb = n - 32 * lane;
                    if (nb < 32) wd &= (1u << nb) - 1u;
                }
                const int nhi = (int)__reduce_add_sync(0xffffffffu, (unsigned)__popc(wd));
                hi_tail += (unsigned)nhi;
                const bool final_blk = tok + C::kLoTok >= tok1;
                const unsigned pend = hi_tail - hi_head;
                const int hi_now = (int)(pend / C::kHiTok) + ((final_blk && (pend % C::kHiTok) != 0) ? 1 : 0);
                if (nhi < n) {
                    // ------------------------------------------------ LO tile
                    const int ks = seq % kNK, ds = seq % kND, vs = seq % kNV;
                    if (!acquire_k(ks) || !acquire_d(ds) || (VALUE && !acquire_v(vs))) { ok = false; break; }
                    int *d = sm.kdesc[ds];
                    if (lane == 0) {
                        d[0] = kTypeLo | (first ? kFlagFirst : 0) | ((final_blk && hi_now == 0) ? kFlagLast : 0);
                        d[1] = unit; d[2] = tok; d[3] = n; d[4] = pslot; d[5] = qs;
                    }
                    if (lane < C::kLoTok / 32) d[8 + lane] = (int)wd;
                    first = false;
                    __syncwarp();
                    // lane 0 issues the copies and arrives for itself and for the gather warps
                    // (which have nothing to add to a LO tile); the other lanes' arrivals
                    // release their descriptor writes.  4-bit rows go to the gather warps instead.
                    const int nb = (n + 255) >> 8;   // 256-row boxes of 32-byte rows
                    if (Q4 && !p.rank0) {
                        // 4-bit rows: the producer dequantizes the first half of a LO tile's rows and
                        // the gather warps the second half (they arrive for themselves)
                        const size_t base = (size_t)unit * p.T + tok;
                        if (VALUE)
                            quant::lo_rows_kv<C::kLoTok / 64, 32>(sm.kslot[ks], sm.vslot[vs], p.QK_lo, p.EK, p.QV_lo,
                                                                  p.EV, base, n, lane);
                        else
                            quant::lo_rows<C::kLoTok / 64, 32>(sm.kslot[ks], p.QK_lo, p.EK, base, n, lane);
                        fence_proxy_async();          // the score MMA reads these rows through the async proxy
                        if (!push_gather(ks, vs, ds, n, unit, 0, nullptr, 0u, kTypeLo, tok)) { ok = false; break; }
                        mbar_arrive(&sm.kfull[ks]);
                        if (VALUE) mbar_arrive(&sm.vfull[vs]);
                    } else if (lane == 0) {
                        if (!p.rank0) {
                            fence_proxy_async();
                            mbar_arrive_tx(&sm.kfull[ks], (uint32_t)nb * 8192u);
                            for (int b = 0; b < nb; ++b)
                                tma_3d(sm.kslot[ks] + 8192 * b, &p.tm_ck, 0, tok + 256 * b, unit, &sm.kfull[ks]);
                            if (VALUE) {
                                mbar_arrive_tx(&sm.vfull[vs], (uint32_t)nb * 8192u);
                                for (int b = 0; b < nb; ++b)
                                    tma_3d(sm.vslot[vs] + 8192 * b, &p.tm_cv, 0, tok + 256 * b, unit, &sm.vfull[vs]);
                            }
                        } else {
                            mbar_arrive(&sm.kfull[ks]);
                            if (VALUE) mbar_arrive(&sm.vfull[vs]);
                        }
                        mbar_arrive_cnt(&sm.kfull[ks], kGatherThreads);
                        if (VALUE) mbar_arrive_cnt(&sm.vfull[vs], kGatherThreads);
                    } else {
                        mbar_arrive(&sm.kfull[ks]);
                        if (VALUE) mbar_arrive(&sm.vfull[vs]);
                    }
                    ++seq;
                }
                for (int i = 0; i < hi_now && ok; ++i) {
                    // ------------------------------------------------ HI tile: positions and rows by the gather warps
                    const int ks = seq % kNK, ds = seq % kND, vs = seq % kNV;
                    if (!acquire_k(ks) || !acquire_d(ds) || (VALUE && !acquire_v(vs))) { ok = false; break; }
                    const int nh = (int)min((unsigned)C::kHiTok, hi_tail - hi_head);
                    // the bulk copy starts on a 16-byte boundary of the list (p.Tp is a multiple of 8):
                    // the tile's first position is entry `skew` of the copied run
                    const size_t idx = hi_base + hi_head;
                    const int skew = (int)(idx & 7u);
                    const uint32_t bytes = ((uint32_t)(skew + nh) * 2u + 15u) & ~15u;
                    int *d = sm.kdesc[ds];
                    if (lane == 0) {
                        d[0] = kTypeHi | (first ? kFlagFirst : 0) | ((final_blk && i == hi_now - 1) ? kFlagLast : 0);
                        d[1] = unit; d[2] = skew; d[3] = nh; d[4] = pslot; d[5] = qs;
                    }
                    first = false;
                    __syncwarp();
                    if (!push_gather(ks, vs, ds, nh, unit, skew, p.hipos + (idx - (size_t)skew), bytes)) {
                        ok = false;
                        break;
                    }
                    mbar_arrive(&sm.kfull[ks]);       // releases this lane's descriptor writes
                    if (VALUE) mbar_arrive(&sm.vfull[vs]);
                    hi_head += (unsigned)nh;
                    ++seq;
                }
            }
        }
        // end markers: the K ring's (the MMA warp passes it on to the consumers) and the gather warp's
        bool ended = false;
        if (ok) {
            const int ks = seq % kNK, ds = seq % kND;
            if (acquire_k(ks) && acquire_d(ds)) {
                if (lane == 0) sm.kdesc[ds][0] = kTypeEnd;
                __syncwarp();
                mbar_arrive(&sm.kfull[ks]);
                if (lane == 0) mbar_arrive_cnt(&sm.kfull[ks], kGatherThreads);
                ended = push_gather(-1, 0, 0, 0, 0, 0, nullptr, 0u);
            }
            ok = ended;
        }
        if (!ok) *abort = 1;
        // Copies still in flight (possible only when a role gave up) must land before the block
        // exits: wait for the data phases of the last tiles of each ring.  A parity wait is only
        // meaningful while its phase is the slot's latest, so on the K ring the slot that carried
        // the end marker (whose tile was consumed before the marker could be written) is skipped.
        const uint32_t kfirst = seq >= (uint32_t)kNK ? seq - kNK + (ended ? 1u : 0u) : 0u;
        for (uint32_t k = kfirst; k < seq; ++k) {
            const long long t0 = clock64();
            while (!mbar_try_wait(&sm.kfull[k % kNK], (k / kNK) & 1u) && clock64() - t0 < kWaitCycles) {}
        }
        if (VALUE) {
            for (uint32_t k = (seq > (uint32_t)kNV ? seq - kNV : 0u); k < seq; ++k) {
                const long long t0 = clock64();
                while (!mbar_try_wait(&sm.vfull[k % kNV], (k / kNV) & 1u) && clock64() - t0 < kWaitCycles) {}
            }
        }
    } else if (warp >= kGatherWarp && warp < kGatherWarp + 2) {
        // =============================================================== gather warps
        // 128-byte rows (C_lo + C_hi, 16-byte chunk c of row r at c ^ (r & 7)) of a HI tile's
        // tokens into its K slot (and V slot); V rows past n are zero-filled (their p is zero, and
        // 0 * stale data must stay 0).  Thread g copies chunk g % 8 of rows g / 8 + 8 i, so its
        // source column and its swizzled destination column are fixed.
        const int g = threadIdx.x - kGatherWarp * 32, ch = g & 7, r0 = g >> 3;
        const int dcol = (ch ^ (r0 & 7)) << 4;
        auto gather = [&](unsigned char *dst, const uint16_t *lo, const uint16_t *hi, const uint16_t *pos, int n,
                          size_t ubase, bool zero) {
            const uint16_t *base = ch < 2 ? lo + ch * 8 : hi + (ch - 2) * 8;
            const int stride = ch < 2 ? 16 : 48;
            #pragma unroll 4
            for (int r = r0; r < C::kHiTok; r += kGatherThreads / 8) {
                const bool valid = r < n;
                const uint16_t *src = base + (ubase + (valid ? pos[r] : 0)) * stride;
                unsigned char *dp = dst + r * 128 + dcol;
                if (zero) cp_async16_zfill(dp, src, valid);
                else if (valid) cp_async16(dp, src);
            }
        };
        uint32_t h = 0;
        while (true) {
            const int hq = h % kNQ;
            if (!mbar_wait(&sm.gready[hq], (h / kNQ) & 1u, abort)) break;
            const int *e = sm.hiq[hq];
            const int ks = e[0], vs = e[1], ds = e[2], n = e[3], unit = e[4], skew = e[5], etype = e[6], etok = e[7];
            mbar_arrive(&sm.gfree[hq]);
            if (ks < 0) break;
            // the positions (landed with the queue entry) stay valid until the consumers free the
            // descriptor, which needs this tile's data first
            const uint16_t *pos = reinterpret_cast<const uint16_t *>(sm.kdesc[ds] + 8) + skew;
            const size_t ubase = (size_t)unit * p.T;
            if constexpr (Q4) {
                if (etype == kTypeLo) {
                    // the second half of a LO tile's rows (the producer dequantizes the first)
                    const size_t base = ubase + etok;
                    constexpr int kHalf = C::kLoTok / 2;
                    if (VALUE)
                        quant::lo_rows_kv<kHalf / kGatherThreads, kGatherThreads>(
                            sm.kslot[ks], sm.vslot[vs], p.QK_lo, p.EK, p.QV_lo, p.EV, base, n, kHalf + g);
                    else
                        quant::lo_rows<kHalf / kGatherThreads, kGatherThreads>(sm.kslot[ks], p.QK_lo, p.EK, base, n,
                                                                              kHalf + g);
                    fence_proxy_async();
                    mbar_arrive(&sm.kfull[ks]);
                    if (VALUE) mbar_arrive(&sm.vfull[vs]);
                    ++h;
                    continue;
                }
                // dequantize a HI tile into the layout of the 16-bit path (128-byte rows, 128-byte
                // swizzle); rows past n are zero
                constexpr int RH = C::kHiTok / kGatherThreads;
                struct HiRows { uint2 w[RH][4]; char2 ee[RH]; };
                auto hi_load = [&](HiRows &H, const uint8_t *QL, const uint8_t *QH, const int8_t *E) {
                    #pragma unroll
                    for (int i = 0; i < RH; ++i) {
                        const int r = g + kGatherThreads * i;
                        #pragma unroll
                        for (int k = 0; k < 4; ++k) H.w[i][k] = make_uint2(0u, 0u);
                        H.ee[i] = make_char2(0, 0);
                        if (r < n) {
                            const size_t row = ubase + pos[r];
                            H.w[i][0] = __ldg(reinterpret_cast<const uint2 *>(QL + row * 8));
                            const uint2 *hq2 = reinterpret_cast<const uint2 *>(QH + row * 24);
                            H.w[i][1] = __ldg(hq2);
                            H.w[i][2] = __ldg(hq2 + 1);
                            H.w[i][3] = __ldg(hq2 + 2);
                            H.ee[i] = __ldg(reinterpret_cast<const char2 *>(E + row * 2));
                        }
                    }
                };
                auto hi_store = [&](const HiRows &H, unsigned char *dst) {
                    #pragma unroll
                    for (int i = 0; i < RH; ++i) {
                        const int r = g + kGatherThreads * i;
                        #pragma unroll
                        for (int c8 = 0; c8 < 8; ++c8) {
                            const uint32_t word = (c8 & 1) ? H.w[i][c8 >> 1].y : H.w[i][c8 >> 1].x;
                            *reinterpret_cast<uint4 *>(dst + r * 128 + ((c8 ^ (r & 7)) << 4)) =
                                quant::dq8(word, c8 < 2 ? H.ee[i].x : H.ee[i].y);
                        }
                    }
                };
                // every load of a tile (K and V) is issued before the first is used, so one memory
                // latency is paid per tile
                {
                    HiRows K4, V4;
                    hi_load(K4, p.QK_lo, p.QK_hi, p.EK);
                    if (VALUE) hi_load(V4, p.QV_lo, p.QV_hi, p.EV);
                    hi_store(K4, sm.kslot[ks]);
                    fence_proxy_async();
                    mbar_arrive(&sm.kfull[ks]);
                    if (VALUE) {
                        hi_store(V4, sm.vslot[vs]);
                        mbar_arrive(&sm.vfull[vs]);
                    }
                }
                ++h;
                continue;
            }
            gather(sm.kslot[ks], p.CK_lo, p.CK_hi, pos, n, ubase, false);
            cp_async_arrive(&sm.kfull[ks]);   // raises the pending count; arrives when the copies land
            mbar_arrive(&sm.kfull[ks]);
            if (VALUE) {
                gather(sm.vslot[vs], p.CV_lo, p.CV_hi, pos, n, ubase, true);
                cp_async_arrive(&sm.vfull[vs]);
                mbar_arrive(&sm.vfull[vs]);
            }
            ++h;
        }
        cp_async_wait_all();
    } else if (warp == 1) {
        // =============================================================== MMA issuer
        if (lane == 0) {
            uint32_t seq = 0, qseq = 0;
            bool issued = false;
            const uint32_t id_s = idesc_bf16_kk(128, kNHP);
            // shared-memory descriptors, formed once: K slot 0 as a LO operand (32-byte rows) and as a
            // HI operand (128-byte rows), and the q~ planes of q slot 0; a slot, q slot, sub-tile or
            // k-step moves the start address, the low field of the descriptor (address / 16)
            const uint64_t dlo0 = desc_kmajor(smem_u32(sm.kslot[0]), 256u, 6u);
            const uint64_t dhi0 = desc_kmajor(smem_u32(sm.kslot[0]), 1024u, 2u);
            const uint64_t dqh0 = desc_kmajor(smem_u32(&sm.qbuf[0][0][0]), 1024u, 2u);
            const uint64_t dql0 = desc_kmajor(smem_u32(&sm.qbuf[0][1][0]), 1024u, 2u);
            constexpr uint32_t kSlotStep = C::kKBytes >> 4, kQStep = (2 * C::kNHP * 128) >> 4;
            while (true) {
                const int ks = seq % kNK, sb = seq % kNS;
                if (!mbar_wait(&sm.kfull[ks], (seq / kNK) & 1u, abort)) break;
                // the S buffer of the tile kNS back must have been read
                if (seq >= (uint32_t)kNS && !mbar_wait(&sm.sfree[sb], ((seq / kNS) - 1) & 1u, abort)) break;
                const int *d = sm.kdesc[seq % kND];
                const int hdr = d[0];
                const int type = hdr & 0xff;
                if (type == kTypeEnd) {
                    mbar_arrive(&sm.sfull[sb]);
                    break;
                }
                const int qs = d[5], n = d[3];
                if (hdr & kFlagFirst) {
                    if (!mbar_wait(&sm.qfull[qs], (qseq >> 1) & 1u, abort)) break;
                    ++qseq;
                }
                const bool has_s = type == kTypeHi || !p.rank0;
                if (has_s) {
                    if (type == kTypeHi || Q4) fence_proxy_async();   // rows written by cp.async or stores
                    tmem_fence_after();
                    const uint32_t dcol = tmem + (uint32_t)(sb * C::kSCols);
                    const uint64_t qh = dqh0 + (uint64_t)(qs * kQStep), ql = dql0 + (uint64_t)(qs * kQStep);
                    if (type == kTypeLo) {
                        const uint64_t a0 = dlo0 + (uint64_t)(ks * kSlotStep);
                        // the q~ hi products of all sub-tiles first (independent accumulators), then
                        // the lo products that add into them
                        const int nsub = (n + kTile - 1) / kTile;
                        for (int sub = 0; sub < nsub; ++sub)
                            umma_bf16(dcol + sub * kNHP, a0 + (uint64_t)(sub * (4096 >> 4)), qh, id_s, 0u);
                        for (int sub = 0; sub < nsub; ++sub)
                            umma_bf16(dcol + sub * kNHP, a0 + (uint64_t)(sub * (4096 >> 4)), ql, id_s, 1u);
                    } else {
                        const uint64_t a0 = dhi0 + (uint64_t)(ks * kSlotStep);
                        #pragma unroll
                        for (int k = 0; k < 4; ++k) {
                            umma_bf16(dcol, a0 + 2u * k, qh + 2u * k, id_s, k > 0 ? 1u : 0u);
                            umma_bf16(dcol, a0 + 2u * k, ql + 2u * k, id_s, 1u);
                        }
                    }
                    umma_commit(&sm.sfull[sb]);
                    umma_commit(&sm.kempty[ks]);
                    issued = true;
                } else {
                    mbar_arrive(&sm.sfull[sb]);   // keeps the rings' phases in step
                    mbar_arrive(&sm.kempty[ks]);
                }
                if (hdr & kFlagLast) umma_commit(&sm.qempty[qs]);
                ++seq;
            }
            // MMAs still in flight (possible only after an abort) must finish before tensor memory
            // is freed: one more commit, to a barrier of its own, arrives once all of them are done
            if (issued) {
                umma_commit(&sm.mdone);
                const long long t0 = clock64();
                while (!mbar_try_wait(&sm.mdone, 0u) && clock64() - t0 < kWaitCycles) {}
            }
        }
        __syncwarp();
    } else {
        // =============================================================== consumers
        // kSplit groups of four warps share each tile: group cg takes heads [cg HS, cg HS + HS)
        constexpr int HS = C::kHS, PHS = C::kPHS, NCW = 4 * C::kSplit;
        const int q = warp & 3;                       // tensor-memory lane quarter
        const int cg = warp >= kConsumer2 ? 1 : 0;
        const int h0 = cg * HS;
        const uint32_t lane_addr = (uint32_t)(32 * q) << 16;
        const int g = lane >> 2, tig = lane & 3;
        uint32_t seq = 0;
        // per-segment state
        float m[HS], l[HS];                            // stats pass: this thread's reference max and sum per head
        float Mh[HS], ILh[HS];                         // value pass: the unit's (M, 1/L) per head
        float u[4][PHS / 8][4];                        // value pass: u^T (ranks on M, heads on N) of this warp
        (void)m; (void)l; (void)Mh; (void)ILh; (void)u;
        int unit = 0, pslot = 0;
        unsigned char *pb = sm.pbuf[VALUE ? 4 * cg + q : 0];
        const uint32_t pb_s = smem_u32(pb);
        float *mrow = nullptr;                         // value pass: the segment's unit's row of the mass
        // Per-lane parts of the value pass's shared-memory addresses.  A k-step's first row is a
        // multiple of 16, so every swizzle term depends on the lane alone.
        const int ra = (lane & 7) + ((lane >> 4) << 3);                // A (C_V^T): row within the k-step
        const int rb = (lane & 7) + (((lane >> 3) & 1) << 3);          // B (P): row within the k-step
        const uint32_t offA_lo = (uint32_t)(ra * 32 + ((((lane >> 3) & 1) ^ ((ra >> 2) & 1)) << 4));
        uint32_t offA_hi[4], offB[(PHS + 15) / 16], offP[PHS / 8];
        #pragma unroll
        for (int mt = 0; mt < 4; ++mt)
            offA_hi[mt] = (uint32_t)(ra * 128 + (((2 * mt + ((lane >> 3) & 1)) ^ (lane & 7)) << 4));
        #pragma unroll
        for (int np = 0; np < (PHS + 15) / 16; ++np) {
            int ch = PHS == 8 ? 0 : 2 * np + (lane >> 4);
            if (PHS == 16) ch ^= (rb >> 2) & 1;
            if (PHS == 32) ch ^= (rb >> 1) & 3;
            offB[np] = (uint32_t)(rb * (PHS * 2) + (ch << 4));
        }
        #pragma unroll
        for (int c = 0; c < PHS / 8; ++c) {
            int pc = c;
            if (PHS == 16) pc = c ^ ((lane >> 2) & 1);
            if (PHS == 32) pc = c ^ ((lane >> 1) & 3);
            offP[c] = (uint32_t)(lane * (PHS * 2) + pc * 16);
        }
        (void)offA_lo; (void)offA_hi; (void)offB; (void)offP; (void)mrow;
        bool failed = false;
        while (!failed) {
            const int sb = seq % kNS, vs = seq % kNV;
            if (!mbar_wait(&sm.sfull[sb], (seq / kNS) & 1u, abort)) break;
            tmem_fence_after();
            const int *d = sm.kdesc[seq % kND];
            const int hdr = d[0];
            const int type = hdr & 0xff;
            if (type == kTypeEnd) break;
            const int n = d[3];
            if (hdr & kFlagFirst) {
                unit = d[1];
                pslot = d[4];
                if (VALUE) {
                    mrow = p.mass != nullptr ? p.mass + (size_t)unit * p.T : nullptr;
                    #pragma unroll
                    for (int h = 0; h < HS; ++h) {
                        float2 st = make_float2(0.f, 0.f);
                        if (h0 + h < p.Hg)
                            st = __ldg(reinterpret_cast<const float2 *>(p.ustat + ((size_t)unit * p.Hg + h0 + h) * 2));
                        Mh[h] = st.x;
                        ILh[h] = st.y;
                    }
                    #pragma unroll
                    for (int a = 0; a < 4; ++a)
                        #pragma unroll
                        for (int b = 0; b < PHS / 8; ++b) u[a][b][0] = u[a][b][1] = u[a][b][2] = u[a][b][3] = 0.f;
                } else {
                    #pragma unroll
                    for (int h = 0; h < HS; ++h) { m[h] = kRefInit; l[h] = 0.f; }
                }
            }
            const bool has_s = type == kTypeHi || !p.rank0;
            const int nsub = type == kTypeLo ? (n + kTile - 1) / kTile : 1;
            const uint32_t vb = smem_u32(sm.vslot[vs]);
            bool v_ready = false;
            // the scores of one sub-tile (this group's heads) are loaded from tensor memory before each wait
            for (int sub = 0; sub < nsub && !failed; ++sub) {
                if (sub * kTile + 32 * q >= n) continue;   // no token of this warp here
                constexpr int NL = HS <= 4 ? 4 : HS <= 8 ? 8 : HS <= 16 ? 16 : 32;   // columns loaded
                float sc[NL];
                if (has_s) {
                    tmem_ld<NL>(tmem + lane_addr + (uint32_t)(sb * C::kSCols + sub * kNHP + cg * C::kGCol), sc);
                    tmem_wait_ld();
                } else {
                    #pragma unroll
                    for (int h = 0; h < NL; ++h) sc[h] = 0.f;
                }
                const int r = sub * kTile + 32 * q + lane;    // row of this thread's token in the tile
                bool take;
                int pos;
                if (type == kTypeLo) {
                    const uint32_t wd = (uint32_t)d[8 + 4 * sub + q];
                    take = r < n && !((wd >> lane) & 1u);
                    pos = d[2] + r;
                } else {
                    take = r < n;
                    pos = r < n ? reinterpret_cast<const uint16_t *>(d + 8)[d[2] + r] : 0;
                }
                if (!VALUE) {
                    // ---------------------------------------------------- stats
                    if (take) {
                        // m[h] is kept kLazy above the largest logit at its last move, so the test is
                        // one comparison per head and every term 2^(s - m) is at most 1
                        bool up = false;
                        #pragma unroll
                        for (int h = 0; h < HS; ++h) up |= sc[h] > m[h];
                        if (up) {
                            #pragma unroll
                            for (int h = 0; h < HS; ++h)
                                if (sc[h] > m[h]) {
                                    l[h] *= ex2(m[h] - (sc[h] + kLazy));
                                    m[h] = sc[h] + kLazy;
                                }
                        }
                        #pragma unroll
                        for (int h = 0; h < HS; ++h) l[h] += ex2(sc[h] - m[h]);
                    }
                } else {
                    // ---------------------------------------------------- value
                    float pr[PHS];
                    float ms0 = 0.f, ms1 = 0.f;
                    #pragma unroll
                    for (int h = 0; h < PHS; ++h) {
                        if (h < HS) {
                            const float e = take ? ex2(sc[h] - Mh[h]) : 0.f;
                            pr[h] = e;
                            if (h & 1) ms1 = fmaf(e, ILh[h], ms1);
                            else ms0 = fmaf(e, ILh[h], ms0);
                        } else {
                            pr[h] = 0.f;
                        }
                    }
                    // the token's attention mass: each head group adds its heads' share into the
                    // zeroed output (two addends onto zero: the same sum in either order)
                    if (take && mrow != nullptr) {
                        if (C::kSplit == 1) mrow[pos] = ms0 + ms1;
                        else red_add_f32(mrow + pos, ms0 + ms1);
                    }
                    const bool do_u = type == kTypeHi || !p.rank0;
                    if (do_u && !v_ready) {
                        if (!mbar_wait(&sm.vfull[vs], (seq / C::kNV) & 1u, abort)) { failed = true; break; }
                        v_ready = true;
                    }
                    if (do_u) {
                        // this thread's P row (PHS bf16), 16-byte chunks swizzled against bank conflicts
                        #pragma unroll
                        for (int c = 0; c < PHS / 8; ++c) {
                            uint4 v;
                            v.x = pack_bf16(pr[8 * c + 0], pr[8 * c + 1]);
                            v.y = pack_bf16(pr[8 * c + 2], pr[8 * c + 3]);
                            v.z = pack_bf16(pr[8 * c + 4], pr[8 * c + 5]);
                            v.w = pack_bf16(pr[8 * c + 6], pr[8 * c + 7]);
                            *reinterpret_cast<uint4 *>(pb + offP[c]) = v;
                        }
                        __syncwarp();
                        // u^T += C_V^T P over the warp's 32 tokens (two k-steps of 16)
                        const uint32_t a_lo = vb + (uint32_t)((sub * kTile + 32 * q) * 32) + offA_lo;
                        const uint32_t a_hi = vb + (uint32_t)((32 * q) * 128);
                        #pragma unroll 1
                        for (int kk = 0; kk < 2; ++kk) {
                            uint32_t bfr[PHS / 8][2];
                            #pragma unroll
                            for (int np = 0; np < (PHS + 15) / 16; ++np) {
                                const uint32_t ba = pb_s + (uint32_t)(kk * 16 * PHS * 2) + offB[np];
                                uint32_t r0, r1, r2, r3;
                                if (PHS == 8) {
                                    // x2: tokens 0-7 and 8-15 of the 8 heads
                                    asm volatile("ldmatrix.sync.aligned.m8n8.x2.trans.shared.b16 {%0,%1}, [%2];"
                                                 : "=r"(r0), "=r"(r1) : "r"(ba));
                                    bfr[0][0] = r0;
                                    bfr[0][1] = r1;
                                } else {
                                    ldsm_x4_t(ba, r0, r1, r2, r3);
                                    bfr[2 * np][0] = r0;
                                    bfr[2 * np][1] = r1;
                                    bfr[2 * np + 1][0] = r2;
                                    bfr[2 * np + 1][1] = r3;
                                }
                            }
                            if (type == kTypeLo) {
                                uint32_t a[4];
                                ldsm_x4_t(a_lo + (uint32_t)(kk * 16 * 32), a[0], a[1], a[2], a[3]);
                                #pragma unroll
                                for (int nt = 0; nt < PHS / 8; ++nt) mma_bf16(u[0][nt], a, bfr[nt][0], bfr[nt][1]);
                            } else {
                                #pragma unroll
                                for (int mt = 0; mt < 4; ++mt) {
                                    uint32_t a[4];
                                    ldsm_x4_t(a_hi + (uint32_t)(kk * 16 * 128) + offA_hi[mt], a[0], a[1], a[2], a[3]);
                                    #pragma unroll
                                    for (int nt = 0; nt < PHS / 8; ++nt) mma_bf16(u[mt][nt], a, bfr[nt][0], bfr[nt][1]);
                                }
                            }
                        }
                        __syncwarp();
                    }
                }
            }
            if (failed) break;
            // the V slot (value pass) and the S buffer are free once every consumer warp is done
            if (VALUE) {
                if (!v_ready && !mbar_wait(&sm.vfull[vs], (seq / kNV) & 1u, abort)) break;
                __syncwarp();
                if (lane == 0) mbar_arrive(&sm.vempty[vs]);
            }
            tmem_fence_before();
            __syncwarp();
            if (lane == 0) {
                mbar_arrive(&sm.sfree[sb]);
                mbar_arrive(&sm.dfree[seq % kND]);
            }

            if (hdr & kFlagLast) {
                // ---------------------------------------------------------- the segment's partial
                if (!VALUE) {
                    // (m, l) per head: over the warp's lanes, then over the four warps in a fixed order
                    #pragma unroll
                    for (int h = 0; h < HS; ++h) {
                        float mw = m[h];
                        #pragma unroll
                        for (int o = 16; o > 0; o >>= 1) mw = fmaxf(mw, __shfl_xor_sync(0xffffffffu, mw, o));
                        float lw = l[h] * ex2(m[h] - mw);
                        #pragma unroll
                        for (int o = 16; o > 0; o >>= 1) lw += __shfl_xor_sync(0xffffffffu, lw, o);
                        if (lane == 0) {
                            sm.merge[q][2 * (h0 + h)] = mw;
                            sm.merge[q][2 * (h0 + h) + 1] = lw;
                        }
                    }
                    named_sync(1, 32 * NCW);
                    if (q == 0 && cg == 0 && lane < NH && lane < p.Hg) {
                        float mx = sm.merge[0][2 * lane];
                        #pragma unroll
                        for (int w = 1; w < 4; ++w) mx = fmaxf(mx, sm.merge[w][2 * lane]);
                        float sum = 0.f;
                        #pragma unroll
                        for (int w = 0; w < 4; ++w) sum += sm.merge[w][2 * lane + 1] * ex2(sm.merge[w][2 * lane] - mx);
                        float *dst = p.part + (((size_t)unit * p.nslot + pslot) * p.Hg + lane) * 2;
                        dst[0] = mx;
                        dst[1] = sum;
                    }
                    named_sync(1, 32 * NCW);
                } else {
                    // u per head: warps 1-3 of each group park theirs in shared memory, warp 0 adds them
                    // in order
                    if (q != 0) {
                        #pragma unroll
                        for (int mt = 0; mt < 4; ++mt)
                            #pragma unroll
                            for (int nt = 0; nt < PHS / 8; ++nt)
                                #pragma unroll
                                for (int e = 0; e < 4; ++e) {
                                    const int rr = 16 * mt + g + 8 * (e >> 1), hh = 8 * nt + 2 * tig + (e & 1);
                                    if (hh < HS) sm.merge[q - 1][(h0 + hh) * 64 + rr] = u[mt][nt][e];
                                }
                    }
                    named_sync(1, 32 * NCW);
                    if (q == 0) {
                        float *dst = p.part + ((size_t)unit * p.nslot + pslot) * p.Hg * 64;
                        #pragma unroll
                        for (int mt = 0; mt < 4; ++mt)
                            #pragma unroll
                            for (int nt = 0; nt < PHS / 8; ++nt)
                                #pragma unroll
                                for (int e = 0; e < 4; ++e) {
                                    const int rr = 16 * mt + g + 8 * (e >> 1), hh = 8 * nt + 2 * tig + (e & 1);
                                    if (hh < HS && h0 + hh < p.Hg) {
                                        const int H = h0 + hh;
                                        float v = u[mt][nt][e];
                                        v += sm.merge[0][H * 64 + rr];
                                        v += sm.merge[1][H * 64 + rr];
                                        v += sm.merge[2][H * 64 + rr];
                                        dst[H * 64 + rr] = v;
                                    }
                                }
                    }
                    named_sync(1, 32 * NCW);
                }
            }
            ++seq;
        }
        if (failed) *abort = 1;
    }

    tmem_fence_before();
    __syncthreads();
    if (warp == 1) {
        tmem_fence_after();
        tmem_dealloc(tmem, C::kTmemCols);
    }
}

// ------------------------------------------------------------------ full-rank positions

// Each unit's full-rank token positions in ascending order (hipos[unit][0 .. count)) and, per
// 128-token tile, the count of full-rank tokens before it (hicnt[unit][tile]): the visual
// passes' HI tiles are runs of that list.  A group of tpg threads (32 .. 1024, the unit's word
// count rounded up to a power of two) per unit, blockDim / tpg units per block (blockIdx.y picks
// the mask: the visual tokens', or the compressed text tokens' own); thread t of a group scans a
// contiguous run of words.
constexpr int kHpThreads = 1024;     // most threads per block (blocks are 256 threads unless a unit needs more)
constexpr int kHpWords = 8;       // mask words a thread keeps in registers
struct HiposParams {
    const uint32_t *mask;    // [units][nwords]
    uint16_t *hipos;         // [units][Tp]
    int *hicnt;              // [units][tpu]
    float *mass;             // [units][T], zeroed here when the value pass adds into it (or null)
    int units, T, nwords, tpu, Tp, tpg;
};

__host__ __device__ inline int hipos_group(int nwords) {
    int t = 32;
    while (t < kHpThreads && t < nwords) t <<= 1;
    return t;
}

__global__ void __launch_bounds__(kHpThreads) hipos_kernel(const HiposParams a, const HiposParams b) {
    griddep_launch_dependents();
    const HiposParams &p = blockIdx.y == 0 ? a : b;
    const int tpg = p.tpg, t = threadIdx.x % tpg, warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int unit = blockIdx.x * (blockDim.x / tpg) + threadIdx.x / tpg;
    const int w_first = (threadIdx.x / tpg) * (tpg / 32);   // the group's first warp
    __shared__ int wsum[kHpThreads / 32];
    const bool live = unit < p.units;
    if (live && p.mass != nullptr) {
        float *ms = p.mass + (size_t)unit * p.T;
        for (int i = t; i < p.T; i += tpg) ms[i] = 0.f;
    }
    const int wpt = (p.nwords + tpg - 1) / tpg;
    const int w0 = min(p.nwords, t * wpt), w1 = min(p.nwords, w0 + wpt);
    const uint32_t *mk = p.mask + (size_t)(live ? unit : 0) * p.nwords;
    auto word = [&](int w) -> uint32_t {
        uint32_t v = __ldg(mk + w);
        const int nb = p.T - 32 * w;
        if (nb < 32) v &= (1u << nb) - 1u;
        return v;
    };
    // a thread's words stay in registers when they are at most kHpWords (masks up to 65536 tokens)
    uint32_t wv[kHpWords];
    int c = 0;
    #pragma unroll
    for (int i = 0; i < kHpWords; ++i) {
        wv[i] = live && w0 + i < w1 ? word(w0 + i) : 0u;
        c += __popc(wv[i]);
    }
    if (live)
        for (int w = w0 + kHpWords; w < w1; ++w) c += __popc(word(w));
    int incl = c;
    #pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
        const int v = __shfl_up_sync(0xffffffffu, incl, o);
        if (lane >= o) incl += v;
    }
    if (lane == 31) wsum[warp] = incl;
    __syncthreads();
    if (live) {
        int base = incl - c;
        for (int i = w_first; i < warp; ++i) base += wsum[i];
        uint16_t *out = p.hipos + (size_t)unit * p.Tp;
        int *cnt = p.hicnt + (size_t)unit * p.tpu;
        auto emit = [&](int w, uint32_t bits) {
            if ((w & 3) == 0) cnt[w >> 2] = base;   // a tile is four words
            while (bits) {
                out[base++] = (uint16_t)(32 * w + __ffs(bits) - 1);
                bits &= bits - 1u;
            }
        };
        #pragma unroll
        for (int i = 0; i < kHpWords; ++i)
            if (w0 + i < w1) emit(w0 + i, wv[i]);
        for (int w = w0 + kHpWords; w < w1; ++w) emit(w, word(w));
    }
    // the next kernel's wait then also covers the kernel before this one
    griddep_wait();
}

// ------------------------------------------------------------------ combine

// Per unit and query head (one warp per unit, a lane per head): the unit-wide max M and
// sum L over the statistics pass's segment partials, those of the text tokens' own
// rank-space pass when the text is compressed too, and the text tail's chunk partials;
// writes (M, 1/L) for the value passes and the finish.
struct Segs {
    const float *part;      // [units][nslot][Hg][2] = (m, l), or null
    int nslot, tpu, ctas;
    long long ntiles;
};

// partials of a unit: one per CTA that holds some of its tiles
__device__ __forceinline__ int seg_count(const Segs &s, int unit) {
    const long long f = (long long)unit * s.tpu;
    return (int)(cta_of_tile(f + s.tpu - 1, s.ctas, s.ntiles) - cta_of_tile(f, s.ctas, s.ntiles)) + 1;
}

__global__ void __launch_bounds__(256) combine_kernel(const Segs sv, const Segs st, const float *__restrict__ tpart,
                                                      float *__restrict__ ustat, int units, int Hg, int Sc) {
    griddep_launch_dependents();
    griddep_wait();
    const int unit = blockIdx.x * 8 + (threadIdx.x >> 5), h = threadIdx.x & 31;
    if (unit >= units || h >= Hg) return;
    const float *tp = tpart + (size_t)unit * Sc * Hg * kTxtPart + (size_t)h * kTxtPart;
    float mx = -INFINITY, sum = 0.f;
    #pragma unroll
    for (int pass = 0; pass < 2; ++pass) {       // the maximum first, then the sum
        for (int which = 0; which < 2; ++which) {
            const Segs &sg = which == 0 ? sv : st;
            if (sg.part == nullptr) continue;
            const int n = seg_count(sg, unit);
            const float *sp = sg.part + ((size_t)unit * sg.nslot * Hg + h) * 2;
            for (int k = 0; k < n; ++k) {
                const float m = sp[(size_t)k * Hg * 2];
                if (pass == 0) mx = fmaxf(mx, m);
                else sum += sp[(size_t)k * Hg * 2 + 1] * ex2(m - mx);
            }
        }
        for (int c = 0; c < Sc; ++c) {
            const float mc = tp[(size_t)c * Hg * kTxtPart];
            if (pass == 0) mx = fmaxf(mx, mc);
            else if (mc != -INFINITY) sum += tp[(size_t)c * Hg * kTxtPart + 1] * ex2(mc - mx);
        }
    }
    *reinterpret_cast<float2 *>(ustat + ((size_t)unit * Hg + h) * 2) = make_float2(mx, 1.f / sum);
}

// ------------------------------------------------------------------ finish

struct FinishParams {
    const uint16_t *BV;       // [units][64][512]
    const float *vpart;       // [units][nslot][Hg][64]: u = sum p' C_V per segment
    const uint16_t *BV2;      // the text tokens' own B_V, or null
    const float *vpart2;      // [units][nslot2][Hg][64]: their u per segment
    int nslot2, tpu2, cta_v2;
    long long ntiles2;
    const float *tpart;       // [units][Sc][Hg][kTxtPart] or null
    const float *ustat;       // [units][Hg][2]: (M, 1/L)
    uint16_t *out;            // [(layer, batch)][n_q][128]
    int Hg, per_kv, n_q, groups, Sc, nslot, tpu, cta_v;
    long long ntiles;
};

// One block per (unit, JPB KV heads), two warps per KV head j.  Thread (g, f) of a KV head owns
// output features 8f .. 8f+7 (f < 16) and rank group g < 4 (ranks 16g .. 16g+15, and the text
// chunks c = g mod 4): u_h = the sum of the unit's segment partials, w_h = the text chunks' sums
// weighted by 2^(m_c - M_h), then
//   o_h = (u_h B_V[:, 128 j ..] + u2_h B_V2[:, 128 j ..] + w_h) / L_h
// for the PK query heads of the KV head (u2, B_V2: the text tokens' own rank space, when the
// text is compressed).  B_V rows are read 16 bytes at a time and issued first; the four rank
// groups' sums meet through a shuffle (the two groups of a warp) and shared memory (the two
// warps).  JPB = 4 (a whole unit per block) when units are many, 1 when few, so that the launch
// fills the GPU either way.
constexpr int kFinishMaxChunks = 64;   // text chunks whose weights are staged; longer tails loop

template <int PK>
__device__ __forceinline__ void finish_project(const uint16_t *__restrict__ bv, const float (*uf)[64], int hb, int rg,
                                               float (&acc)[PK][8]) {
    uint4 raw[16];
    #pragma unroll
    for (int i = 0; i < 16; ++i) raw[i] = __ldcs(reinterpret_cast<const uint4 *>(bv + (size_t)(16 * rg + i) * 512));
    #pragma unroll
    for (int i = 0; i < 16; ++i) {
        const uint32_t w[4] = {raw[i].x, raw[i].y, raw[i].z, raw[i].w};
        float b[8];
        #pragma unroll
        for (int e = 0; e < 4; ++e) {
            b[2 * e] = __uint_as_float(w[e] << 16);
            b[2 * e + 1] = __uint_as_float(w[e] & 0xffff0000u);
        }
        #pragma unroll
        for (int hh = 0; hh < PK; ++hh) {
            const float u = uf[hb + hh][16 * rg + i];
            #pragma unroll
            for (int f = 0; f < 8; ++f) acc[hh][f] = fmaf(u, b[f], acc[hh][f]);
        }
    }
}

template <int PK, int JPB>
__global__ void __launch_bounds__(64 * JPB) finish_kernel(const FinishParams p) {
    constexpr int NHB = PK * JPB;           // query heads of the block
    __shared__ float uf[NHB][64];
    __shared__ float uf2[NHB][64];
    __shared__ float ew[NHB][kFinishMaxChunks];
    __shared__ float ms[NHB][2];
    __shared__ float red[JPB][PK][128];
    griddep_wait();
    constexpr int kBlocksPerUnit = 4 / JPB;
    const int unit = blockIdx.x / kBlocksPerUnit, tid = threadIdx.x, lane = tid & 31;
    const int j0 = (blockIdx.x % kBlocksPerUnit) * JPB, jj = tid >> 6;
    const int half = (tid >> 5) & 1, fg = lane & 15, rg = 2 * half + (lane >> 4);
    const int hb0 = j0 * PK;                // first query head of the block (within the unit)
    const int hb = jj * PK;                 // this KV head's first query head within the block
    if (tid < NHB) {
        const float2 st = __ldg(reinterpret_cast<const float2 *>(p.ustat + ((size_t)unit * p.Hg + hb0 + tid) * 2));
        ms[tid][0] = st.x;
        ms[tid][1] = st.y;
    }
    const long long f = (long long)unit * p.tpu;
    const int ns = (int)(cta_of_tile(f + p.tpu - 1, p.cta_v, p.ntiles) - cta_of_tile(f, p.cta_v, p.ntiles)) + 1;
    for (int i = tid; i < NHB * 64; i += 64 * JPB) {
        const int hh = i >> 6, r = i & 63;
        const float *src = p.vpart + ((size_t)unit * p.nslot * p.Hg + hb0 + hh) * 64 + r;
        float a = 0.f;
        for (int k = 0; k < ns; ++k) a += __ldcg(src + (size_t)k * p.Hg * 64);
        uf[hh][r] = a;
    }
    if (p.vpart2 != nullptr) {
        const long long f2 = (long long)unit * p.tpu2;
        const int ns2 = (int)(cta_of_tile(f2 + p.tpu2 - 1, p.cta_v2, p.ntiles2) - cta_of_tile(f2, p.cta_v2, p.ntiles2)) + 1;
        for (int i = tid; i < NHB * 64; i += 64 * JPB) {
            const int hh = i >> 6, r = i & 63;
            const float *src = p.vpart2 + ((size_t)unit * p.nslot2 * p.Hg + hb0 + hh) * 64 + r;
            float a = 0.f;
            for (int k = 0; k < ns2; ++k) a += __ldcg(src + (size_t)k * p.Hg * 64);
            uf2[hh][r] = a;
        }
    }
    __syncthreads();
    float acc[PK][8];
    #pragma unroll
    for (int hh = 0; hh < PK; ++hh)
        #pragma unroll
        for (int e = 0; e < 8; ++e) acc[hh][e] = 0.f;
    const size_t col = (size_t)unit * 64 * 512 + 128 * (j0 + jj) + 8 * fg;
    finish_project<PK>(p.BV + col, uf, hb, rg, acc);
    if (p.BV2 != nullptr) finish_project<PK>(p.BV2 + col, uf2, hb, rg, acc);
    if (p.tpart != nullptr) {
        const float *tp0 = p.tpart + ((size_t)unit * p.Sc * p.Hg + hb0) * kTxtPart;
        for (int c0 = 0; c0 < p.Sc; c0 += kFinishMaxChunks) {
            const int nc = min(kFinishMaxChunks, p.Sc - c0);
            __syncthreads();
            for (int i = tid; i < NHB * nc; i += 64 * JPB) {
                const int hh = i / nc, c = i % nc;
                const float mc = __ldcg(tp0 + ((size_t)(c0 + c) * p.Hg + hh) * kTxtPart);
                ew[hh][c] = mc != -INFINITY ? ex2(mc - ms[hh][0]) : 0.f;
            }
            __syncthreads();
            for (int c = rg; c < nc; c += 4) {
                #pragma unroll
                for (int hh = 0; hh < PK; ++hh) {
                    const float wgt = ew[hb + hh][c];
                    const float *src = tp0 + ((size_t)(c0 + c) * p.Hg + hb + hh) * kTxtPart + 2 + 8 * fg;
                    // rows of kTxtPart = 130 floats: 8-byte aligned, read as float2
                    #pragma unroll
                    for (int e = 0; e < 4; ++e) {
                        const float2 v = __ldcg(reinterpret_cast<const float2 *>(src) + e);
                        acc[hh][2 * e] = fmaf(wgt, v.x, acc[hh][2 * e]);
                        acc[hh][2 * e + 1] = fmaf(wgt, v.y, acc[hh][2 * e + 1]);
                    }
                }
            }
        }
    }
    // the four rank groups: lanes f and f + 16 of a warp, then the KV head's two warps
    #pragma unroll
    for (int hh = 0; hh < PK; ++hh)
        #pragma unroll
        for (int e = 0; e < 8; ++e) acc[hh][e] += __shfl_xor_sync(0xffffffffu, acc[hh][e], 16);
    if (half == 1 && lane < 16) {
        #pragma unroll
        for (int hh = 0; hh < PK; ++hh)
            #pragma unroll
            for (int e = 0; e < 8; ++e) red[jj][hh][8 * fg + e] = acc[hh][e];
    }
    __syncthreads();
    if (half == 0 && lane < 16) {
        const int lb = unit / p.groups, G = unit % p.groups;
        #pragma unroll
        for (int hh = 0; hh < PK; ++hh) {
            const float il = ms[hb + hh][1];
            uint32_t w[4];
            #pragma unroll
            for (int e = 0; e < 4; ++e)
                w[e] = pack_bf16((acc[hh][2 * e] + red[jj][hh][8 * fg + 2 * e]) * il,
                                 (acc[hh][2 * e + 1] + red[jj][hh][8 * fg + 2 * e + 1]) * il);
            uint16_t *dst = p.out + ((size_t)lb * p.n_q + (size_t)G * p.Hg + hb0 + hb + hh) * 128 + 8 * fg;
            *reinterpret_cast<uint4 *>(dst) = make_uint4(w[0], w[1], w[2], w[3]);
        }
    }
}

}  // namespace rs
}  // namespace decode
}  // namespace kvpack
