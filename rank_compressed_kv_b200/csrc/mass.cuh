// mass.cuh -- the attention mass of every visual token after a decode step.
//
// Method ("Attention-aware Inference Optimizations for Large Vision-Language
// Models with Memory-efficient Decoding", technical summaries 2.B, fr/es/de
// pages): the importance that chooses the next step's full-rank tokens is the
// softmax weight a token receives, summed over the unit's query heads:
//     mass_t = sum_h 2^(s_ht - M_h) / L_h
// with s_ht the token's logit at its own rank (16 or 64; log2 domain) and
// (M_h, L_h) the unit-wide max and sum over the visual and text tokens, fixed
// by finish_kernel.  This pass recomputes the logits from C_K alone, after
// the attention pass: it reads 32 bytes of C_K lo per token plus 128 bytes of
// C_K per full-rank token, and writes 4 bytes.  No pass waits on another.
#pragma once

#include <cuda.h>

#include <type_traits>

#include "common.cuh"
#include "decode.cuh"

namespace kvpack {
namespace decode {
namespace mass {

constexpr int kWarps = 8;
constexpr int kThreads = kWarps * 32;
constexpr int kChunk = 64;          // tokens of one unit per chunk
constexpr int kSlots = 4;           // ring slots per warp
constexpr int kSlotBytes = 2048;    // 64 C_K lo rows (32 B), or kHiTok gathered C_K rows (128 B)
constexpr int kHiTok = 16;          // full-rank tokens per gathered stage
constexpr int kMeta = 8;            // chunk metadata ring (the issue side runs at most kSlots chunks ahead)

struct Params {
    CUtensorMap tm_ck;              // C_K lo: 3D {16, T, units}, box {16, 32, 1}, 32-byte swizzle
    const uint16_t *CK_lo, *CK_hi;  // [units][T][16], [units][T][48]
    const unsigned char *qt;        // [units][qblock_bytes(Hg)]: q~ hi, lo
    const float *ustat;             // [units][Hg][2]: (M, 1/L) per head
    const uint32_t *mask;           // [units][nwords]
    float *mass;                    // [units][T]
    int T, Hg, nwords, cpu, n_chunks;   // cpu = chunks per unit
};

struct Smem {
    alignas(1024) unsigned char ring[kWarps][kSlots][kSlotBytes];
    uint8_t hi_list[kWarps][kMeta][kChunk];   // chunk-relative positions of the full-rank tokens
    int meta[kWarps][kMeta][6];               // unit, t0, n, n_hi, mask words 0 and 1
    uint64_t full[kWarps][kSlots];
    int abort;
};

constexpr size_t smem_bytes() { return sizeof(Smem) + 1024; }

// Every warp owns a contiguous range of chunks (unit, 64 tokens) and streams
// it through a private ring: per chunk one TMA stage of C_K lo rows (skipped
// when every token is full-rank) and one gathered stage per 16 full-rank
// tokens.  Logits with tokens on M and heads on N (NT tiles of 8) of mma.sync
// m16n8k16, q~ as a bf16 hi + lo pair held in registers for the whole unit.
template <int NT>
__global__ void __launch_bounds__(kThreads, NT <= 2 ? 2 : 1) mass_kernel(const __grid_constant__ Params p) {
    extern __shared__ __align__(1024) unsigned char smem_raw[];
    const uint32_t base = smem_u32(smem_raw);
    Smem &sm = *reinterpret_cast<Smem *>(smem_raw + ((1024u - (base & 1023u)) & 1023u));
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int g = lane >> 2, tig = lane & 3;
    if (threadIdx.x == 0) {
        for (int w = 0; w < kWarps; ++w)
            for (int s = 0; s < kSlots; ++s) mbar_init(&sm.full[w][s], 32);
        sm.abort = 0;
        asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
    }
    __syncthreads();
    volatile int *abort = &sm.abort;

    const long long W = (long long)gridDim.x * kWarps, wg = (long long)blockIdx.x * kWarps + warp;
    const int c_begin = (int)(wg * p.n_chunks / W), c_end = (int)((wg + 1) * p.n_chunks / W);

    // ------------------------------------------------------------ issue side
    int i_c = c_begin, i_st = 0, i_nst = 0;
    uint32_t i_seq = 0, c_seq = 0;
    bool i_done = c_begin >= c_end;
    auto begin_chunk = [&](int c) {
        const int ms = (c - c_begin) % kMeta;
        const int unit = c / p.cpu, t0 = (c % p.cpu) * kChunk;
        const int n = min(kChunk, p.T - t0);
        uint32_t w = 0u;
        if (lane < 2 && 32 * lane < n) {
            w = __ldg(p.mask + (size_t)unit * p.nwords + (t0 >> 5) + lane);
            const int nb = n - 32 * lane;
            if (nb < 32) w &= (1u << nb) - 1u;
        }
        const uint32_t w0 = __shfl_sync(0xffffffffu, w, 0), w1 = __shfl_sync(0xffffffffu, w, 1);
        const int c0 = __popc(w0), n_hi = c0 + __popc(w1);
        const uint32_t below = (1u << lane) - 1u;
        if ((w0 >> lane) & 1u) sm.hi_list[warp][ms][__popc(w0 & below)] = (uint8_t)lane;
        if ((w1 >> lane) & 1u) sm.hi_list[warp][ms][c0 + __popc(w1 & below)] = (uint8_t)(32 + lane);
        if (lane == 0) {
            int *m = sm.meta[warp][ms];
            m[0] = unit; m[1] = t0; m[2] = n; m[3] = n_hi; m[4] = (int)w0; m[5] = (int)w1;
        }
        __syncwarp();
        i_nst = (n_hi < n ? 1 : 0) + (n_hi + kHiTok - 1) / kHiTok;
        i_st = 0;
    };
    auto issue_stage = [&]() {
        const int ms = (i_c - c_begin) % kMeta;
        const int *m = sm.meta[warp][ms];
        const int unit = m[0], t0 = m[1], n = m[2], n_hi = m[3];
        const int slot = i_seq % kSlots;
        unsigned char *dst = sm.ring[warp][slot];
        uint64_t *bar = &sm.full[warp][slot];
        __syncwarp();
        if (i_st == 0 && n_hi < n) {
            const int nb = (n + 31) >> 5;
            if (lane == 0) {
                fence_proxy_async();
                mbar_arrive_tx(bar, (uint32_t)nb * 1024u);
                for (int b = 0; b < nb; ++b) tma_3d(dst + 1024 * b, &p.tm_ck, 0, t0 + 32 * b, unit, bar);
            } else {
                mbar_arrive(bar);
            }
        } else {
            // kHiTok full-rank tokens: C_lo + C_hi rows gathered into 128-byte rows
            // (16-byte chunk c of row r stored at c ^ (r & 7)); rows past the count are left alone
            const int hs = i_st - (n_hi < n ? 1 : 0);
            const int cnt = min(kHiTok, n_hi - kHiTok * hs);
            const size_t ubase = (size_t)unit * p.T + t0;
            #pragma unroll
            for (int i = 0; i < kHiTok / 4; ++i) {
                const int idx = lane + 32 * i;
                const int r = idx >> 3, ch = idx & 7;
                if (r < cnt) {
                    const size_t row = ubase + sm.hi_list[warp][ms][kHiTok * hs + r];
                    const uint16_t *src = ch < 2 ? p.CK_lo + row * 16 + ch * 8 : p.CK_hi + row * 48 + (ch - 2) * 8;
                    cp_async16(dst + r * 128 + ((ch ^ (r & 7)) << 4), src);
                }
            }
            cp_async_arrive_noinc(bar);
        }
        ++i_st;
        ++i_seq;
    };
    // issue while the ring has room, at most kMeta - 1 chunks ahead of the consumer
    int c_c = c_begin;   // chunk the consumer is on
    auto pump = [&]() {
        while (!i_done && i_seq - c_seq < (uint32_t)kSlots) {
            if (i_st == i_nst) {
                if (i_c + 1 >= c_end) { i_done = true; return; }
                if (i_c + 1 - c_c >= kMeta) return;
                ++i_c;
                begin_chunk(i_c);
                continue;
            }
            issue_stage();
        }
    };
    if (!i_done) {
        begin_chunk(i_c);
        pump();
    }

    // ---------------------------------------------------------- consumer side
    uint32_t qh[4][NT][2], ql[4][NT][2];   // q~^T as B fragments: k-step kb, head tile nt
    float Ms[NT][2], IL[NT][2];            // (M, 1/L) of heads 8 nt + 2 tig + e
    int cur_unit = -1;
    auto load_unit = [&](int unit) {
        const uint16_t *qb = reinterpret_cast<const uint16_t *>(p.qt + (size_t)unit * qblock_bytes(p.Hg));
        #pragma unroll
        for (int nt = 0; nt < NT; ++nt) {
            const int h = 8 * nt + g;
            #pragma unroll
            for (int kb = 0; kb < 4; ++kb)
                #pragma unroll
                for (int hf = 0; hf < 2; ++hf) {
                    const int i = 16 * kb + 8 * hf + 2 * tig;
                    const int off = h * 64 + ((((i >> 3) ^ (h & 7)) & 7) << 3) + (i & 7);
                    qh[kb][nt][hf] = h < p.Hg ? __ldg(reinterpret_cast<const uint32_t *>(qb + off)) : 0u;
                    ql[kb][nt][hf] = h < p.Hg ? __ldg(reinterpret_cast<const uint32_t *>(qb + p.Hg * 64 + off)) : 0u;
                }
            #pragma unroll
            for (int e = 0; e < 2; ++e) {
                const int hh = 8 * nt + 2 * tig + e;
                const float2 st = hh < p.Hg ? __ldg(reinterpret_cast<const float2 *>(p.ustat + ((size_t)unit * p.Hg + hh) * 2))
                                            : make_float2(0.f, 0.f);
                Ms[nt][e] = st.x;
                IL[nt][e] = st.y;
            }
        }
    };
    // the mass of tokens g and g + 8 of a 16-token tile from its logits
    auto tile_mass = [&](const float (&s)[NT][4], float &v0, float &v1) {
        v0 = 0.f;
        v1 = 0.f;
        #pragma unroll
        for (int nt = 0; nt < NT; ++nt)
            #pragma unroll
            for (int e = 0; e < 2; ++e) {
                v0 = fmaf(ex2(s[nt][e] - Ms[nt][e]), IL[nt][e], v0);
                v1 = fmaf(ex2(s[nt][2 + e] - Ms[nt][e]), IL[nt][e], v1);
            }
        v0 += __shfl_xor_sync(0xffffffffu, v0, 1);
        v1 += __shfl_xor_sync(0xffffffffu, v1, 1);
        v0 += __shfl_xor_sync(0xffffffffu, v0, 2);
        v1 += __shfl_xor_sync(0xffffffffu, v1, 2);
    };

    for (; c_c < c_end; ++c_c) {
        pump();
        const int ms = (c_c - c_begin) % kMeta;
        const int unit = sm.meta[warp][ms][0], t0 = sm.meta[warp][ms][1], n = sm.meta[warp][ms][2];
        const int n_hi = sm.meta[warp][ms][3];
        const uint32_t w0 = (uint32_t)sm.meta[warp][ms][4], w1 = (uint32_t)sm.meta[warp][ms][5];
        if (unit != cur_unit) {
            load_unit(unit);
            cur_unit = unit;
        }
        float *mrow = p.mass + (size_t)unit * p.T + t0;
        const int nst = (n_hi < n ? 1 : 0) + (n_hi + kHiTok - 1) / kHiTok;
        bool ok = true;
        for (int st = 0; st < nst; ++st) {
            const int slot = c_seq % kSlots;
            if (!mbar_wait(&sm.full[warp][slot], (c_seq / kSlots) & 1u, abort)) { ok = false; break; }
            const uint32_t sb = smem_u32(sm.ring[warp][slot]);
            if (st == 0 && n_hi < n) {
                // C_K lo rows of the chunk (32-byte rows, 32-byte swizzle: chunk c of row r at c ^ ((r >> 2) & 1))
                #pragma unroll
                for (int mt = 0; mt < kChunk / 16; ++mt) {
                    if (16 * mt < n) {
                        uint32_t a[4];
                        const int row = 16 * mt + (lane & 7) + (((lane >> 3) & 1) << 3);
                        const int ch = lane >> 4;
                        ldsm_x4(sb + row * 32 + ((ch ^ ((row >> 2) & 1)) << 4), a[0], a[1], a[2], a[3]);
                        float s[NT][4];
                        #pragma unroll
                        for (int nt = 0; nt < NT; ++nt) {
                            s[nt][0] = s[nt][1] = s[nt][2] = s[nt][3] = 0.f;
                            mma_bf16(s[nt], a, qh[0][nt][0], qh[0][nt][1]);
                            mma_bf16(s[nt], a, ql[0][nt][0], ql[0][nt][1]);
                        }
                        float v0, v1;
                        tile_mass(s, v0, v1);
                        if (tig < 2) {
                            const int r = 16 * mt + g + 8 * tig;
                            const uint32_t wd = r < 32 ? w0 : w1;
                            if (r < n && !((wd >> (r & 31)) & 1u)) mrow[r] = tig ? v1 : v0;
                        }
                    }
                }
            } else {
                const int hs = st - (n_hi < n ? 1 : 0);
                const int cnt = min(kHiTok, n_hi - kHiTok * hs);
                float s[NT][4];
                #pragma unroll
                for (int nt = 0; nt < NT; ++nt) s[nt][0] = s[nt][1] = s[nt][2] = s[nt][3] = 0.f;
                #pragma unroll
                for (int kb = 0; kb < 4; ++kb) {
                    uint32_t a[4];
                    const int row = (lane & 7) + (((lane >> 3) & 1) << 3);
                    const int ch = 2 * kb + (lane >> 4);
                    ldsm_x4(sb + row * 128 + ((ch ^ (row & 7)) << 4), a[0], a[1], a[2], a[3]);
                    #pragma unroll
                    for (int nt = 0; nt < NT; ++nt) {
                        mma_bf16(s[nt], a, qh[kb][nt][0], qh[kb][nt][1]);
                        mma_bf16(s[nt], a, ql[kb][nt][0], ql[kb][nt][1]);
                    }
                }
                float v0, v1;
                tile_mass(s, v0, v1);
                if (tig < 2) {
                    const int r = g + 8 * tig;
                    if (r < cnt) mrow[sm.hi_list[warp][ms][kHiTok * hs + r]] = tig ? v1 : v0;
                }
            }
            ++c_seq;
            __syncwarp();
            pump();
        }
        if (!ok) {
            *abort = 1;
            break;
        }
    }
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

}  // namespace mass
}  // namespace decode
}  // namespace kvpack
