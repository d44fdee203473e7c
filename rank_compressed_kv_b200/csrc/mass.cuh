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
constexpr int kSegChunks = 32;      // chunks of one unit per segment: 2048 tokens, 64 mask words
constexpr int kSegTok = kSegChunks * kChunk;

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
    uint16_t hi_list[kWarps][kSegTok];        // segment-relative positions of the issue side's full-rank tokens
    uint32_t mw[kWarps][kSegTok / 32];        // that segment's mask words
    int desc[kWarps][kSlots][6];              // per ring slot: type, unit, t0, n, mask words 0 and 1
    uint16_t pos[kWarps][kSlots][kHiTok];     // per gathered slot: the tokens' positions in the unit
    uint64_t full[kWarps][kSlots];
    int abort;
};

constexpr size_t smem_bytes() { return sizeof(Smem) + 1024; }

// Every warp owns a contiguous range of chunks (unit, 64 tokens), taken in
// segments of up to 32 chunks of one unit, and streams it through a private
// ring: per chunk one TMA stage of C_K lo rows (skipped when every token is
// full-rank), then the segment's full-rank tokens 16 at a time (C_lo + C_hi
// rows gathered by cp.async; the issue side lists them once per segment).
// Logits with tokens on M and heads on N (NT tiles of 8) of mma.sync
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
    constexpr int kTypeLo = 0, kTypeHi = 1;
    int i_c = c_begin;                               // first chunk of the next segment
    int i_unit = 0, i_t0 = 0, i_n = 0;               // the segment being issued
    int i_sub = 0, i_lo = 0, i_hi = 0, i_nhi = 0, i_left = 0;
    uint32_t i_seq = 0, c_seq = 0;
    bool i_done = c_begin >= c_end;
    auto begin_segment = [&]() -> bool {
        if (i_c >= c_end) return false;
        i_unit = i_c / p.cpu;
        const int k0 = i_c % p.cpu;
        const int nch = min(min(kSegChunks, p.cpu - k0), c_end - i_c);
        i_c += nch;
        i_t0 = k0 * kChunk;
        i_n = min(nch * kChunk, p.T - i_t0);
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
            const int c_pair = c + __shfl_down_sync(0xffffffffu, c, 1);
            const bool lo_st = (lane & 1) == 0 && wi < nw && c_pair < min(kChunk, i_n - 32 * wi);
            n_lo_st += __popc(__ballot_sync(0xffffffffu, lo_st));
            base += __shfl_sync(0xffffffffu, incl, 31);
        }
        i_nhi = base;
        i_hi = 0;
        i_sub = 0;
        i_lo = n_lo_st;
        i_left = n_lo_st + (i_nhi + kHiTok - 1) / kHiTok;
        __syncwarp();
        return true;
    };
    auto issue_stage = [&]() {
        const int slot = i_seq % kSlots;
        unsigned char *dst = sm.ring[warp][slot];
        uint64_t *bar = &sm.full[warp][slot];
        int type, n, t0 = 0;
        uint32_t w0 = 0u, w1 = 0u;
        __syncwarp();
        if (i_lo > 0) {
            // the next chunk with a reduced-rank token (one exists)
            while (true) {
                n = min(kChunk, i_n - kChunk * i_sub);
                w0 = sm.mw[warp][2 * i_sub];
                w1 = n > 32 ? sm.mw[warp][2 * i_sub + 1] : 0u;
                if (__popc(w0) + __popc(w1) < n) break;
                ++i_sub;
            }
            type = kTypeLo;
            t0 = i_t0 + kChunk * i_sub;
            const int nb = (n + 31) >> 5;
            if (lane == 0) {
                fence_proxy_async();
                mbar_arrive_tx(bar, (uint32_t)nb * 1024u);
                for (int b = 0; b < nb; ++b) tma_3d(dst + 1024 * b, &p.tm_ck, 0, t0 + 32 * b, i_unit, bar);
            } else {
                mbar_arrive(bar);
            }
            ++i_sub;
            --i_lo;
        } else {
            // kHiTok full-rank tokens: C_lo + C_hi into 128-byte rows (16-byte chunk c of row r at
            // c ^ (r & 7)); rows past the count are left alone
            type = kTypeHi;
            n = min(kHiTok, i_nhi - i_hi);
            const size_t ubase = (size_t)i_unit * p.T + i_t0;
            if (lane < n) sm.pos[warp][slot][lane] = (uint16_t)(i_t0 + sm.hi_list[warp][i_hi + lane]);
            #pragma unroll
            for (int i = 0; i < kHiTok / 4; ++i) {
                const int idx = lane + 32 * i;
                const int r = idx >> 3, ch = idx & 7;
                if (r < n) {
                    const size_t row = ubase + sm.hi_list[warp][i_hi + r];
                    const uint16_t *src = ch < 2 ? p.CK_lo + row * 16 + ch * 8 : p.CK_hi + row * 48 + (ch - 2) * 8;
                    cp_async16(dst + r * 128 + ((ch ^ (r & 7)) << 4), src);
                }
            }
            cp_async_arrive_noinc(bar);
            i_hi += n;
        }
        --i_left;
        if (lane == 0) {
            int *d = sm.desc[warp][slot];
            d[0] = type; d[1] = i_unit; d[2] = t0; d[3] = n; d[4] = (int)w0; d[5] = (int)w1;
        }
        __syncwarp();
        ++i_seq;
    };
    auto pump = [&]() {
        while (!i_done && i_seq - c_seq < (uint32_t)kSlots) {
            if (i_left == 0 && !begin_segment()) {
                i_done = true;
                return;
            }
            issue_stage();
        }
    };
    pump();

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

    bool ok = true;
    while (true) {
        pump();
        if (c_seq == i_seq) break;   // nothing in flight, nothing left to issue
        const int slot = c_seq % kSlots;
        if (!mbar_wait(&sm.full[warp][slot], (c_seq / kSlots) & 1u, abort)) { ok = false; break; }
        const int *dsc = sm.desc[warp][slot];
        const int type = dsc[0], unit = dsc[1], t0 = dsc[2], n = dsc[3];
        if (unit != cur_unit) {
            load_unit(unit);
            cur_unit = unit;
        }
        float *mrow = p.mass + (size_t)unit * p.T;
        const uint32_t sb = smem_u32(sm.ring[warp][slot]);
        if (type == kTypeLo) {
            // C_K lo rows of the chunk (32-byte rows, 32-byte swizzle: chunk c of row r at c ^ ((r >> 2) & 1))
            const uint32_t w0 = (uint32_t)dsc[4], w1 = (uint32_t)dsc[5];
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
                        if (r < n && !((wd >> (r & 31)) & 1u)) mrow[t0 + r] = tig ? v1 : v0;
                    }
                }
            }
        } else {
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
                if (r < n) mrow[sm.pos[warp][slot][r]] = tig ? v1 : v0;
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

}  // namespace mass
}  // namespace decode
}  // namespace kvpack
