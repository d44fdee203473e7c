// select.cuh -- importance update and top-k rank mask (AttentionPack decode,
// technical summary 2.B on the fr page: a moving average of the accumulated
// attention ranks the tokens; the top 25 % keep the full rank).
//
// One unit's T keys are held in registers, KPT consecutive tokens per thread
// (blocked layout, so thread order is token order).  The k-th largest key
// theta is built bit by bit from the most significant end: a candidate bit
// is kept when at least k keys are >= the candidate (32 counting passes over
// registers, no data movement).  Then every key > theta is selected, plus the
// first (k - #greater) keys equal to theta in token order (an exclusive scan
// of per-thread equal counts).  Keys are fp32 mapped to order-preserving
// uint32 (-0 as +0, NaN lowest), so the result is exact and matches any
// correct sort with ties to the lower index.
//
// Small T (<= 2048): one warp per unit, 8 units per block.
// Large T (<= 65536): one 1024-thread block per unit.
#pragma once

#include "common.cuh"

namespace kvpack {
namespace select {

__device__ __forceinline__ uint32_t ordered_key(float x) {
    if (x != x) return 0u;           // NaN ranks below every number
    if (x == 0.0f) x = 0.0f;         // -0 ranks as +0
    const uint32_t u = __float_as_uint(x);
    return (u & 0x80000000u) ? ~u : (u | 0x80000000u);
}

struct Params {
    const float *mass;
    float *score;
    float alpha;
    int k, T, nwords, n_units;
    uint32_t *mask;
};

// Sum over the threads that share a unit.  NW == 1: the warp; otherwise the block.
template <int NW>
__device__ __forceinline__ int group_sum(int v, int *red) {
    v = __reduce_add_sync(0xffffffffu, v);
    if constexpr (NW == 1) {
        return v;
    } else {
        const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
        if (lane == 0) red[warp] = v;
        __syncthreads();
        int s = (lane < NW) ? red[lane] : 0;
        s = __reduce_add_sync(0xffffffffu, s);
        __syncthreads();
        return s;
    }
}

// Exclusive prefix sum over the unit's threads in thread order.
template <int NW>
__device__ __forceinline__ int group_exclusive_scan(int v, int *red) {
    const int lane = threadIdx.x & 31;
    int incl = v;
    #pragma unroll
    for (int d = 1; d < 32; d <<= 1) {
        const int o = __shfl_up_sync(0xffffffffu, incl, d);
        if (lane >= d) incl += o;
    }
    if constexpr (NW == 1) {
        return incl - v;
    } else {
        const int warp = threadIdx.x >> 5;
        if (lane == 31) red[warp] = incl;
        __syncthreads();
        if (warp == 0) {
            int w = (lane < NW) ? red[lane] : 0;
            int wi = w;
            #pragma unroll
            for (int d = 1; d < 32; d <<= 1) {
                const int o = __shfl_up_sync(0xffffffffu, wi, d);
                if (lane >= d) wi += o;
            }
            red[32 + lane] = wi - w;
        }
        __syncthreads();
        const int base = red[32 + warp];
        __syncthreads();
        return base + incl - v;
    }
}

// Keys of the unit: KR per thread in registers, the other KS = KPT - KR in shared memory
// (a 1024-thread block has 64 registers per thread, too few for 64 keys and the rest).
template <int KPT, int NW>
struct KeySplit {
    static constexpr int KR = (NW > 1 && KPT > 32) ? 32 : KPT;
    static constexpr int KS = KPT - KR;
};

template <int KPT, int NW>
constexpr size_t select_smem_bytes() { return (size_t)KeySplit<KPT, NW>::KS * 32 * NW * sizeof(uint32_t); }

template <int KPT, int NW>
__global__ void __launch_bounds__(NW == 1 ? 256 : 32 * NW) select_kernel(Params p) {
    constexpr int KR = KeySplit<KPT, NW>::KR, KS = KeySplit<KPT, NW>::KS;
    __shared__ int red[64];
    extern __shared__ uint32_t skeys[];     // [KS][threads]: key KR + i of thread r at [i][r]
    int unit, r;
    if constexpr (NW == 1) {
        unit = blockIdx.x * (blockDim.x >> 5) + (threadIdx.x >> 5);
        r = threadIdx.x & 31;
        if (unit >= p.n_units) return;      // whole warp leaves together
    } else {
        unit = blockIdx.x;
        r = threadIdx.x;
    }
    const int T = p.T;
    const size_t ub = (size_t)unit * T;
    const float one_minus = __fsub_rn(1.0f, p.alpha);

    auto load_key = [&](int i) -> uint32_t {
        const int t = r * KPT + i;
        if (t >= T) return 0u;
        const float m = p.mass[ub + t];
        float x;
        if (p.alpha == 0.0f) x = m;
        else x = __fmaf_rn(p.alpha, p.score[ub + t], __fmul_rn(one_minus, m));
        if (p.score != nullptr) p.score[ub + t] = x;
        return ordered_key(x);
    };
    uint32_t key[KR];
    #pragma unroll
    for (int i = 0; i < KR; ++i) key[i] = load_key(i);
    if constexpr (KS > 0) {
        for (int i = 0; i < KS; ++i) skeys[i * blockDim.x + r] = load_key(KR + i);
    }
    auto skey = [&](int i) -> uint32_t { return skeys[i * blockDim.x + r]; };

    uint32_t *out = p.mask + (size_t)unit * p.nwords;
    if (p.k <= 0) {
        for (int wd = r; wd < p.nwords; wd += 32 * NW) out[wd] = 0u;
        return;
    }

    // theta = largest x with #{key >= x} >= k  (the k-th largest key)
    uint32_t theta = 0u;
    for (int bit = 31; bit >= 0; --bit) {
        const uint32_t cand = theta | (1u << bit);
        int c = 0;
        #pragma unroll
        for (int i = 0; i < KR; ++i) c += (key[i] >= cand) ? 1 : 0;
        if constexpr (KS > 0) {
            #pragma unroll 8
            for (int i = 0; i < KS; ++i) c += (skey(i) >= cand) ? 1 : 0;
        }
        if (group_sum<NW>(c, red) >= p.k) theta = cand;
    }
    int gt = 0, eq = 0;
    #pragma unroll
    for (int i = 0; i < KR; ++i) {
        gt += (key[i] > theta) ? 1 : 0;
        eq += (key[i] == theta) ? 1 : 0;
    }
    if constexpr (KS > 0) {
        for (int i = 0; i < KS; ++i) {
            const uint32_t kk = skey(i);
            gt += (kk > theta) ? 1 : 0;
            eq += (kk == theta) ? 1 : 0;
        }
    }
    const int need = p.k - group_sum<NW>(gt, red);      // equal keys to take, >= 1
    int before = group_exclusive_scan<NW>(eq, red);     // equal keys at lower token indices

    // bits of this thread's KPT tokens, then whole mask words
    if constexpr (KPT >= 32) {
        #pragma unroll
        for (int wd = 0; wd < KPT / 32; ++wd) {
            uint32_t bits = 0u;
            #pragma unroll
            for (int b = 0; b < 32; ++b) {
                const int i = wd * 32 + b;
                uint32_t kk;
                if (i < KR) kk = key[i < KR ? i : 0];
                else kk = skey(i - KR);
                bool s = kk > theta;
                if (kk == theta) { s = before < need; ++before; }
                if (s) bits |= 1u << b;
            }
            const int widx = r * (KPT / 32) + wd;
            if (widx < p.nwords) out[widx] = bits;
        }
    } else {
        uint32_t bits = 0u;
        #pragma unroll
        for (int i = 0; i < KPT; ++i) {
            bool s = key[i] > theta;
            if (key[i] == theta) { s = before < need; ++before; }
            if (s) bits |= 1u << (((r * KPT) & 31) + i);
        }
        constexpr int share = 32 / KPT;      // threads per mask word
        #pragma unroll
        for (int d = 1; d < share; d <<= 1) bits |= __shfl_xor_sync(0xffffffffu, bits, d);
        const int widx = (r * KPT) >> 5;
        if ((r % share) == 0 && widx < p.nwords) out[widx] = bits;
    }
}

}  // namespace select
}  // namespace kvpack
