// select.cuh -- importance update and top-k rank mask (AttentionPack decode,
// technical summary 2.B on the fr page: a moving average of the accumulated
// attention ranks the tokens; the top 25 % keep the full rank).
//
// One unit's T keys are held in registers, KPT per thread: strided (key i of
// thread r is token i * threads + r) in the warp and block forms, blocked (KPT
// consecutive tokens) in the cluster form.  The k-th largest key theta is
// built from the most significant end: a candidate bit is kept when at least
// k keys are >= the candidate (counting passes over registers, no data
// movement; one bit per pass, two in the cluster kernel, whose passes end at
// a cluster barrier).  The search stops early at an accepted candidate with
// exactly k keys at or above it: those k keys are the top k.  Then every key
// > theta is selected, plus the first (k - #greater) keys equal to theta in
// token order.  Keys are fp32 mapped to order-preserving uint32 (-0 as +0,
// NaN lowest), so the result is exact and matches any correct sort with ties
// to the lower index.
//
// Small T (<= 2048): one warp per unit, 8 units per block (up to 64 keys per lane).
// Medium T (<= 8192): one block of 256 threads per unit (9 to 32 keys per thread).
// Large T (<= 65536): a cluster of 8 CTAs of 256 threads per unit (up to 32 keys per thread).
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

// Mask bits of a thread's KPT consecutive tokens (blocked layout, thread index r of the unit):
// keys above theta, and the first `need` keys equal to theta in token order (`before` of them
// precede this thread's).  KPT >= 32: whole words per thread; otherwise the words are shared within a warp.
template <int KPT>
__device__ __forceinline__ void write_bits(const uint32_t (&key)[KPT], uint32_t theta, int need, int before, int r,
                                           uint32_t *out, int nwords) {
    if constexpr (KPT >= 32) {
        #pragma unroll
        for (int wd = 0; wd < KPT / 32; ++wd) {
            uint32_t bits = 0u;
            #pragma unroll
            for (int b = 0; b < 32; ++b) {
                const int i = wd * 32 + b;
                bool s = key[i] > theta;
                if (key[i] == theta) { s = before < need; ++before; }
                if (s) bits |= 1u << b;
            }
            const int widx = r * (KPT / 32) + wd;
            if (widx < nwords) out[widx] = bits;
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
        if ((r % share) == 0 && widx < nwords) out[widx] = bits;
    }
}

// Two bits of theta per counting pass (the cluster kernel, where a pass costs a cluster barrier):
// with the bits above b fixed, the thread counts its keys >= theta | j 2^b for j = 1, 2, 3 (j = 1
// and 2 packed as n1 + (n2 << 16): a CTA's count stays below 2^16), and the pass keeps
// the largest j whose count over the unit is >= k.  The counts fall with j, so this is the same
// theta as two one-bit passes (bit b + 1 kept iff n2 >= k; then bit b iff n3 >= k, or n1 >= k).
template <int KPT>
__device__ __forceinline__ void count3(const uint32_t (&key)[KPT], uint32_t theta, int b, int &n12, int &n3) {
    const uint32_t c1 = theta | (1u << b), c2 = theta | (2u << b), c3 = theta | (3u << b);
    int a = 0, d = 0;
    #pragma unroll
    for (int i = 0; i < KPT; ++i) {
        a += (key[i] >= c1 ? 1 : 0) + (key[i] >= c2 ? 0x10000 : 0);
        d += key[i] >= c3 ? 1 : 0;
    }
    n12 = a;
    n3 = d;
}

__device__ __forceinline__ uint32_t digit2(int n1, int n2, int n3, int k) {
    return n3 >= k ? 3u : n2 >= k ? 2u : n1 >= k ? 1u : 0u;
}

// ------------------------------------------------------------ small T: one warp per unit
//
// Strided layout: key i of lane l is token 32 i + l, so every load is coalesced, mask word i is
// the warp's ballot over row i, and KPT (rows) is ceil(T / 32) rounded up to an instantiated size.
template <int KPT>
__global__ void __launch_bounds__(256) select_warp_kernel(Params p) {
    const int unit = blockIdx.x * 8 + (threadIdx.x >> 5), lane = threadIdx.x & 31;
    if (unit >= p.n_units) return;          // whole warp leaves together
    const int T = p.T;
    const size_t ub = (size_t)unit * T;
    const float one_minus = __fsub_rn(1.0f, p.alpha);
    uint32_t key[KPT];
    #pragma unroll
    for (int i = 0; i < KPT; ++i) {
        const int t = 32 * i + lane;
        key[i] = 0u;
        if (t < T) {
            const float m = p.mass[ub + t];
            float x;
            if (p.alpha == 0.0f) x = m;
            else x = __fmaf_rn(p.alpha, p.score[ub + t], __fmul_rn(one_minus, m));
            if (p.score != nullptr) p.score[ub + t] = x;
            key[i] = ordered_key(x);
        }
    }
    uint32_t *out = p.mask + (size_t)unit * p.nwords;
    if (p.k <= 0) {
        for (int wd = lane; wd < p.nwords; wd += 32) out[wd] = 0u;
        return;
    }
    // theta = largest x with #{key >= x} >= k  (the k-th largest key), or the first accepted
    // candidate with exactly k keys above it
    uint32_t theta = 0u;
    for (int bit = 31; bit >= 0; --bit) {
        const uint32_t cand = theta | (1u << bit);
        int c = 0;
        #pragma unroll
        for (int i = 0; i < KPT; ++i) c += (key[i] >= cand) ? 1 : 0;
        const int n = (int)__reduce_add_sync(0xffffffffu, (unsigned)c);
        if (n >= p.k) theta = cand;
        if (n == p.k) break;
    }
    int gt = 0;
    #pragma unroll
    for (int i = 0; i < KPT; ++i) gt += (key[i] > theta) ? 1 : 0;
    const int need = p.k - (int)__reduce_add_sync(0xffffffffu, (unsigned)gt);   // equal keys to take
    // rows in token order: keys above theta, and the first `need` keys equal to theta (padding
    // keys, t >= T, are 0 and come last)
    const uint32_t lower = (1u << lane) - 1u;
    int before = 0;                         // equal keys in the rows above
    uint32_t word = 0u;
    #pragma unroll
    for (int i = 0; i < KPT; ++i) {
        const bool eq = key[i] == theta;
        const uint32_t eqm = __ballot_sync(0xffffffffu, eq);
        const bool sel = key[i] > theta || (eq && before + __popc(eqm & lower) < need);
        const uint32_t w = __ballot_sync(0xffffffffu, sel);
        before += __popc(eqm);
        if (lane == (i & 31)) word = w;
        if ((i & 31) == 31 || i == KPT - 1) {   // lanes 0 .. (i & 31) hold words (i & ~31) + lane
            const int wd = (i & ~31) + lane;
            if (lane <= (i & 31) && wd < p.nwords) out[wd] = word;
        }
    }
}

// ------------------------------------------------------------ medium T: one block per unit
//
// 256 threads, strided as the warp form: key i of thread r is token 256 i + r (row i = mask
// words 8 i .. 8 i + 7, one per warp), KPT = ceil(T / 256) rounded up to an instantiated size.
// A counting pass sums the warps' counts through shared memory with one barrier; the two count
// buffers alternate between passes, so a thread that runs ahead never overwrites counts another
// is still reading.  When not every key equal to theta is taken, a key's rank among the equal
// ones comes from per-row, per-warp counts in shared memory.
constexpr int kBlockThreads = 256;

template <int KPT>
__global__ void __launch_bounds__(kBlockThreads) select_block_kernel(Params p) {
    constexpr int kWarps = kBlockThreads / 32;
    static_assert(kBlockThreads * KPT < 0x10000, "packed counts");
    __shared__ int red[2][kWarps];
    __shared__ int rows[KPT][kWarps];       // keys equal to theta per row and warp (ordered ties)
    const int unit = blockIdx.x;
    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const int T = p.T;
    const size_t ub = (size_t)unit * T;
    const float one_minus = __fsub_rn(1.0f, p.alpha);
    uint32_t key[KPT];
    #pragma unroll
    for (int i = 0; i < KPT; ++i) {
        const int t = kBlockThreads * i + tid;
        key[i] = 0u;
        if (t < T) {
            const float m = p.mass[ub + t];
            float x;
            if (p.alpha == 0.0f) x = m;
            else x = __fmaf_rn(p.alpha, p.score[ub + t], __fmul_rn(one_minus, m));
            if (p.score != nullptr) p.score[ub + t] = x;
            key[i] = ordered_key(x);
        }
    }
    uint32_t *out = p.mask + (size_t)unit * p.nwords;
    if (p.k <= 0) {
        for (int wd = tid; wd < p.nwords; wd += kBlockThreads) out[wd] = 0u;
        return;
    }
    int par = 0;
    auto block_sum = [&](int v) -> int {
        v = (int)__reduce_add_sync(0xffffffffu, (unsigned)v);
        if (lane == 0) red[par][warp] = v;
        __syncthreads();
        int tot = 0;
        #pragma unroll
        for (int w = 0; w < kWarps; ++w) tot += red[par][w];
        par ^= 1;
        return tot;
    };
    uint32_t theta = 0u;
    for (int bit = 31; bit >= 0; --bit) {
        const uint32_t cand = theta | (1u << bit);
        int c = 0;
        #pragma unroll
        for (int i = 0; i < KPT; ++i) c += (key[i] >= cand) ? 1 : 0;
        const int n = block_sum(c);          // the same value in every thread: all leave together
        if (n >= p.k) theta = cand;
        if (n == p.k) break;
    }
    int gt = 0, eq = 0;
    #pragma unroll
    for (int i = 0; i < KPT; ++i) {
        gt += (key[i] > theta) ? 1 : 0;
        eq += (key[i] == theta) ? 1 : 0;
    }
    const int both = block_sum(gt + (eq << 16));
    const int need = p.k - (both & 0xFFFF);  // equal keys to take
    const bool take_all = (both >> 16) <= need;   // block-uniform
    if (!take_all) {
        #pragma unroll
        for (int i = 0; i < KPT; ++i) {
            const uint32_t eqm = __ballot_sync(0xffffffffu, key[i] == theta);
            if (lane == 0) rows[i][warp] = __popc(eqm);
        }
        __syncthreads();
    }
    const uint32_t lower = (1u << lane) - 1u;
    int before = 0;                          // equal keys in the rows above (ordered ties only)
    uint32_t word = 0u;
    #pragma unroll
    for (int i = 0; i < KPT; ++i) {
        const bool eqk = key[i] == theta;
        bool sel = key[i] > theta;
        if (take_all) {
            sel = sel || eqk;
        } else {
            const uint32_t eqm = __ballot_sync(0xffffffffu, eqk);
            int b = before + __popc(eqm & lower);
            for (int w = 0; w < warp; ++w) b += rows[i][w];
            if (eqk) sel = b < need;
            #pragma unroll
            for (int w = 0; w < kWarps; ++w) before += rows[i][w];
        }
        const uint32_t wbits = __ballot_sync(0xffffffffu, sel);
        if (lane == (i & 31)) word = wbits;
        if ((i & 31) == 31 || i == KPT - 1) {   // lanes 0 .. (i & 31) hold rows (i & ~31) + lane
            const int wd = ((i & ~31) + lane) * kWarps + warp;
            if (lane <= (i & 31) && wd < p.nwords) out[wd] = word;
        }
    }
}

// ------------------------------------------------------------ large T: a cluster of CTAs per unit
//
// The unit's keys are spread over kClusterCtas CTAs of 256 threads (KPT keys per thread, in
// registers).  Each counting pass sums the CTA's count, stores it into every CTA's shared
// memory (distributed shared memory) and meets the others at one cluster barrier; the count
// buffers alternate between passes, so a CTA that runs ahead never overwrites counts another
// is still reading.  CTA rank order is token order, so the tie scan over CTAs is a prefix of
// their equal-key counts.
constexpr int kClusterCtas = 8;
constexpr int kClusterThreads = 256;

__device__ __forceinline__ void cluster_sync_all() {
    asm volatile("barrier.cluster.arrive.release.aligned;\n\tbarrier.cluster.wait.acquire.aligned;" ::: "memory");
}

__device__ __forceinline__ uint32_t cluster_rank() {
    uint32_t r;
    asm volatile("mov.u32 %0, %%cluster_ctarank;" : "=r"(r));
    return r;
}

// store v into word `idx` of the shared array `arr` of the CTA with cluster rank `cta`
__device__ __forceinline__ void st_cluster(int *arr, int idx, uint32_t cta, int v) {
    uint32_t local = smem_u32(arr + idx), remote;
    asm volatile("mapa.shared::cluster.u32 %0, %1, %2;" : "=r"(remote) : "r"(local), "r"(cta));
    asm volatile("st.shared::cluster.u32 [%0], %1;" :: "r"(remote), "r"(v) : "memory");
}

template <int KPT>
__global__ void __cluster_dims__(kClusterCtas, 1, 1) __launch_bounds__(kClusterThreads)
    select_cluster_kernel(Params p) {
    static_assert(kClusterThreads * KPT < 0x10000, "packed counts");
    static_assert(kClusterThreads / 32 == 8 && kClusterCtas == 8, "warp and CTA sums: groups of 8 lanes");
    __shared__ int red[2][2][kClusterThreads / 32];   // [parity][packed pair, third count][warp]
    __shared__ int counts[2][2][kClusterCtas];       // [parity][packed pair, third count][cta]
    const uint32_t rank = cluster_rank();
    const int unit = blockIdx.x / kClusterCtas;
    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const int r = (int)rank * kClusterThreads + tid;   // thread index within the unit
    const int T = p.T;
    const size_t ub = (size_t)unit * T;
    const float one_minus = __fsub_rn(1.0f, p.alpha);
    uint32_t key[KPT];
    #pragma unroll
    for (int i = 0; i < KPT; ++i) {
        const int t = r * KPT + i;
        key[i] = 0u;
        if (t < T) {
            const float m = p.mass[ub + t];
            float x;
            if (p.alpha == 0.0f) x = m;
            else x = __fmaf_rn(p.alpha, p.score[ub + t], __fmul_rn(one_minus, m));
            if (p.score != nullptr) p.score[ub + t] = x;
            key[i] = ordered_key(x);
        }
    }
    uint32_t *out = p.mask + (size_t)unit * p.nwords;
    if (p.k <= 0) {   // uniform across the cluster: no barrier is skipped by only some CTAs
        for (int wd = r; wd < p.nwords; wd += kClusterCtas * kClusterThreads) out[wd] = 0u;
        return;
    }
    cluster_sync_all();   // every CTA of the cluster has started before any stores into its shared memory
    // sums over the unit's threads of a packed pair of counts (ab = a + (b << 16)) and of a third
    // count c: each CTA's sums go into every CTA's buffers of this parity (lane 8 j + d of warp 0
    // stores sum j into CTA d), one cluster barrier, then each CTA adds the 8 CTAs' fields; also
    // the b field summed over the CTAs of lower rank
    int par = 0;
    auto cluster_sum = [&](int ab, int c, int &a_tot, int &b_tot, int &c_tot, int &b_lower) {
        ab = (int)__reduce_add_sync(0xffffffffu, (unsigned)ab);
        c = (int)__reduce_add_sync(0xffffffffu, (unsigned)c);
        if (lane == 0) {
            red[par][0][warp] = ab;
            red[par][1][warp] = c;
        }
        __syncthreads();
        if (warp == 0) {
            int s = lane < 16 ? red[par][lane >> 3][lane & 7] : 0;
            s += __shfl_xor_sync(0xffffffffu, s, 1);
            s += __shfl_xor_sync(0xffffffffu, s, 2);
            s += __shfl_xor_sync(0xffffffffu, s, 4);
            if (lane < 16) st_cluster(&counts[par][lane >> 3][0], (int)rank, (uint32_t)(lane & 7), s);
        }
        cluster_sync_all();
        int sa = 0, sb = 0, sc = 0, lb = 0;
        #pragma unroll
        for (int d = 0; d < kClusterCtas; ++d) {
            const int x = counts[par][0][d];
            sa += x & 0xFFFF;
            sb += x >> 16;
            sc += counts[par][1][d];
            lb += d < (int)rank ? x >> 16 : 0;
        }
        a_tot = sa;
        b_tot = sb;
        c_tot = sc;
        b_lower = lb;
        par ^= 1;
    };
    uint32_t theta = 0u;
    for (int b = 30; b >= 0; b -= 2) {
        int n12, n3, t1, t2, t3, unused;
        count3<KPT>(key, theta, b, n12, n3);
        cluster_sum(n12, n3, t1, t2, t3, unused);     // the same sums in every CTA: all leave together
        const uint32_t d = digit2(t1, t2, t3, p.k);
        theta |= d << b;
        if (d != 0u && (d == 3u ? t3 : d == 2u ? t2 : t1) == p.k) break;
    }
    int gt = 0, eq = 0;
    #pragma unroll
    for (int i = 0; i < KPT; ++i) {
        gt += (key[i] > theta) ? 1 : 0;
        eq += (key[i] == theta) ? 1 : 0;
    }
    // equal keys at lower token indices: CTAs of lower rank, then lower threads of this CTA
    int incl = eq;
    #pragma unroll
    for (int d = 1; d < 32; d <<= 1) {
        const int o = __shfl_up_sync(0xffffffffu, incl, d);
        if (lane >= d) incl += o;
    }
    __shared__ int wsum[kClusterThreads / 32];
    if (lane == 31) wsum[warp] = incl;                     // read after the sum's barriers
    int gt_tot, eq_tot, unused, low_ctas;
    cluster_sum(gt + (eq << 16), 0, gt_tot, eq_tot, unused, low_ctas);
    const int need = p.k - gt_tot;                         // equal keys to take
    int low_warps = 0;
    for (int w2 = 0; w2 < warp; ++w2) low_warps += wsum[w2];
    int before = low_ctas + low_warps + incl - eq;
    write_bits<KPT>(key, theta, need, before, r, out, p.nwords);
    cluster_sync_all();   // no CTA leaves while another may still store into its shared memory
}

}  // namespace select
}  // namespace kvpack
