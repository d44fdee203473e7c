// kvpack.cu -- the C ABI of libkvpack (see include/kvpack.h): argument
// validation, workspace planning and kernel launches.  Everything that
// computes runs in the kernels of decode.cuh, select.cuh and compress.cuh.
#include <cstdint>
#include <cstring>
#include <mutex>

#include <cuda.h>
#include <cudaTypedefs.h>

#include "kvpack.h"
#include "common.cuh"
#include "decode.cuh"
#include "mass.cuh"
#include "select.cuh"
#include "compress.cuh"

namespace {

constexpr int kMaxDevices = 64;
constexpr int kMaxT = KVPACK_MAX_T;

inline bool aligned16(const void *p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

inline size_t align256(size_t x) { return (x + 255) & ~size_t(255); }

kvpack_status check_dims(const kvpack_dims *d, int32_t n_layers) {
    if (d == nullptr || n_layers <= 0) return KVPACK_ERR_INVALID_ARG;
    if (d->batch <= 0 || d->n_q_heads <= 0 || d->n_kv_heads <= 0 || d->T_vis <= 0 || d->L_text_cap < 0)
        return KVPACK_ERR_INVALID_ARG;
    if (d->group != KVPACK_GROUP || d->head_dim != KVPACK_HEAD_DIM || d->rank != KVPACK_RANK ||
        d->rank_lo != KVPACK_RANK_LO)
        return KVPACK_ERR_UNSUPPORTED;
    if (d->n_kv_heads % KVPACK_GROUP != 0 || d->n_q_heads % d->n_kv_heads != 0) return KVPACK_ERR_UNSUPPORTED;
    if ((d->n_q_heads / d->n_kv_heads) * KVPACK_GROUP > 32) return KVPACK_ERR_UNSUPPORTED;
    if (d->T_vis > kMaxT || d->L_text_cap > KVPACK_MAX_TEXT) return KVPACK_ERR_UNSUPPORTED;
    const long long units = (long long)n_layers * d->batch * (d->n_kv_heads / KVPACK_GROUP);
    if (units > (1LL << 30)) return KVPACK_ERR_UNSUPPORTED;
    return KVPACK_OK;
}

inline int n_units(const kvpack_dims *d, int32_t n_layers) {
    return n_layers * d->batch * (d->n_kv_heads / KVPACK_GROUP);
}

inline int hg(const kvpack_dims *d) { return (d->n_q_heads / d->n_kv_heads) * KVPACK_GROUP; }

// Text tail: work items of kTextChunk tokens per (unit, KV head).
constexpr int kTextChunk = 64;

struct DecodePlan {
    int nmb, S, tps, units, Hg, Sc_max;
    size_t off_qt, off_tp, off_vp, off_ustat, off_counter, total;
};

DecodePlan plan_decode(const kvpack_dims *d, int32_t n_layers) {
    DecodePlan pl{};
    pl.Hg = hg(d);
    pl.nmb = (pl.Hg <= 16) ? 1 : 2;
    pl.units = n_units(d, n_layers);
    // Visual items (unit, chunk of tps tokens) for warps that fetch work from a counter:
    // about six per warp of a full B200 (148 SMs x 16 or 8 warps), so the last round is
    // short; chunks are whole 64-token sub-chunks, between 256 and 2048 tokens, and a
    // unit's chunks are as even as the 64-token grain allows.  The plan depends on the
    // shapes alone, so the workspace size does too.
    const int T = d->T_vis;
    const long long warps = (pl.nmb == 1) ? 148LL * 16 : 148LL * 8;
    long long tgt = ((long long)pl.units * T) / (6 * warps);
    tgt = (tgt + 63) / 64 * 64;
    if (tgt < 256) tgt = 256;
    if (tgt > 2048) tgt = 2048;
    const int S0 = (int)((T + tgt - 1) / tgt);
    pl.tps = ((T + S0 - 1) / S0 + 63) / 64 * 64;
    pl.S = (T + pl.tps - 1) / pl.tps;
    static_assert(kvpack::decode::vis::kMaxItemTok >= 2048, "visual items of up to 2048 tokens");
    pl.Sc_max = (d->L_text_cap + kTextChunk - 1) / kTextChunk;
    size_t off = 0;
    pl.off_qt = off;
    off = align256(off + (size_t)pl.units * kvpack::decode::qblock_bytes(pl.Hg));
    pl.off_tp = off;
    off = align256(off + (size_t)pl.units * pl.Sc_max * pl.Hg * kvpack::decode::kTxtPart * sizeof(float));
    pl.off_vp = off;
    off = align256(off + (size_t)pl.units * pl.S * pl.Hg * kvpack::decode::kVisPart * sizeof(float));
    pl.off_ustat = off;
    off = align256(off + (size_t)pl.units * pl.Hg * 2 * sizeof(float));
    pl.off_counter = off;   // work counters: [0] text kernel, [1] visual kernel
    off = align256(off + 4 * sizeof(unsigned int));
    pl.total = off;
    return pl;
}

struct DeviceInfo {
    bool ready = false;
    unsigned long long ctx_id = 0;       // the context the attributes below were set in
    int sms = 0;
    int mass_blocks[4] = {0, 0, 0, 0};   // resident blocks per SM of mass_kernel<1..4>
};
DeviceInfo g_dev[kMaxDevices];
std::mutex g_dev_mu;

// finish_kernel is instantiated for 1..8 query heads per KV head
template <int PK>
bool finish_attr_one() {
    return cudaFuncSetAttribute(kvpack::decode::finish_kernel<PK>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                (int)kvpack::decode::kFinishSmemMax) == cudaSuccess;
}
bool finish_attrs() {
    return finish_attr_one<1>() && finish_attr_one<2>() && finish_attr_one<3>() && finish_attr_one<4>() &&
           finish_attr_one<5>() && finish_attr_one<6>() && finish_attr_one<7>() && finish_attr_one<8>();
}
cudaError_t launch_finish(int per_kv, const kvpack::decode::FinishParams &fp, int units, size_t smem, cudaStream_t st) {
    namespace dc = kvpack::decode;
    switch (per_kv) {
        case 1: dc::finish_kernel<1><<<units, 256, smem, st>>>(fp); break;
        case 2: dc::finish_kernel<2><<<units, 256, smem, st>>>(fp); break;
        case 3: dc::finish_kernel<3><<<units, 256, smem, st>>>(fp); break;
        case 4: dc::finish_kernel<4><<<units, 256, smem, st>>>(fp); break;
        case 5: dc::finish_kernel<5><<<units, 256, smem, st>>>(fp); break;
        case 6: dc::finish_kernel<6><<<units, 256, smem, st>>>(fp); break;
        case 7: dc::finish_kernel<7><<<units, 256, smem, st>>>(fp); break;
        default: dc::finish_kernel<8><<<units, 256, smem, st>>>(fp); break;
    }
    return cudaGetLastError();
}

// Unique id of the calling thread's current context (cuCtxGetId, looked up once through the
// runtime).  Kernel attributes belong to a context: one torn down and created again
// (cudaDeviceReset) needs them set afresh.
kvpack_status current_context_id(unsigned long long *id) {
    using GetCtx = CUresult (*)(CUcontext *);
    using GetId = CUresult (*)(CUcontext, unsigned long long *);
    static GetCtx get_ctx = nullptr;
    static GetId get_id = nullptr;
    static std::once_flag once;
    std::call_once(once, [] {
        void *f1 = nullptr, *f2 = nullptr;
        cudaDriverEntryPointQueryResult q1, q2;
        if (cudaGetDriverEntryPoint("cuCtxGetCurrent", &f1, cudaEnableDefault, &q1) == cudaSuccess &&
            q1 == cudaDriverEntryPointSuccess &&
            cudaGetDriverEntryPoint("cuCtxGetId", &f2, cudaEnableDefault, &q2) == cudaSuccess &&
            q2 == cudaDriverEntryPointSuccess) {
            get_ctx = reinterpret_cast<GetCtx>(f1);
            get_id = reinterpret_cast<GetId>(f2);
        }
    });
    if (get_ctx == nullptr || get_id == nullptr) return KVPACK_ERR_CUDA;
    CUcontext ctx = nullptr;
    if (get_ctx(&ctx) != CUDA_SUCCESS) return KVPACK_ERR_CUDA;
    if (ctx == nullptr) {   // a thread without a current context: bind the device's primary context
        int dev = 0;
        if (cudaGetDevice(&dev) != cudaSuccess || cudaSetDevice(dev) != cudaSuccess) return KVPACK_ERR_CUDA;
        if (get_ctx(&ctx) != CUDA_SUCCESS || ctx == nullptr) return KVPACK_ERR_CUDA;
    }
    if (get_id(ctx, id) != CUDA_SUCCESS) return KVPACK_ERR_CUDA;
    return KVPACK_OK;
}

kvpack_status device_info(DeviceInfo **out) {
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) return KVPACK_ERR_CUDA;
    unsigned long long ctx_id = 0;
    if (current_context_id(&ctx_id) != KVPACK_OK) return KVPACK_ERR_CUDA;
    std::lock_guard<std::mutex> lk(g_dev_mu);
    DeviceInfo &di = g_dev[dev];
    if (!di.ready || di.ctx_id != ctx_id) {
        di.ready = false;
        di.ctx_id = ctx_id;
        if (cudaDeviceGetAttribute(&di.sms, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess) return KVPACK_ERR_CUDA;
        namespace dc = kvpack::decode;
        if (cudaFuncSetAttribute(dc::vis::vis_kernel<1>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                 (int)dc::vis::smem_bytes<1>()) != cudaSuccess ||
            cudaFuncSetAttribute(dc::vis::vis_kernel<2>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                 (int)dc::vis::smem_bytes<2>()) != cudaSuccess ||
            cudaFuncSetAttribute(dc::text::text_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                 (int)dc::text::smem_bytes()) != cudaSuccess ||
            !finish_attrs())
            return KVPACK_ERR_CUDA;
        // all of the SM's shared memory for these kernels (two visual blocks of the 16-row variant)
        if (cudaFuncSetAttribute(dc::vis::vis_kernel<1>, cudaFuncAttributePreferredSharedMemoryCarveout, 100) != cudaSuccess ||
            cudaFuncSetAttribute(dc::vis::vis_kernel<2>, cudaFuncAttributePreferredSharedMemoryCarveout, 100) != cudaSuccess ||
            cudaFuncSetAttribute(dc::text::text_kernel, cudaFuncAttributePreferredSharedMemoryCarveout, 100) != cudaSuccess)
            return KVPACK_ERR_CUDA;
        {
            const void *mk[4] = {(const void *)dc::mass::mass_kernel<1>, (const void *)dc::mass::mass_kernel<2>,
                                 (const void *)dc::mass::mass_kernel<3>, (const void *)dc::mass::mass_kernel<4>};
            for (int i = 0; i < 4; ++i) {
                if (cudaFuncSetAttribute(mk[i], cudaFuncAttributeMaxDynamicSharedMemorySize, (int)dc::mass::smem_bytes()) != cudaSuccess ||
                    cudaFuncSetAttribute(mk[i], cudaFuncAttributePreferredSharedMemoryCarveout, 100) != cudaSuccess ||
                    cudaOccupancyMaxActiveBlocksPerMultiprocessor(&di.mass_blocks[i], mk[i], dc::mass::kThreads,
                                                                  dc::mass::smem_bytes()) != cudaSuccess ||
                    di.mass_blocks[i] < 1)
                    return KVPACK_ERR_CUDA;
            }
        }
        int b1 = 0, b2 = 0, bt = 0;
        if (cudaOccupancyMaxActiveBlocksPerMultiprocessor(&b1, dc::vis::vis_kernel<1>, dc::vis::kThreads,
                                                          dc::vis::smem_bytes<1>()) != cudaSuccess ||
            cudaOccupancyMaxActiveBlocksPerMultiprocessor(&b2, dc::vis::vis_kernel<2>, dc::vis::kThreads,
                                                          dc::vis::smem_bytes<2>()) != cudaSuccess ||
            cudaOccupancyMaxActiveBlocksPerMultiprocessor(&bt, dc::text::text_kernel, dc::text::kThreads,
                                                          dc::text::smem_bytes()) != cudaSuccess)
            return KVPACK_ERR_CUDA;
        // the visual kernels are sized for Cfg::kBlocks resident blocks per SM
        if (b1 != dc::vis::Cfg<1>::kBlocks || b2 != dc::vis::Cfg<2>::kBlocks || bt < 1) return KVPACK_ERR_CUDA;
        kvpack_status cs = kvpack::compress::prepare_device();
        if (cs != KVPACK_OK) return cs;
        di.ready = true;
    }
    *out = &di;
    return KVPACK_OK;
}

// cuTensorMapEncodeTiled from the driver, looked up once through the runtime
PFN_cuTensorMapEncodeTiled_v12000 g_encode = nullptr;
std::mutex g_encode_mu;

kvpack_status tensor_map_encoder(PFN_cuTensorMapEncodeTiled_v12000 *out) {
    std::lock_guard<std::mutex> lk(g_encode_mu);
    if (g_encode == nullptr) {
        void *fn = nullptr;
        cudaDriverEntryPointQueryResult q;
        if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &fn, cudaEnableDefault, &q) != cudaSuccess ||
            q != cudaDriverEntryPointSuccess || fn == nullptr)
            return KVPACK_ERR_CUDA;
        g_encode = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(fn);
    }
    *out = g_encode;
    return KVPACK_OK;
}

// bf16 tensor map of `rank` dims (innermost first), byte strides of dims 1.., box, swizzle
bool encode_bf16(PFN_cuTensorMapEncodeTiled_v12000 enc, CUtensorMap *m, const void *ptr, int rank,
                 const cuuint64_t *dims, const cuuint64_t *strides, const cuuint32_t *box, CUtensorMapSwizzle sw) {
    cuuint32_t es[4] = {1, 1, 1, 1};
    return enc(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, (cuuint32_t)rank, const_cast<void *>(ptr), dims, strides, box, es,
               CU_TENSOR_MAP_INTERLEAVE_NONE, sw, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
               CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

template <int KPT, int NW>
cudaError_t launch_select(const kvpack::select::Params &p, cudaStream_t st) {
    if (NW == 1) {
        const int grid = (p.n_units + 7) / 8;
        kvpack::select::select_kernel<KPT, 1><<<grid, 256, 0, st>>>(p);
    } else {
        kvpack::select::select_kernel<KPT, 32><<<p.n_units, 1024, 0, st>>>(p);
    }
    return cudaGetLastError();
}

template <int NW>
cudaError_t select_dispatch(int kpt, const kvpack::select::Params &p, cudaStream_t st) {
    switch (kpt) {
        case 1: return launch_select<1, NW>(p, st);
        case 2: return launch_select<2, NW>(p, st);
        case 4: return launch_select<4, NW>(p, st);
        case 8: return launch_select<8, NW>(p, st);
        case 16: return launch_select<16, NW>(p, st);
        case 32: return launch_select<32, NW>(p, st);
        default: return launch_select<64, NW>(p, st);
    }
}

}  // namespace

extern "C" {

int32_t kvpack_version(void) { return KVPACK_VERSION; }

const char *kvpack_status_string(kvpack_status s) {
    switch (s) {
        case KVPACK_OK: return "KVPACK_OK";
        case KVPACK_ERR_INVALID_ARG: return "KVPACK_ERR_INVALID_ARG";
        case KVPACK_ERR_ALIGNMENT: return "KVPACK_ERR_ALIGNMENT";
        case KVPACK_ERR_UNSUPPORTED: return "KVPACK_ERR_UNSUPPORTED";
        case KVPACK_ERR_WORKSPACE: return "KVPACK_ERR_WORKSPACE";
        case KVPACK_ERR_CUDA: return "KVPACK_ERR_CUDA";
        case KVPACK_ERR_NOCONVERGE: return "KVPACK_ERR_NOCONVERGE";
        case KVPACK_ERR_TIMEOUT: return "KVPACK_ERR_TIMEOUT";
    }
    return "KVPACK_ERR_UNKNOWN";
}

kvpack_status kvpack_last_device_status(void *stream) {
    if (cudaStreamSynchronize(static_cast<cudaStream_t>(stream)) != cudaSuccess) return KVPACK_ERR_CUDA;
    unsigned int v = 0, zero = 0;
    if (cudaMemcpyFromSymbol(&v, kvpack::g_error_word, sizeof(v)) != cudaSuccess) return KVPACK_ERR_CUDA;
    if (cudaMemcpyToSymbol(kvpack::g_error_word, &zero, sizeof(zero)) != cudaSuccess) return KVPACK_ERR_CUDA;
    return static_cast<kvpack_status>(v);
}

kvpack_status kvpack_footprint(const kvpack_dims *d, int32_t n_layers, int32_t L_text, uint64_t out[3]) {
    kvpack_status s = check_dims(d, n_layers);
    if (s != KVPACK_OK) return s;
    if (out == nullptr || L_text < 0) return KVPACK_ERR_INVALID_ARG;
    const uint64_t units = (uint64_t)n_units(d, n_layers);
    const uint64_t T = (uint64_t)d->T_vis, L = (uint64_t)L_text, n = KVPACK_GROUP * KVPACK_HEAD_DIM;
    out[0] = units * (T + L) * n * 2 * 2;
    out[1] = units * (T * KVPACK_RANK * 2 * 2 + L * n * 2 * 2);
    out[2] = units * (uint64_t)KVPACK_RANK * n * 2 * 2;
    return KVPACK_OK;
}

// ------------------------------------------------------------------ decode

size_t kvpack_decode_workspace(const kvpack_dims *d, int32_t n_layers) {
    if (check_dims(d, n_layers) != KVPACK_OK) return 0;
    return plan_decode(d, n_layers).total;
}

kvpack_status kvpack_decode_attn(const kvpack_dims *d, int32_t n_layers, const uint16_t *q,
                                 const uint16_t *CK_lo, const uint16_t *CK_hi, const uint16_t *BK,
                                 const uint16_t *CV_lo, const uint16_t *CV_hi, const uint16_t *BV,
                                 const uint16_t *K_text, const uint16_t *V_text, int32_t L_text,
                                 const uint32_t *mask, float softmax_scale, uint16_t *out, float *mass,
                                 void *ws, size_t ws_bytes, void *stream) {
    kvpack_status s = check_dims(d, n_layers);
    if (s != KVPACK_OK) return s;
    if (L_text < 0 || L_text > d->L_text_cap) return KVPACK_ERR_INVALID_ARG;
    if (!q || !CK_lo || !CK_hi || !BK || !CV_lo || !CV_hi || !BV || !mask || !out) return KVPACK_ERR_INVALID_ARG;
    if (L_text > 0 && (!K_text || !V_text)) return KVPACK_ERR_INVALID_ARG;
    if (!(softmax_scale == softmax_scale) || softmax_scale <= 0.f) return KVPACK_ERR_INVALID_ARG;
    const void *ptrs[] = {q, CK_lo, CK_hi, BK, CV_lo, CV_hi, BV, mask, out, mass, ws,
                          L_text > 0 ? K_text : nullptr, L_text > 0 ? V_text : nullptr};
    for (const void *ptr : ptrs)
        if (ptr && !aligned16(ptr)) return KVPACK_ERR_ALIGNMENT;
    const DecodePlan pl = plan_decode(d, n_layers);
    if (pl.S <= 0) return KVPACK_ERR_UNSUPPORTED;
    if ((long long)pl.units * d->T_vis * 3 >= (1LL << 31)) return KVPACK_ERR_UNSUPPORTED;   // int32 gather rows
    if (ws == nullptr || ws_bytes < pl.total) return KVPACK_ERR_WORKSPACE;
    DeviceInfo *di = nullptr;
    if ((s = device_info(&di)) != KVPACK_OK) return s;

    PFN_cuTensorMapEncodeTiled_v12000 enc = nullptr;
    if ((s = tensor_map_encoder(&enc)) != KVPACK_OK) return s;
    namespace dc = kvpack::decode;

    const int T = d->T_vis, Hg = pl.Hg, per_kv = d->n_q_heads / d->n_kv_heads;
    const int groups = d->n_kv_heads / KVPACK_GROUP;
    const int Sc = (L_text + kTextChunk - 1) / kTextChunk;
    const float scale2 = softmax_scale * 1.4426950408889634f;
    unsigned char *w = static_cast<unsigned char *>(ws);
    unsigned char *qt = w + pl.off_qt;
    float *tpart = reinterpret_cast<float *>(w + pl.off_tp);
    float *vpart = reinterpret_cast<float *>(w + pl.off_vp);
    float *ustat = reinterpret_cast<float *>(w + pl.off_ustat);
    unsigned int *counter = reinterpret_cast<unsigned int *>(w + pl.off_counter);
    cudaStream_t st = static_cast<cudaStream_t>(stream);

    // the work counters start at zero
    if (cudaMemsetAsync(counter, 0, 4 * sizeof(unsigned int), st) != cudaSuccess) return KVPACK_ERR_CUDA;

    // 1. q~ per (unit, KV head) and the text tail partials, one persistent launch
    {
        dc::text::Params tp;
        std::memset(&tp, 0, sizeof(tp));
        if (L_text > 0) {
            const cuuint64_t dims[4] = {128, 4, (cuuint64_t)L_text, (cuuint64_t)pl.units};
            const cuuint64_t strides[3] = {256, 1024, (cuuint64_t)d->L_text_cap * 1024};
            const cuuint32_t box[4] = {64, 1, 16, 1};
            if (!encode_bf16(enc, &tp.tm_k, K_text, 4, dims, strides, box, CU_TENSOR_MAP_SWIZZLE_128B) ||
                !encode_bf16(enc, &tp.tm_v, V_text, 4, dims, strides, box, CU_TENSOR_MAP_SWIZZLE_128B))
                return KVPACK_ERR_CUDA;
        }
        {
            const cuuint64_t dims[3] = {512, 64, (cuuint64_t)pl.units};
            const cuuint64_t strides[2] = {1024, 64 * 1024};
            const cuuint32_t box[3] = {64, 64, 1};
            if (!encode_bf16(enc, &tp.tm_bk, BK, 3, dims, strides, box, CU_TENSOR_MAP_SWIZZLE_128B))
                return KVPACK_ERR_CUDA;
        }
        tp.q = q; tp.part = tpart; tp.qt = qt; tp.counter = counter;
        tp.n_units = pl.units; tp.L = L_text; tp.Hg = Hg; tp.per_kv = per_kv; tp.n_q = d->n_q_heads;
        tp.groups = groups; tp.Sc = Sc; tp.ct = kTextChunk; tp.n_qitems = pl.units * 4;
        tp.n_items = tp.n_qitems + pl.units * 4 * Sc; tp.scale2 = scale2;
        const int grid = tp.n_items < di->sms ? tp.n_items : di->sms;
        dc::text::text_kernel<<<grid, dc::text::kThreads, dc::text::smem_bytes(), st>>>(tp);
        if (cudaGetLastError() != cudaSuccess) return KVPACK_ERR_CUDA;
    }

    // 2. the text tail's (max, sum) per head of each unit, into its query block
    dc::text::text_stats_kernel<<<(pl.units + 7) / 8, 256, 0, st>>>(tpart, qt, pl.units, Hg, Sc);
    if (cudaGetLastError() != cudaSuccess) return KVPACK_ERR_CUDA;

    // 3. visual partials and the attention mass
    {
        dc::vis::Params vp;
        std::memset(&vp, 0, sizeof(vp));
        const cuuint64_t dims[3] = {16, (cuuint64_t)T, (cuuint64_t)pl.units};
        const cuuint64_t strides[2] = {32, (cuuint64_t)T * 32};
        const cuuint32_t box[3] = {16, 32, 1};
        if (!encode_bf16(enc, &vp.tm_ck, CK_lo, 3, dims, strides, box, CU_TENSOR_MAP_SWIZZLE_32B) ||
            !encode_bf16(enc, &vp.tm_cv, CV_lo, 3, dims, strides, box, CU_TENSOR_MAP_SWIZZLE_32B))
            return KVPACK_ERR_CUDA;
        vp.CK_lo = CK_lo; vp.CK_hi = CK_hi; vp.CV_lo = CV_lo; vp.CV_hi = CV_hi;
        vp.qt = qt; vp.mask = mask; vp.part = vpart; vp.counter = counter + 1;
        vp.n_units = pl.units; vp.T = T; vp.Hg = Hg; vp.S = pl.S; vp.tps = pl.tps; vp.nwords = (T + 31) / 32;
        vp.n_items = pl.units * pl.S;
        const int resident = di->sms * (pl.nmb == 1 ? dc::vis::Cfg<1>::kBlocks : dc::vis::Cfg<2>::kBlocks);
        const int need = (vp.n_items + dc::vis::kWarps - 1) / dc::vis::kWarps;
        const int grid = need < resident ? need : resident;
        void *args[] = {&vp};
        const void *fn = (pl.nmb == 1) ? (const void *)dc::vis::vis_kernel<1> : (const void *)dc::vis::vis_kernel<2>;
        const size_t smem = (pl.nmb == 1) ? dc::vis::smem_bytes<1>() : dc::vis::smem_bytes<2>();
        const cudaError_t e = cudaLaunchKernel(fn, dim3(grid), dim3(dc::vis::kThreads), args, smem, st);
        if (e != cudaSuccess) return KVPACK_ERR_CUDA;
    }

    // 4. combine and project through B_V
    dc::FinishParams fp{BV, vpart, Sc > 0 ? tpart : nullptr, out, mass != nullptr ? ustat : nullptr,
                        Hg, per_kv, d->n_q_heads, groups, pl.S, Sc};
    if (launch_finish(per_kv, fp, pl.units, dc::finish_smem_bytes(pl.S, Sc, Hg), st) != cudaSuccess)
        return KVPACK_ERR_CUDA;
    if (cudaGetLastError() != cudaSuccess) return KVPACK_ERR_CUDA;
    if (mass == nullptr) return KVPACK_OK;

    // 5. the attention mass of every visual token under the unit's final (max, sum)
    {
        dc::mass::Params mp;
        std::memset(&mp, 0, sizeof(mp));
        const cuuint64_t dims[3] = {16, (cuuint64_t)T, (cuuint64_t)pl.units};
        const cuuint64_t strides[2] = {32, (cuuint64_t)T * 32};
        const cuuint32_t box[3] = {16, 32, 1};
        if (!encode_bf16(enc, &mp.tm_ck, CK_lo, 3, dims, strides, box, CU_TENSOR_MAP_SWIZZLE_32B)) return KVPACK_ERR_CUDA;
        mp.CK_lo = CK_lo; mp.CK_hi = CK_hi; mp.qt = qt; mp.ustat = ustat; mp.mask = mask; mp.mass = mass;
        mp.T = T; mp.Hg = Hg; mp.nwords = (T + 31) / 32; mp.cpu = (T + dc::mass::kChunk - 1) / dc::mass::kChunk;
        mp.n_chunks = pl.units * mp.cpu;
        const int nt = (Hg + 7) / 8;
        const int resident = di->sms * di->mass_blocks[nt - 1];
        const int need = (mp.n_chunks + dc::mass::kWarps - 1) / dc::mass::kWarps;
        const int grid = need < resident ? need : resident;
        const size_t smem = dc::mass::smem_bytes();
        switch (nt) {
            case 1: dc::mass::mass_kernel<1><<<grid, dc::mass::kThreads, smem, st>>>(mp); break;
            case 2: dc::mass::mass_kernel<2><<<grid, dc::mass::kThreads, smem, st>>>(mp); break;
            case 3: dc::mass::mass_kernel<3><<<grid, dc::mass::kThreads, smem, st>>>(mp); break;
            default: dc::mass::mass_kernel<4><<<grid, dc::mass::kThreads, smem, st>>>(mp); break;
        }
    }
    return (cudaGetLastError() == cudaSuccess) ? KVPACK_OK : KVPACK_ERR_CUDA;
}

}  // extern "C"

// ------------------------------------------------------------------ decode without allocation
//
// For callers that cannot give the library device memory (a framework-owned
// plugin with no workspace hook, a serving loop that bans allocator calls):
// the decode scratch lives in this fixed device array, which every GPU holds
// from the library's first use there until exit.  Host code must not pass the
// array's name to a kernel -- on the host it is only a stand-in -- so its
// device address is looked up with the caller's device current.  The lookup
// runs on every call and is not cached: a context torn down and created
// again (cudaDeviceReset) places the array at a new address.

namespace {

static __device__ __align__(256) unsigned char g_noalloc_scratch[KVPACK_NOALLOC_SCRATCH_BYTES];

kvpack_status noalloc_scratch(void **out) {
    void *p = nullptr;
    if (cudaGetSymbolAddress(&p, g_noalloc_scratch) != cudaSuccess || p == nullptr) return KVPACK_ERR_CUDA;
    *out = p;
    return KVPACK_OK;
}

}  // namespace

extern "C" {

size_t kvpack_noalloc_scratch_bytes(void) { return KVPACK_NOALLOC_SCRATCH_BYTES; }

kvpack_status kvpack_decode_attn_noalloc(const kvpack_dims *d, int32_t n_layers, const uint16_t *q,
                                         const uint16_t *CK_lo, const uint16_t *CK_hi, const uint16_t *BK,
                                         const uint16_t *CV_lo, const uint16_t *CV_hi, const uint16_t *BV,
                                         const uint16_t *K_text, const uint16_t *V_text, int32_t L_text,
                                         const uint32_t *mask, float softmax_scale, uint16_t *out, float *mass,
                                         void *stream) {
    kvpack_status s = check_dims(d, n_layers);
    if (s != KVPACK_OK) return s;
    if (plan_decode(d, n_layers).total > KVPACK_NOALLOC_SCRATCH_BYTES) return KVPACK_ERR_WORKSPACE;
    void *ws = nullptr;
    if ((s = noalloc_scratch(&ws)) != KVPACK_OK) return s;
    return kvpack_decode_attn(d, n_layers, q, CK_lo, CK_hi, BK, CV_lo, CV_hi, BV, K_text, V_text, L_text, mask,
                              softmax_scale, out, mass, ws, KVPACK_NOALLOC_SCRATCH_BYTES, stream);
}

// ------------------------------------------------------------------ select

kvpack_status kvpack_select(const kvpack_dims *d, int32_t n_layers, const float *mass, float *score, float alpha,
                            int32_t k_hi, uint32_t *mask_out, void *stream) {
    kvpack_status s = check_dims(d, n_layers);
    if (s != KVPACK_OK) return s;
    if (!mass || !mask_out) return KVPACK_ERR_INVALID_ARG;
    if (k_hi < 0 || k_hi > d->T_vis) return KVPACK_ERR_INVALID_ARG;
    if (!(alpha >= 0.f && alpha < 1.f)) return KVPACK_ERR_INVALID_ARG;
    if (alpha != 0.f && score == nullptr) return KVPACK_ERR_INVALID_ARG;
    if (!aligned16(mass) || !aligned16(mask_out) || (score && !aligned16(score))) return KVPACK_ERR_ALIGNMENT;
    kvpack::select::Params p{};
    p.mass = mass; p.score = score; p.alpha = alpha; p.k = k_hi; p.T = d->T_vis;
    p.nwords = (d->T_vis + 31) / 32; p.n_units = n_units(d, n_layers); p.mask = mask_out;
    cudaStream_t st = static_cast<cudaStream_t>(stream);
    cudaError_t e;
    const int T = d->T_vis;
    if (T <= 32 * 64) {
        int kpt = 1;
        while (32 * kpt < T) kpt <<= 1;
        e = select_dispatch<1>(kpt, p, st);
    } else {
        int kpt = 1;
        while (1024 * kpt < T) kpt <<= 1;
        e = select_dispatch<32>(kpt, p, st);
    }
    return (e == cudaSuccess) ? KVPACK_OK : KVPACK_ERR_CUDA;
}

// ------------------------------------------------------------------ compress

size_t kvpack_compress_workspace(const kvpack_dims *d, int32_t n_layers) {
    if (check_dims(d, n_layers) != KVPACK_OK) return 0;
    return kvpack::compress::workspace_bytes(n_units(d, n_layers), d->T_vis);
}

kvpack_status kvpack_compress(const kvpack_dims *d, int32_t n_layers, const uint16_t *X, uint16_t *C_lo,
                              uint16_t *C_hi, uint16_t *B, float *sigma, void *ws, size_t ws_bytes, void *stream) {
    kvpack_status s = check_dims(d, n_layers);
    if (s != KVPACK_OK) return s;
    if (!X || !C_lo || !C_hi || !B) return KVPACK_ERR_INVALID_ARG;
    const void *ptrs[] = {X, C_lo, C_hi, B, sigma, ws};
    for (const void *ptr : ptrs)
        if (ptr && !aligned16(ptr)) return KVPACK_ERR_ALIGNMENT;
    const int units = n_units(d, n_layers);
    if (ws == nullptr || ws_bytes < kvpack::compress::workspace_bytes(units, d->T_vis)) return KVPACK_ERR_WORKSPACE;
    DeviceInfo *di = nullptr;
    if ((s = device_info(&di)) != KVPACK_OK) return s;
    PFN_cuTensorMapEncodeTiled_v12000 enc = nullptr;
    if ((s = tensor_map_encoder(&enc)) != KVPACK_OK) return s;
    CUtensorMap tm_x;
    {
        const cuuint64_t dims[3] = {512, (cuuint64_t)d->T_vis, (cuuint64_t)units};
        const cuuint64_t strides[2] = {1024, (cuuint64_t)d->T_vis * 1024};
        const cuuint32_t box[3] = {64, 64, 1};
        if (!encode_bf16(enc, &tm_x, X, 3, dims, strides, box, CU_TENSOR_MAP_SWIZZLE_128B)) return KVPACK_ERR_CUDA;
    }
    return kvpack::compress::run(units, d->T_vis, X, tm_x, C_lo, C_hi, B, sigma, ws, di->sms,
                                 static_cast<cudaStream_t>(stream));
}

}  // extern "C"
