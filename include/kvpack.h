/*
 * kvpack.h -- C ABI of libkvpack: decode-time attention over a multi-head,
 * SVD-compressed visual KV cache with attention-aware partial decompression
 * (AttentionPack), for NVIDIA B200 (sm_100a).
 *
 * Source of the method: "Attention-aware Inference Optimizations for Large
 * Vision-Language Models with Memory-efficient Decoding" (arXiv 2603.23914),
 * as summarised on its gist.science pages (es, fr, de).  Section names below
 * refer to the technical summaries on those pages.
 *
 * ---------------------------------------------------------------- units
 * The cache is cut into independent UNITS.  A unit is one (layer l, batch
 * row b, KV-head group G): the K (or V) vectors of its g = 4 KV heads,
 * concatenated along the feature axis, form one T x 512 matrix that is
 * compressed by one SVD (multi-head compression joins a group's heads before
 * factoring: Methodologie 2.A on the fr page).  Unit index: u = (l * batch + b) * n_groups + G, with
 * n_groups = n_kv_heads / 4, so one layer is a contiguous run of units.
 * Query head h of (l, b) belongs to group G = h / Hg, Hg = 4 * n_q / n_kv,
 * and within its group reads KV head j(h) = (h % Hg) / (n_q / n_kv).
 *
 * Every call covers n_layers consecutive layers; every per-unit pointer
 * points at the first unit of the first of those layers, every per-(l, b)
 * pointer at its first row.  The caller owns every buffer; the library
 * never allocates, frees or synchronises (except kvpack_last_device_status).
 * All calls are asynchronous on the given CUDA stream (a cudaStream_t passed
 * as void*; NULL is the legacy default stream) and run on the current device.
 *
 * ------------------------------------------------------------- layouts
 * bf16 values are passed as uint16_t bit patterns, row-major, no padding:
 *   X       [units][T][512]        visual K or V of each unit (compression input)
 *   C_lo    [units][T][16]         leading r_lo = 16 coefficients of each token
 *   C_hi    [units][T][48]         coefficients 16..63 of each token
 *   B       [units][64][512]       basis (decompression matrix), orthonormal rows
 *   sigma   [units][64]  fp32      singular values, descending
 *   K_text, V_text [units][L_cap][4][128]   uncompressed text tail
 *   q, out  [n_layers*batch][n_q][128]      decode queries / attention outputs
 *   mask    [units][ceil(T/32)] uint32      rank mask: bit t = (mask[t>>5] >> (t&31)) & 1
 *   mass, score [units][T] fp32
 * The coefficient planes are split at r_lo so that a reduced-rank token is
 * one contiguous 32-byte row and a full-rank token adds one 96-byte row.
 * Every pointer must be 16-byte aligned (KVPACK_ERR_ALIGNMENT otherwise).
 *
 * --------------------------------------------------------------- errors
 * Argument errors return a status before anything is launched.  Device-side
 * failures (an iteration cap reached, a bounded wait that expired) never
 * trap: they set a per-device error word that kvpack_last_device_status()
 * reads and clears.
 */
#ifndef KVPACK_H
#define KVPACK_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

#define KVPACK_VERSION 1
#define KVPACK_GROUP 4       /* g: KV heads merged into one SVD */
#define KVPACK_HEAD_DIM 128  /* d */
#define KVPACK_RANK 64       /* r: rank of the compressed cache */
#define KVPACK_RANK_LO 16    /* r_lo = r / 4: rank of low-importance tokens */
#define KVPACK_MAX_T 65536        /* visual tokens per unit, at most */
#define KVPACK_MAX_TEXT 65536     /* text-tail capacity per unit, at most */

typedef enum {
    KVPACK_OK = 0,
    KVPACK_ERR_INVALID_ARG = 1,   /* null pointer, non-positive size, k_hi out of range, ... */
    KVPACK_ERR_ALIGNMENT = 2,     /* a pointer is not 16-byte aligned */
    KVPACK_ERR_UNSUPPORTED = 3,   /* a shape outside the supported set (see kvpack_dims) */
    KVPACK_ERR_WORKSPACE = 4,     /* workspace pointer null or smaller than the query says */
    KVPACK_ERR_CUDA = 5,          /* a CUDA runtime call failed (launch, attribute, ...) */
    KVPACK_ERR_NOCONVERGE = 6,    /* device: eigen-solver hit its iteration cap */
    KVPACK_ERR_TIMEOUT = 7        /* device: a bounded wait expired */
} kvpack_status;

/*
 * Shape of the cache.  Supported: group == 4, head_dim == 128, rank == 64,
 * rank_lo == 16 (a low-importance token is decompressed at rank 16), or
 * rank_lo == 0 (it is not decompressed at all: its key and value are taken as
 * zero -- the variant of Methodik 2.B on the de page; the coefficient layout is
 * the same), n_kv_heads a positive multiple of 4, n_q_heads a positive
 * multiple of n_kv_heads with Hg = 4 * n_q / n_kv <= 32, batch >= 1,
 * 1 <= T_vis <= KVPACK_MAX_T, 0 <= L_text_cap <= KVPACK_MAX_TEXT.
 */
typedef struct {
    int32_t batch;
    int32_t n_q_heads;
    int32_t n_kv_heads;
    int32_t group;
    int32_t head_dim;
    int32_t T_vis;
    int32_t L_text_cap;
    int32_t rank;
    int32_t rank_lo;
} kvpack_dims;

/* ------------------------------------------------------------------ compression
 * kvpack_compress -- multi-head SVD compression of one of K or V for every
 * unit of n_layers layers (Methodologie 2.A on the fr page: K = K* . D_k with
 * K* the T x R coefficients and D_k the R x (H D) decompression matrix; the
 * storage falls from T x H x D to T x R + R x H x D).  Here C = U_r Sigma_r
 * and B = V_r^T of the rank-64 truncated SVD of each unit's X, computed as:
 *   1. G = X^T X (512 x 512, fp32) on the tensor cores;
 *   2. the top-64 eigenpairs of G by blocked subspace iteration with a
 *      Rayleigh-Ritz step (sigma_i = sqrt(lambda_i), B = eigenvectors^T);
 *   3. C = X B^T, rounded to bf16 and split into the C_lo / C_hi planes.
 * The sign of each singular vector, and any rotation inside a cluster of
 * equal singular values, is arbitrary.  sigma may be NULL.
 * ws must hold kvpack_compress_workspace(dims, n_layers) bytes; its contents
 * on entry do not matter.  Device status KVPACK_ERR_NOCONVERGE if the
 * eigen-solver did not settle within its iteration cap (results are still
 * written, from the last iterate).
 */
size_t kvpack_compress_workspace(const kvpack_dims *dims, int32_t n_layers);
kvpack_status kvpack_compress(const kvpack_dims *dims, int32_t n_layers,
                              const uint16_t *X, uint16_t *C_lo, uint16_t *C_hi, uint16_t *B,
                              float *sigma, void *ws, size_t ws_bytes, void *stream);

/* ------------------------------------------------------------------ decode step
 * kvpack_decode_attn -- one decode step of every unit of n_layers layers,
 * with attention-aware partial decompression (Methodologie 2.B on the fr
 * page: high-score tokens are decompressed at the full rank R_kv, the others
 * at R_kv/4).  For each query head h of the unit, j = j(h):
 *   q~_h    = B_K[:, 128 j : 128 j + 128] q_h                       (rank space, 64)
 *   rho_t   = 64 if mask bit t else dims.rank_lo (16, or 0: logit 0, no value)
 *   s_h,t   = scale * sum_{i < rho_t} C_K[t, i] q~_h[i]             (visual, t < T)
 *   s_h,T+u = scale * q_h . K_text[u, j]                           (text, u < L_text)
 *   p_h     = softmax over the T + L_text logits
 *   o_h     = (sum_t p_h,t C_V[t, :rho_t]) B_V[:rho_t, 128 j : +128] + sum_u p_h,T+u V_text[u, j]
 *   mass_t  = sum_h p_h,t over the unit's Hg query heads           (visual tokens only)
 * This equals decompressing every token at its rank and attending over the
 * decompressed cache; K and V are never materialised.  Accumulation is fp32;
 * out is rounded to bf16.  mass may be NULL.  0 <= L_text <= L_text_cap.
 * ws must hold kvpack_decode_workspace(dims, n_layers) bytes; contents on
 * entry do not matter.  The work split depends on the shapes alone, so
 * repeated calls give identical bits.  No thread block waits on another; device status
 * KVPACK_ERR_TIMEOUT means a bounded wait for a copy into shared memory
 * expired (out and mass are then invalid).
 */
size_t kvpack_decode_workspace(const kvpack_dims *dims, int32_t n_layers);
kvpack_status kvpack_decode_attn(const kvpack_dims *dims, int32_t n_layers,
                                 const uint16_t *q,
                                 const uint16_t *CK_lo, const uint16_t *CK_hi, const uint16_t *BK,
                                 const uint16_t *CV_lo, const uint16_t *CV_hi, const uint16_t *BV,
                                 const uint16_t *K_text, const uint16_t *V_text, int32_t L_text,
                                 const uint32_t *mask, float softmax_scale,
                                 uint16_t *out, float *mass,
                                 void *ws, size_t ws_bytes, void *stream);

/* ------------------------------------------- decode step, text compressed too
 * kvpack_decode_attn_tb -- the decode step of kvpack_decode_attn when the text
 * tokens are SVD-compressed as well, with a basis of their own (the visual and
 * the text tokens are factored separately: Methodologie 2.A on the fr page,
 * Metodologia 2.A on the es page).  A unit's attention then runs over
 *   T visual tokens    at their mask's rank, through the visual basis (as in
 *                      kvpack_decode_attn),
 *   tb->L_c text tokens at the full rank 64, through the text basis:
 *                      s_h,t = scale * C_K'[t, :] . (B_K'[:, 128 j : +128] q_h),
 *                      value C_V'[t, :] B_V'[:, 128 j : +128],
 *   L_text tokens      of the uncompressed tail (the tokens generated since the
 *                      text was compressed), as in kvpack_decode_attn,
 * with one softmax over all T + L_c + L_text logits.  The text planes follow the
 * visual layouts with L_c in place of T (C_K' lo [units][L_c][16], hi
 * [units][L_c][48], B_K' [units][64][512], the same for V); mass covers the
 * visual tokens only.  tb->L_c = 0 gives exactly kvpack_decode_attn.
 * ws must hold kvpack_decode_tb_workspace(dims, n_layers, tb->L_c) bytes; all
 * other arguments, results and errors are those of kvpack_decode_attn, plus
 * KVPACK_ERR_INVALID_ARG for a null tb, L_c < 0 or > KVPACK_MAX_T, or a null
 * text plane when L_c > 0.
 */
typedef struct kvpack_text_basis {
    const uint16_t *CK_lo, *CK_hi, *BK;
    const uint16_t *CV_lo, *CV_hi, *BV;
    int32_t L_c;
} kvpack_text_basis;

size_t kvpack_decode_tb_workspace(const kvpack_dims *dims, int32_t n_layers, int32_t L_c);
kvpack_status kvpack_decode_attn_tb(const kvpack_dims *dims, int32_t n_layers,
                                    const uint16_t *q,
                                    const uint16_t *CK_lo, const uint16_t *CK_hi, const uint16_t *BK,
                                    const uint16_t *CV_lo, const uint16_t *CV_hi, const uint16_t *BV,
                                    const kvpack_text_basis *tb,
                                    const uint16_t *K_text, const uint16_t *V_text, int32_t L_text,
                                    const uint32_t *mask, float softmax_scale,
                                    uint16_t *out, float *mass,
                                    void *ws, size_t ws_bytes, void *stream);

/* -------------------------------------------------------- 4-bit coefficients
 * The pages compose the compression with 4-bit quantisation (Contribuciones §3 on
 * the es page, Compatibilite §4 on the fr page, Ergebnisse §4 on the de page) but
 * fix no format.  This library's format: per token and plane (ranks 0..15 and
 * 16..63) symmetric int4 codes q in [-7, 7] and one power-of-two scale 2^e, e the
 * smallest integer with 7 * 2^e >= max |c| (0 for an all-zero plane, clamped to
 * [-127, 127]); q = round-half-even(c / 2^e) -- the block format of the OCP
 * microscaling (MX) specification with an E8M0 scale.  The value is q * 2^e.
 *   Q_lo [units][T][8]   codes of ranks 0..15, code 2k in the low nibble of byte k
 *   Q_hi [units][T][24]  codes of ranks 16..63, same packing
 *   E    [units][T][2]   int8 exponents (e of ranks 0..15, e of ranks 16..63)
 * A reduced-rank token then costs 9 bytes per plane set and a full-rank one 34.
 *
 * kvpack_quantize4 -- codes and exponents of the 16-bit planes C_lo, C_hi (every
 * token of n_layers layers' units; T tokens per unit).
 * kvpack_decode_attn_q4 -- kvpack_decode_attn with the visual coefficients given as
 * 4-bit planes (K: QK_lo, QK_hi, EK; V: QV_lo, QV_hi, EV): the attention of the
 * dequantized coefficients, dequantized on the fly inside the decode (never
 * written to memory).  Workspace, other arguments, results and errors are those
 * of kvpack_decode_attn.
 */
kvpack_status kvpack_quantize4(const kvpack_dims *dims, int32_t n_layers, int32_t T,
                               const uint16_t *C_lo, const uint16_t *C_hi,
                               uint8_t *Q_lo, uint8_t *Q_hi, int8_t *E, void *stream);
kvpack_status kvpack_decode_attn_q4(const kvpack_dims *dims, int32_t n_layers,
                                    const uint16_t *q,
                                    const uint8_t *QK_lo, const uint8_t *QK_hi, const int8_t *EK, const uint16_t *BK,
                                    const uint8_t *QV_lo, const uint8_t *QV_hi, const int8_t *EV, const uint16_t *BV,
                                    const uint16_t *K_text, const uint16_t *V_text, int32_t L_text,
                                    const uint32_t *mask, float softmax_scale,
                                    uint16_t *out, float *mass,
                                    void *ws, size_t ws_bytes, void *stream);

/* ---------------------------------------------------- decode step, no allocation
 * kvpack_decode_attn_noalloc -- the same decode step as kvpack_decode_attn,
 * for callers that cannot hand the library any device memory of their own:
 * for example a plugin or custom operator hosted by a framework that owns
 * all device memory and offers no workspace hook, or a serving loop that
 * forbids allocator calls after start-up because cudaMalloc and cudaFree
 * can stall on device-wide synchronisation.  This entry point has no
 * counterpart in the paper; it only changes where the scratch lives.
 *
 * The scratch (rank-space queries, per-chunk partial results, the units'
 * softmax statistics and the work counters) is a fixed array of
 * KVPACK_NOALLOC_SCRATCH_BYTES compiled into the library as device memory.
 * The call itself allocates nothing and calls no allocating routine.
 *
 * - Where the array lives: CUDA loads the library's device code, and places
 *   the array, on a device the first time any kvpack call runs there (lazy
 *   module loading, the default); from then on that GPU holds the array
 *   until the process exits.  Make one kvpack call per device at start-up,
 *   before any stream capture, so that this happens outside the serving loop.
 * - Every call looks the array's device address up afresh (with the
 *   caller's device current), so a context that was torn down and created
 *   again (cudaDeviceReset) is handled like a first use.
 * - A call whose kvpack_decode_workspace(dims, n_layers) exceeds
 *   KVPACK_NOALLOC_SCRATCH_BYTES returns KVPACK_ERR_WORKSPACE and launches
 *   nothing; split the layers over several calls instead.
 * - All calls on a device share the one array, and it keeps the last call's
 *   contents.  The kernels rewrite every part they read, and the work
 *   counters are cleared on the stream before use.  Calls that overlap on the GPU
 *   (two streams, or two threads with their own streams) race on the array
 *   and give wrong results: order them on one stream or with events.
 * Arguments and results are those of kvpack_decode_attn minus ws / ws_bytes.
 * kvpack_noalloc_scratch_bytes() returns KVPACK_NOALLOC_SCRATCH_BYTES.
 */
#define KVPACK_NOALLOC_SCRATCH_BYTES ((size_t)64 << 20)
kvpack_status kvpack_decode_attn_noalloc(const kvpack_dims *dims, int32_t n_layers,
                                         const uint16_t *q,
                                         const uint16_t *CK_lo, const uint16_t *CK_hi, const uint16_t *BK,
                                         const uint16_t *CV_lo, const uint16_t *CV_hi, const uint16_t *BV,
                                         const uint16_t *K_text, const uint16_t *V_text, int32_t L_text,
                                         const uint32_t *mask, float softmax_scale,
                                         uint16_t *out, float *mass, void *stream);
size_t kvpack_noalloc_scratch_bytes(void);

/* ------------------------------------------------------------------ rank choice
 * kvpack_select -- importance update and rank mask for the next step, every
 * unit of n_layers layers (Methodologie 2.B on the fr page: a moving average,
 * parameter alpha, of the accumulated attention scores ranks the tokens; the
 * top 25 % get the full rank, Resultados on the es page).  In fp32:
 *   key_t = mass_t                                          if alpha == 0
 *   key_t = fmaf(alpha, score_t, (1 - alpha) * mass_t)      otherwise
 * score (may be NULL when alpha == 0) receives key.  mask_out gets bit t set
 * for the k_hi tokens with the largest key, ties to the lower index; -0 ranks
 * as +0 and NaN below every number; every other bit, including those past T
 * in the last word, is cleared.  0 <= k_hi <= T_vis, 0 <= alpha < 1.
 */
kvpack_status kvpack_select(const kvpack_dims *dims, int32_t n_layers,
                            const float *mass, float *score, float alpha, int32_t k_hi,
                            uint32_t *mask_out, void *stream);

/* ------------------------------------------------------------------ baselines
 * The two routes the rank-space decode is measured against.  The fr summary
 * (§4, results) credits the method's fused kernels with a 2.4x lower latency
 * than a standard implementation; these entry points give that comparison a
 * B200 counterpart.  They share the text kernel's streaming attention.
 *
 * kvpack_dense_decode_attn -- standard decode attention over an uncompressed
 * bf16 cache: for each query head h of a unit (KV head j = j(h)),
 *   o_h = softmax_u(scale * q_h . K[u, j]) V[u, j]   over the first L rows
 * of K, V [units][L_cap][4][128] (visual and text tokens alike).  ws must hold
 * kvpack_dense_decode_workspace(dims, n_layers, L_cap) bytes.  1 <= L <= L_cap
 * <= 4 * KVPACK_MAX_T.  dims.T_vis is not used beyond argument checks.
 *
 * kvpack_decompress -- decompress every visual token at its own rank, the
 * first half of the decompress-then-attend route (fr summary 2.B):
 *   K^_t = sum_{i < rho_t} C_K[t, i] B_K[i, :],  V^_t likewise,
 *   rho_t = 64 if mask bit t, else dims.rank_lo (16, or 0 for tokens that are
 *   not decompressed at all)
 * written in bf16 (round to nearest even, fp32 accumulation) to rows 0 .. T-1
 * of K_out, V_out [units][L_cap][4][128]; rows T .. L_cap-1 are left as they
 * are (the caller's text tail), so kvpack_dense_decode_attn over T + L_text
 * rows then attends over the decompressed cache.  L_cap >= T_vis.
 */
size_t kvpack_dense_decode_workspace(const kvpack_dims *dims, int32_t n_layers, int32_t L_cap);
kvpack_status kvpack_dense_decode_attn(const kvpack_dims *dims, int32_t n_layers, const uint16_t *q,
                                       const uint16_t *K, const uint16_t *V, int32_t L_cap, int32_t L,
                                       float softmax_scale, uint16_t *out, void *ws, size_t ws_bytes, void *stream);
kvpack_status kvpack_decompress(const kvpack_dims *dims, int32_t n_layers,
                                const uint16_t *CK_lo, const uint16_t *CK_hi, const uint16_t *BK,
                                const uint16_t *CV_lo, const uint16_t *CV_hi, const uint16_t *BV,
                                const uint32_t *mask, uint16_t *K_out, uint16_t *V_out, int32_t L_cap, void *stream);

/* ------------------------------------------------------------------ helpers */

/* Human-readable name of a status. */
const char *kvpack_status_string(kvpack_status s);

/* Synchronises the stream, returns and clears the current device's error word
 * (KVPACK_OK if no kernel reported a failure since the last call). */
kvpack_status kvpack_last_device_status(void *stream);

/*
 * Cache footprint of n_layers layers with L_text text tokens per unit, in
 * bytes (storage accounting of Methodologie 2.A on the fr page):
 *   out[0] dense bf16 K+V cache, visual and text:  units * (T + L) * 512 * 2 * 2
 *   out[1] compressed coefficients of K and V plus the uncompressed text tail:
 *          units * (T * 64 * 2 * 2 + L * 512 * 2 * 2)
 *   out[2] the bases B_K and B_V:                    units * 64 * 512 * 2 * 2
 */
kvpack_status kvpack_footprint(const kvpack_dims *dims, int32_t n_layers, int32_t L_text, uint64_t out[3]);

int32_t kvpack_version(void);

/*
 * Diagnostic, no counterpart in the paper: checks the library's failure path.
 * Launches one thread that waits on a shared-memory barrier for a 16-byte
 * transfer that is never issued, with the bounded wait every kernel here uses
 * but a limit of `cycles` SM clocks (1 .. about 2e9) instead of about one
 * second.  The wait expires, the kernel records KVPACK_ERR_TIMEOUT in the
 * device error word and returns: kvpack_last_device_status() then reports
 * KVPACK_ERR_TIMEOUT and the context stays usable.  Nothing is copied.
 */
kvpack_status kvpack_selftest_bounded_wait(int64_t cycles, void *stream);

#ifdef __cplusplus
}
#endif

#endif /* KVPACK_H */
