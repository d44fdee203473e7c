/*
 * oracle.c -- plain, slow, fp64 CPU oracle for the AttentionPack decode hot path.
 *
 * TEST INFRASTRUCTURE ONLY.  Only tests/, __graft_entry__.smoke() and the
 * cpu_baseline leg of bench.py may load this library.  The product library
 * (libkvpack.so) never links, calls or includes anything from here, and this
 * file includes nothing from the product.
 *
 * Method: "Attention-aware Inference Optimizations for Large Vision-Language
 * Models with Memory-efficient Decoding" (AttentionPack), as summarised on the
 * gist.science pages for arXiv 2603.23914 (es / fr / de).  Every function
 * names the passage it follows:
 *
 *   - Multi-head compression: the K (and separately V) vectors of a group of
 *     heads are concatenated along the feature axis and factored by SVD into
 *     per-token coefficients and a decompression matrix, K ~ K* . D_k
 *     (es page, Technical summary 2.A; fr page, Methodologie 2.A; de page,
 *     Methodik 2.A).  The group is g = 4 KV heads of d = 128 features, r = 64.
 *   - Attention-aware partial decompression: tokens with high importance are
 *     decompressed at the full rank R, the others at a reduced rank R/4
 *     (fr page, Methodologie 2.B; es page 2.B; de page 2.B).
 *   - Importance: a moving average (parameter alpha) of the accumulated
 *     attention (same passages); with alpha = 0 it is the previous step's
 *     attention mass, and the top 25 % of tokens get the full rank
 *     (es page, Resultados, "Analisis de Sensibilidad").
 *
 * Every routine here is written straight from those definitions, in fp64,
 * with no blocking, fusion or reordering beyond what the definition states.
 * The one place that is not fp64 is the top-k selection, which compares fp32
 * keys exactly as the GPU kernel does, because there floating point decides
 * an integer (which bit of the rank mask is set).
 */
#include <math.h>
#include <omp.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>

#define GROUP_HEADS 4   /* g: KV heads merged into one SVD */
#define HEAD_DIM 128    /* d */
#define FEAT (GROUP_HEADS * HEAD_DIM)   /* n = g*d = 512 */

/* ---------------------------------------------------------------- bf16 */

/* Exact widening of a bf16 bit pattern (the upper half of an IEEE binary32). */
double ora_bf16_to_f64(uint16_t h)
{
    uint32_t u = (uint32_t)h << 16;
    float f;
    memcpy(&f, &u, sizeof f);
    return (double)f;
}

/*
 * Round a double to the nearest bf16 (8 significant bits, binary32 exponent
 * range), ties to even, in one rounding step (no intermediate binary32).
 */
uint16_t ora_f64_to_bf16(double x)
{
    if (isnan(x)) return (uint16_t)0x7fc0;
    double ax = fabs(x), r;
    if (ax == 0.0 || isinf(ax)) {
        r = ax;
    } else {
        int e;
        frexp(ax, &e);                 /* ax = m * 2^e, m in [0.5, 1) */
        int q = e - 8;                 /* spacing of 8-bit significands in [2^(e-1), 2^e) */
        if (q < -133) q = -133;        /* bf16 subnormal spacing */
        r = ldexp(nearbyint(ldexp(ax, -q)), q);   /* default mode: nearest, ties to even */
        if (r >= 0x1p128) r = INFINITY;
    }
    float f = (float)r;                /* exact: r has at most 8 significant bits */
    uint32_t u;
    memcpy(&u, &f, sizeof u);
    u >>= 16;
    if (signbit(x)) u |= 0x8000u;
    return (uint16_t)u;
}

void ora_bf16_to_f64_array(const uint16_t *in, double *out, int64_t n)
{
    for (int64_t i = 0; i < n; ++i) out[i] = ora_bf16_to_f64(in[i]);
}

void ora_f64_to_bf16_array(const double *in, uint16_t *out, int64_t n)
{
    for (int64_t i = 0; i < n; ++i) out[i] = ora_f64_to_bf16(in[i]);
}

/* ------------------------------------------------------- SVD (compression) */

/*
 * Householder QR of A (m x n, column-major, m >= n), in place.  On return the
 * upper triangle of the leading n x n block holds R.  Only R is needed: the
 * right singular vectors and singular values of A equal those of R.
 */
static void householder_r(double *A, int64_t m, int n)
{
    double *v = (double *)malloc(sizeof(double) * (size_t)m);
    for (int k = 0; k < n; ++k) {
        double *ak = A + (int64_t)k * m;
        double nrm2 = 0.0;
        for (int64_t i = k; i < m; ++i) nrm2 += ak[i] * ak[i];
        double nrm = sqrt(nrm2);
        if (nrm == 0.0) continue;
        double alpha = (ak[k] >= 0.0) ? -nrm : nrm;
        /* v = x - alpha e1, H = I - 2 v v^T / (v^T v) */
        for (int64_t i = k; i < m; ++i) v[i] = ak[i];
        v[k] -= alpha;
        double vtv = 0.0;
        for (int64_t i = k; i < m; ++i) vtv += v[i] * v[i];
        ak[k] = alpha;
        for (int64_t i = k + 1; i < m; ++i) ak[i] = 0.0;
        if (vtv == 0.0) continue;
        #pragma omp parallel for schedule(static)
        for (int j = k + 1; j < n; ++j) {
            double *aj = A + (int64_t)j * m;
            double dot = 0.0;
            for (int64_t i = k; i < m; ++i) dot += v[i] * aj[i];
            double f = 2.0 * dot / vtv;
            for (int64_t i = k; i < m; ++i) aj[i] -= f * v[i];
        }
    }
    free(v);
}

/*
 * One-sided Jacobi SVD (Hestenes): rotate pairs of columns of A (m x n,
 * column-major) until every pair is orthogonal to within tol, accumulating
 * the rotations in V (n x n, column-major).  Cyclic-by-row pair order.
 * On return the column norms of A are the singular values, V the right
 * singular vectors.  Returns the number of sweeps, or -1 if max_sweeps
 * passed without convergence.
 */
static int jacobi_one_sided(double *A, int64_t m, int n, double *V, double tol, int max_sweeps)
{
    for (int j = 0; j < n; ++j)
        for (int i = 0; i < n; ++i) V[(int64_t)j * n + i] = (i == j) ? 1.0 : 0.0;
    /* ||A||_F^2 is invariant under the rotations; a pair whose inner product is
     * below eps^2 of it is orthogonal to working precision (this matters for
     * rank-deficient inputs, whose null-space columns are roundoff noise). */
    double fro2 = 0.0;
    for (int64_t i = 0; i < m * n; ++i) fro2 += A[i] * A[i];
    const double floor_abs = 0x1p-104 * fro2;   /* (2^-52)^2 ||A||_F^2 */
    for (int sweep = 1; sweep <= max_sweeps; ++sweep) {
        int rotated = 0;
        for (int p = 0; p < n - 1; ++p) {
            for (int q = p + 1; q < n; ++q) {
                double *ap = A + (int64_t)p * m, *aq = A + (int64_t)q * m;
                double alpha = 0.0, beta = 0.0, gamma = 0.0;
                for (int64_t i = 0; i < m; ++i) {
                    alpha += ap[i] * ap[i];
                    beta += aq[i] * aq[i];
                    gamma += ap[i] * aq[i];
                }
                if (alpha == 0.0 || beta == 0.0) continue;
                if (fabs(gamma) <= tol * sqrt(alpha * beta) || fabs(gamma) <= floor_abs) continue;
                rotated = 1;
                /* choose t = tan(theta) that zeroes the off-diagonal of the 2x2 Gram */
                double zeta = (beta - alpha) / (2.0 * gamma);
                double t = ((zeta >= 0.0) ? 1.0 : -1.0) / (fabs(zeta) + sqrt(1.0 + zeta * zeta));
                double c = 1.0 / sqrt(1.0 + t * t), s = c * t;
                for (int64_t i = 0; i < m; ++i) {
                    double x = ap[i], y = aq[i];
                    ap[i] = c * x - s * y;
                    aq[i] = s * x + c * y;
                }
                double *vp = V + (int64_t)p * n, *vq = V + (int64_t)q * n;
                for (int i = 0; i < n; ++i) {
                    double x = vp[i], y = vq[i];
                    vp[i] = c * x - s * y;
                    vq[i] = s * x + c * y;
                }
            }
        }
        if (!rotated) return sweep;
    }
    return -1;
}

/*
 * Full SVD of X (T x n, row-major): singular values sigma[min(T,n)] in
 * descending order and right singular vectors V (n x n, row-major, column j
 * is the j-th vector; columns past min(T,n) span the null space).
 * QR-preconditioned when T > n: Householder R of X, then one-sided Jacobi on
 * R.  Returns the Jacobi sweep count, or -1 on non-convergence.
 */
int ora_svd(const double *X, int64_t T, int n, double *sigma, double *V_out)
{
    int64_t m = (T > n) ? n : T;           /* rows of the matrix Jacobi works on */
    double *W = (double *)malloc(sizeof(double) * (size_t)((T > n ? T : m) * n));
    /* column-major copy of X */
    for (int j = 0; j < n; ++j)
        for (int64_t i = 0; i < T; ++i) W[(int64_t)j * T + i] = X[i * n + j];
    double *A = W;
    double *R = NULL;
    if (T > n) {
        householder_r(W, T, n);
        R = (double *)malloc(sizeof(double) * (size_t)n * n);
        for (int j = 0; j < n; ++j)
            for (int i = 0; i < n; ++i) R[(int64_t)j * n + i] = (i <= j) ? W[(int64_t)j * T + i] : 0.0;
        A = R;
    }
    double *V = (double *)malloc(sizeof(double) * (size_t)n * n);
    int sweeps = jacobi_one_sided(A, m, n, V, 1e-15, 80);
    /* column norms -> singular values; sort descending (stable on index) */
    double *nrm = (double *)malloc(sizeof(double) * n);
    int *order = (int *)malloc(sizeof(int) * n);
    for (int j = 0; j < n; ++j) {
        double s = 0.0;
        for (int64_t i = 0; i < m; ++i) s += A[(int64_t)j * m + i] * A[(int64_t)j * m + i];
        nrm[j] = sqrt(s);
        order[j] = j;
    }
    for (int a = 1; a < n; ++a) {          /* insertion sort: n <= 512 */
        int key = order[a], b = a - 1;
        while (b >= 0 && nrm[order[b]] < nrm[key]) { order[b + 1] = order[b]; --b; }
        order[b + 1] = key;
    }
    int64_t kmin = (T < n) ? T : n;
    for (int64_t j = 0; j < kmin; ++j) sigma[j] = nrm[order[j]];
    for (int j = 0; j < n; ++j)
        for (int i = 0; i < n; ++i) V_out[(int64_t)i * n + j] = V[(int64_t)order[j] * n + i];
    free(nrm); free(order); free(V); free(R); free(W);
    return sweeps;
}

/*
 * Truncated factorisation of one unit (es page 2.A; fr page 2.A: T x H x D is
 * stored as T x R coefficients plus an R x (H D) decompression matrix):
 *   C = X . V_r  (= U_r Sigma_r, T x r),  B = V_r^T  (r x n, orthonormal rows),
 * sigma = all min(T, n) singular values, descending.
 */
int ora_compress_unit(const double *X, int64_t T, int n, int r, double *C, double *B, double *sigma)
{
    double *V = (double *)malloc(sizeof(double) * (size_t)n * n);
    int sweeps = ora_svd(X, T, n, sigma, V);
    for (int i = 0; i < r; ++i)
        for (int c = 0; c < n; ++c) B[(int64_t)i * n + c] = V[(int64_t)c * n + i];
    for (int64_t t = 0; t < T; ++t)
        for (int i = 0; i < r; ++i) {
            double s = 0.0;
            for (int c = 0; c < n; ++c) s += X[t * n + c] * V[(int64_t)c * n + i];
            C[t * r + i] = s;
        }
    free(V);
    return sweeps;
}

/* ------------------------------------------------------------- decode step */

static int mask_bit(const uint32_t *mask, int64_t t) { return (int)((mask[t >> 5] >> (t & 31)) & 1u); }

/*
 * One decode step of one unit (one group of 4 KV heads), written as the
 * pages state it: decompress every cached visual token at its own rank --
 * rank r if its mask bit is set, else the leading r_lo components (fr page
 * 2.B: full rank R_kv for high-score tokens, R_kv/4 for the rest) -- then
 * attend with an ordinary softmax over the visual tokens and the
 * uncompressed text tail.
 *
 *   Khat_t = sum_{i < rho_t} CK[t,i] BK[i,:],   Vhat_t likewise      (rho_t = r or r_lo)
 *   s_{h,t} = scale * q_h . Khat_t[j(h)],       s_{h,T+tau} = scale * q_h . Ktext[tau, j(h)]
 *   p_h = softmax over all T + L logits
 *   o_h = sum_t p_{h,t} Vhat_t[j(h)] + sum_tau p_{h,T+tau} Vtext[tau, j(h)]
 *   mass_t = sum_h p_{h,t}      (visual tokens only: the attention each token received)
 *
 * j(h) = h / (Hg / 4) is the KV head of query head h within the group.
 * Layouts (all row-major): CK, CV: T x r; BK, BV: r x 512; Ktext, Vtext:
 * L x 4 x 128; q, out: Hg x 128; mask: ceil(T/32) words; mass: T (nullable).
 */
void ora_decode_unit(int64_t T, int64_t L, int Hg, int r, int r_lo,
                     const double *CK, const double *BK, const double *CV, const double *BV,
                     const double *Ktext, const double *Vtext, const uint32_t *mask,
                     const double *q, double scale, double *out, double *mass)
{
    int per_kv = Hg / GROUP_HEADS;
    int64_t N = T + L;
    double *Kh = (double *)malloc(sizeof(double) * (size_t)(T * HEAD_DIM + 1));
    double *Vh = (double *)malloc(sizeof(double) * (size_t)(T * HEAD_DIM + 1));
    double *s = (double *)malloc(sizeof(double) * (size_t)(N + 1));
    if (mass) for (int64_t t = 0; t < T; ++t) mass[t] = 0.0;
    for (int j = 0; j < GROUP_HEADS; ++j) {
        /* decompress the j-th head slice of every visual token at its rank */
        for (int64_t t = 0; t < T; ++t) {
            int rho = mask_bit(mask, t) ? r : r_lo;
            for (int d = 0; d < HEAD_DIM; ++d) {
                double kk = 0.0, vv = 0.0;
                for (int i = 0; i < rho; ++i) {
                    kk += CK[t * r + i] * BK[(int64_t)i * FEAT + j * HEAD_DIM + d];
                    vv += CV[t * r + i] * BV[(int64_t)i * FEAT + j * HEAD_DIM + d];
                }
                Kh[t * HEAD_DIM + d] = kk;
                Vh[t * HEAD_DIM + d] = vv;
            }
        }
        for (int hh = 0; hh < per_kv; ++hh) {
            int h = j * per_kv + hh;
            const double *qh = q + (int64_t)h * HEAD_DIM;
            for (int64_t t = 0; t < T; ++t) {
                double a = 0.0;
                for (int d = 0; d < HEAD_DIM; ++d) a += qh[d] * Kh[t * HEAD_DIM + d];
                s[t] = scale * a;
            }
            for (int64_t u = 0; u < L; ++u) {
                const double *kt = Ktext + (u * GROUP_HEADS + j) * HEAD_DIM;
                double a = 0.0;
                for (int d = 0; d < HEAD_DIM; ++d) a += qh[d] * kt[d];
                s[T + u] = scale * a;
            }
            double mx = -INFINITY;
            for (int64_t t = 0; t < N; ++t) if (s[t] > mx) mx = s[t];
            double z = 0.0;
            for (int64_t t = 0; t < N; ++t) { s[t] = exp(s[t] - mx); z += s[t]; }
            for (int64_t t = 0; t < N; ++t) s[t] /= z;
            double *oh = out + (int64_t)h * HEAD_DIM;
            for (int d = 0; d < HEAD_DIM; ++d) {
                double a = 0.0;
                for (int64_t t = 0; t < T; ++t) a += s[t] * Vh[t * HEAD_DIM + d];
                for (int64_t u = 0; u < L; ++u) a += s[T + u] * Vtext[(u * GROUP_HEADS + j) * HEAD_DIM + d];
                oh[d] = a;
            }
            if (mass) for (int64_t t = 0; t < T; ++t) mass[t] += s[t];
        }
    }
    free(Kh); free(Vh); free(s);
}

/* ------------------------------------------------------------- selection */

typedef struct { float key; int64_t idx; } keyed;

/* -0 compares as +0; NaN is below every number. */
static float canon(float x) { return (x == 0.0f) ? 0.0f : x; }

static int keyed_cmp(const void *pa, const void *pb)
{
    const keyed *a = (const keyed *)pa, *b = (const keyed *)pb;
    int an = isnan(a->key), bn = isnan(b->key);
    if (an != bn) return an ? 1 : -1;                 /* NaN last */
    if (!an) {
        if (a->key > b->key) return -1;               /* larger key first */
        if (a->key < b->key) return 1;
    }
    return (a->idx < b->idx) ? -1 : (a->idx > b->idx); /* ties: lower index first */
}

/*
 * Importance update and rank choice for the next step, one unit (fr page
 * 2.B: a moving average, parameter alpha, of the accumulated attention
 * decides which tokens keep the full rank):
 *   key_t = mass_t                                  if alpha == 0
 *   key_t = fma(alpha, score_t, (1 - alpha) * mass_t)   otherwise (fp32, as on the GPU)
 * score (nullable) receives key.  The k tokens with the largest key -- ties
 * to the lower index -- get their mask bit set; every other bit is cleared.
 * Works in fp32 because the comparison decides integers.
 */
void ora_select_unit(int64_t T, const float *mass, float *score, float alpha, int64_t k, uint32_t *mask_out)
{
    keyed *arr = (keyed *)malloc(sizeof(keyed) * (size_t)(T + 1));
    float one_minus = 1.0f - alpha;
    for (int64_t t = 0; t < T; ++t) {
        float key = (alpha == 0.0f) ? mass[t] : fmaf(alpha, score[t], one_minus * mass[t]);
        if (score) score[t] = key;
        arr[t].key = canon(key);
        arr[t].idx = t;
    }
    qsort(arr, (size_t)T, sizeof(keyed), keyed_cmp);
    int64_t words = (T + 31) / 32;
    for (int64_t w = 0; w < words; ++w) mask_out[w] = 0u;
    if (k > T) k = T;
    for (int64_t i = 0; i < k; ++i) mask_out[arr[i].idx >> 5] |= 1u << (arr[i].idx & 31);
    free(arr);
}

/* --------------------------------------------------- many units at once */

/* Units are independent (one group of one sequence of one layer each), so
 * the batched entry points below run one unit per OpenMP thread. */

void ora_decode_units(int64_t n_units, int64_t T, int64_t L, int Hg, int r, int r_lo,
                      const double *CK, const double *BK, const double *CV, const double *BV,
                      const double *Ktext, const double *Vtext, const uint32_t *mask,
                      const double *q, double scale, double *out, double *mass)
{
    int64_t words = (T + 31) / 32;
    #pragma omp parallel for schedule(dynamic, 1)
    for (int64_t u = 0; u < n_units; ++u) {
        ora_decode_unit(T, L, Hg, r, r_lo,
                        CK + u * T * r, BK + u * (int64_t)r * FEAT, CV + u * T * r, BV + u * (int64_t)r * FEAT,
                        Ktext + u * L * FEAT, Vtext + u * L * FEAT, mask + u * words,
                        q + u * (int64_t)Hg * HEAD_DIM, scale, out + u * (int64_t)Hg * HEAD_DIM,
                        mass ? mass + u * T : NULL);
    }
}

void ora_select_units(int64_t n_units, int64_t T, const float *mass, float *score, float alpha,
                      int64_t k, uint32_t *mask_out)
{
    int64_t words = (T + 31) / 32;
    #pragma omp parallel for schedule(dynamic, 1)
    for (int64_t u = 0; u < n_units; ++u)
        ora_select_unit(T, mass + u * T, score ? score + u * T : NULL, alpha, k, mask_out + u * words);
}

int ora_compress_units(int64_t n_units, const double *X, int64_t T, int n, int r, double *C, double *B, double *sigma)
{
    int64_t kmin = (T < n) ? T : n;
    int worst = 0;
    for (int64_t u = 0; u < n_units; ++u) {    /* the QR inside is OpenMP-parallel */
        int s = ora_compress_unit(X + u * T * n, T, n, r, C + u * T * r, B + u * (int64_t)r * n, sigma + u * kmin);
        if (s < 0) worst = -1;
        else if (worst >= 0 && s > worst) worst = s;
    }
    return worst;
}

/* Threads the OpenMP loops above use (reported next to any timing of the oracle). */
int ora_num_threads(void) { return omp_get_max_threads(); }
