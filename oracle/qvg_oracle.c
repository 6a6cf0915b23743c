/*
 * qvg_oracle.c -- plain, slow CPU oracle for the Quant VideoGen (QVG) 2-bit
 * KV-cache codec.
 *
 * TEST INFRASTRUCTURE ONLY.  Only the test suite, the package smoke check and
 * the benchmark's CPU-baseline leg may load this library.  The product path
 * (the CUDA library and its Python binding) never calls it, and this file
 * shares no code, header, table or constant with that path.
 *
 * Sources (web pages about arXiv:2602.02958, "Quant VideoGen: Auto-Regressive
 * Long Video Generation via 2-Bit KV-Cache Quantization"):
 *   [163]  m.163.com article on Quant VideoGen (Chinese), sections
 *          一 (KV memory), 三 (semantic-aware smoothing), 四 (progressive
 *          residual quantization), 五 (system co-design: FP8 E4M3 group
 *          scales, uint8 assignments, centroid cache, fused dequant kernel),
 *          七 (K = 256).
 *   [de]   gist.science/de, "Technische Zusammenfassung" 2A/2B/2C.
 *   [pt]   gist.science/pt, "Resumo tecnico" 2A/2B/2C.
 *
 * Where the pages are silent the plainest reading is taken; every such
 * reading is marked READING below.
 *
 * Arithmetic rules: build with -O2 -ffp-contract=off and no fast-math, so that
 * every multiply and add below is one IEEE operation in the written order.
 * Distances are fp64.  Centroid sums are exact (a wide integer), rounded once
 * to fp64 before the divide.  Residuals and quantisation use fp32 operations,
 * as the data is stored in 16/32-bit floats.
 *
 * Parity status: every function here is pinned by the tests under tests/
 * (format round trips against library casts, closed forms, worked examples,
 * invariants, exact-rational brute force).  The whole-pipeline numbers
 * reported by the pages (error reductions, PSNR) are NOT reproduced: parity
 * unpinned for those, as the pages print no worked codec example.
 */
#include <math.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>
#ifdef _OPENMP
#include <omp.h>
#endif

enum { REF_BF16 = 0, REF_FP32 = 1 };

/* ------------------------------------------------------------------ */
/* Number formats, written from their definitions.                      */
/* ------------------------------------------------------------------ */

/* FP8 E4M3 ("FN" variant: 1 sign, 4 exponent bits with bias 7, 3 mantissa
 * bits, no infinities, S.1111.111 is NaN, largest finite 448, subnormal
 * quantum 2^-9).  The pages store the group scales in this format
 * ([163] 五). */
float ref_e4m3_decode(uint8_t c)
{
    int sign = c >> 7, e = (c >> 3) & 15, m = c & 7;
    double v;
    if (e == 15 && m == 7) return NAN;
    if (e == 0) v = ldexp((double)m, -9);
    else v = ldexp(1.0 + m / 8.0, e - 7);
    return (float)(sign ? -v : v);
}

/* Round to nearest, ties to even; magnitudes at or above 448 saturate to
 * 448 (READING: the pages do not say how scales are rounded; RNE with
 * saturation is the conventional "satfinite" conversion). */
uint8_t ref_e4m3_encode(float xf)
{
    double x = xf, a, q;
    uint8_t s;
    int E, e;
    if (isnan(x)) return 0x7F;
    s = signbit(x) ? 0x80 : 0;
    a = fabs(x);
    if (a >= 448.0) return s | 0x7E;
    if (a < ldexp(1.0, -6)) {              /* subnormal range */
        q = nearbyint(a * 512.0);          /* a / 2^-9, exact scaling */
        return s | (uint8_t)q;             /* q == 8 is the smallest normal */
    }
    frexp(a, &E);                          /* a in [2^(E-1), 2^E) */
    e = E - 1;
    q = nearbyint((ldexp(a, -e) - 1.0) * 8.0);
    if (q == 8.0) { q = 0.0; e += 1; }
    return s | (uint8_t)(((e + 7) << 3) | (int)q);
}

float ref_bf16_decode(uint16_t b)
{
    uint32_t u = (uint32_t)b << 16;
    float f;
    memcpy(&f, &u, 4);
    return f;
}

/* bfloat16 (1 sign, 8 exponent, 7 stored mantissa bits) nearest to x, ties
 * to even, in ONE rounding from the double value (no intermediate fp32). */
uint16_t ref_bf16_round(double x)
{
    uint16_t s;
    double a, v, q;
    int E;
    float f;
    uint32_t u;
    if (isnan(x)) return 0x7FC0;
    s = signbit(x) ? 0x8000 : 0;
    a = fabs(x);
    if (isinf(a)) return s | 0x7F80;
    if (a == 0.0) return s;
    if (a < ldexp(1.0, -126)) {            /* subnormal: quantum 2^-133 */
        v = ldexp(nearbyint(ldexp(a, 133)), -133);
    } else {
        frexp(a, &E);                      /* a in [2^(E-1), 2^E) */
        q = nearbyint(ldexp(a, 8 - E));    /* 8 significant bits */
        v = ldexp(q, E - 8);
    }
    if (v >= ldexp(1.0, 128)) return s | 0x7F80;
    f = (float)v;                          /* exact: v has 8 significant bits */
    memcpy(&u, &f, 4);
    return s | (uint16_t)(u >> 16);
}

/* Round a value to the storage dtype S of the cache (READING: centroids and
 * residuals are kept in the dtype the KV data arrives in). */
static float store_round(double x, int dtype)
{
    if (dtype == REF_FP32) return (float)x;
    return ref_bf16_decode(ref_bf16_round(x));
}

static void load_values(const void* src, int dtype, int64_t n, float* dst)
{
    int64_t i;
    if (dtype == REF_FP32) {
        memcpy(dst, src, (size_t)n * sizeof(float));
    } else {
        const uint16_t* b = (const uint16_t*)src;
        for (i = 0; i < n; ++i) dst[i] = ref_bf16_decode(b[i]);
    }
}

static void store_values(const float* src, int dtype, int64_t n, void* dst)
{
    int64_t i;
    if (dtype == REF_FP32) {
        memcpy(dst, src, (size_t)n * sizeof(float));
    } else {
        uint16_t* b = (uint16_t*)dst;
        for (i = 0; i < n; ++i) b[i] = ref_bf16_round((double)src[i]);
    }
}

/* Batch helpers so the tests can sweep whole code spaces. */
void ref_e4m3_encode_array(const float* x, uint8_t* out, int64_t n)
{
    int64_t i;
    for (i = 0; i < n; ++i) out[i] = ref_e4m3_encode(x[i]);
}

void ref_e4m3_decode_array(const uint8_t* c, float* out, int64_t n)
{
    int64_t i;
    for (i = 0; i < n; ++i) out[i] = ref_e4m3_decode(c[i]);
}

void ref_bf16_round_array(const double* x, uint16_t* out, int64_t n)
{
    int64_t i;
    for (i = 0; i < n; ++i) out[i] = ref_bf16_round(x[i]);
}

/* ------------------------------------------------------------------ */
/* Threads (the assignment loop is parallel over tokens; every token's   */
/* arithmetic is the same whatever the thread count).                    */
/* ------------------------------------------------------------------ */
void ref_set_threads(int n)
{
#ifdef _OPENMP
    if (n > 0) omp_set_num_threads(n);
#else
    (void)n;
#endif
}

int ref_get_threads(void)
{
#ifdef _OPENMP
    return omp_get_max_threads();
#else
    return 1;
#endif
}

/* ------------------------------------------------------------------ */
/* k-means on one block (semantic-aware smoothing, [163] 三; [de] 2A;    */
/* [pt] 2A): tokens are grouped by k-means on their latent vectors and   */
/* each group's centroid is the mean of its members.                     */
/* ------------------------------------------------------------------ */

/* Squared Euclidean distance in fp64, channels in ascending order, one
 * subtract, one multiply and one add per channel (READING: the pages do not
 * name the metric; squared L2 is the plain k-means reading). */
double ref_sqdist(const float* r, const float* c, int d)
{
    double D = 0.0;
    int j;
    for (j = 0; j < d; ++j) {
        double diff = (double)r[j] - (double)c[j];
        double sq = diff * diff;
        D = D + sq;
    }
    return D;
}

/* Assignment step: pi_i = argmin_k D(r_i, c_k); an exact tie goes to the
 * lowest k (READING). */
void ref_assign(const float* R, int64_t N, int d, const float* C, int K,
                uint8_t* pi)
{
    int64_t i;
#pragma omp parallel for schedule(static)
    for (i = 0; i < N; ++i) {
        double best = INFINITY;
        int bk = 0, k;
        for (k = 0; k < K; ++k) {
            double D = ref_sqdist(R + i * d, C + (int64_t)k * d, d);
            if (D < best) { best = D; bk = k; }
        }
        pi[i] = (uint8_t)bk;
    }
}

/* k-means objective J = sum_i D(r_i, c_pi_i), fp64, tokens ascending. */
double ref_objective(const float* R, int64_t N, int d, const float* C,
                     const uint8_t* pi)
{
    double J = 0.0;
    int64_t i;
    for (i = 0; i < N; ++i) J = J + ref_sqdist(R + i * d, C + (int64_t)pi[i] * d, d);
    return J;
}

/* Exact sum of fp32 values.  Every fp32 value is an integer multiple of
 * 2^-149 (the smallest subnormal), and |v| < 2^128, so v * 2^149 is an
 * integer below 2^277; a sum of fewer than 2^40 of them fits a signed 320-bit
 * two's-complement integer (five 64-bit words, least significant first). */
typedef struct { uint64_t w[5]; } exact_sum;

static void exact_add(exact_sum* a, float v)
{
    int sh, k, ex;
    uint64_t mag, lo, hi, carry;
    int neg;
    uint32_t bits;
    if (v == 0.0f) return;
    memcpy(&bits, &v, sizeof(bits));     /* IEEE binary32: sign, 8-bit exponent, 23-bit fraction */
    neg = (int)(bits >> 31);
    ex = (int)((bits >> 23) & 0xFF);
    mag = bits & 0x7FFFFFu;
    if (ex == 0) {
        sh = 0;                          /* subnormal: v = fraction * 2^-149 */
    } else {
        mag |= 0x800000u;                /* normal: v = (2^23 + fraction) * 2^(ex - 150) */
        sh = ex - 1;                     /* v * 2^149 = mag * 2^sh */
    }
    /* the shifted magnitude as a 128-bit pair at word sh/64 */
    k = sh / 64;
    lo = mag << (sh % 64);
    hi = (sh % 64) ? mag >> (64 - sh % 64) : 0;
    if (!neg) {
        uint64_t t = a->w[k] + lo;
        carry = t < lo;
        a->w[k] = t;
        if (k + 1 < 5) {
            uint64_t t2 = a->w[k + 1] + hi;
            uint64_t c2 = t2 < hi;
            t2 += carry;
            c2 += t2 < carry;
            a->w[k + 1] = t2;
            carry = c2;
            for (k += 2; k < 5 && carry; ++k) { a->w[k] += 1; carry = a->w[k] == 0; }
        }
    } else {
        uint64_t borrow = a->w[k] < lo;
        a->w[k] -= lo;
        if (k + 1 < 5) {
            uint64_t b2 = a->w[k + 1] < hi;
            a->w[k + 1] -= hi;
            b2 += a->w[k + 1] < borrow;
            a->w[k + 1] -= borrow;
            borrow = b2;
            for (k += 2; k < 5 && borrow; ++k) { borrow = a->w[k] == 0; a->w[k] -= 1; }
        }
    }
}

/* The exact sum rounded once to the nearest double (ties to even). */
static double exact_to_double(const exact_sum* a)
{
    uint64_t w[5];
    int i, neg = (a->w[4] >> 63) != 0, top = -1;
    uint64_t sig = 0, rest_nonzero = 0, half;
    double r;
    for (i = 0; i < 5; ++i) w[i] = a->w[i];
    if (neg) {                           /* two's complement negate */
        uint64_t carry = 1;
        for (i = 0; i < 5; ++i) { w[i] = ~w[i] + carry; carry = carry && w[i] == 0; }
    }
    for (i = 4; i >= 0; --i)             /* the highest set bit */
        if (w[i]) { top = 64 * i + 63 - __builtin_clzll(w[i]); break; }
    if (top < 0) return 0.0;
    if (top <= 52) {                     /* fits 53 bits: exact */
        sig = w[0];
        r = ldexp((double)sig, -149);
        return neg ? -r : r;
    }
    /* bits top-52 .. top form the significand; the bits below round it */
    for (i = 0; i < 53; ++i) {
        const int b = top - 52 + i;
        sig |= ((w[b / 64] >> (b % 64)) & 1) << i;
    }
    half = (w[(top - 53) / 64] >> ((top - 53) % 64)) & 1;
    {                                    /* any set bit below bit top - 53 */
        const int b = top - 53, wb = b / 64, ob = b % 64;
        for (i = 0; i < wb; ++i) rest_nonzero |= w[i] != 0;
        if (ob) rest_nonzero |= (w[wb] & ((1ull << ob) - 1ull)) != 0;
    }
    if (half && (rest_nonzero || (sig & 1))) sig += 1;   /* may carry to 2^53: still exact in a double */
    r = ldexp((double)sig, top - 52 - 149);
    return neg ? -r : r;
}

/* Update step ([163] 三: each group's centroid is the mean of its tokens):
 * c_k = round_S( RN64( RN64(sum_{pi_i = k} r_i) / n_k ) ), where the sum is
 * formed exactly and rounded once to fp64, then one fp64 divide and one
 * rounding to S (READING: the plain mean, with one rounding per step).  A
 * cluster with no members keeps its previous centroid (READING). */
void ref_update(const float* R, int64_t N, int d, const uint8_t* pi, int K,
                int dtype, float* C)
{
    exact_sum* sums = (exact_sum*)calloc((size_t)K * d, sizeof(exact_sum));
    int64_t* cnt = (int64_t*)calloc((size_t)K, sizeof(int64_t));
    int64_t i;
    int k, j;
    for (i = 0; i < N; ++i) cnt[pi[i]] += 1;
    /* Channels are independent and exact sums do not depend on the order of
     * the adds, so the channels may be summed by different threads. */
#pragma omp parallel for schedule(static) private(i)
    for (j = 0; j < d; ++j)
        for (i = 0; i < N; ++i) exact_add(&sums[(int64_t)pi[i] * d + j], R[i * d + j]);
    for (k = 0; k < K; ++k) {
        if (cnt[k] == 0) continue;
        for (j = 0; j < d; ++j)
            C[(int64_t)k * d + j] = store_round(exact_to_double(&sums[(int64_t)k * d + j]) / (double)cnt[k], dtype);
    }
    free(sums);
    free(cnt);
}

/* The exact sum of n fp32 values, rounded once to fp64 (exposed for the
 * tests that pin the update). */
double ref_exact_sum(const float* x, int64_t n)
{
    exact_sum a;
    int64_t i;
    memset(&a, 0, sizeof(a));
    for (i = 0; i < n; ++i) exact_add(&a, x[i]);
    return exact_to_double(&a);
}

/* Lloyd's iteration run exactly `iters` times, each an assignment followed by
 * an update, with no early stop (READING).  C holds the initial centroids on
 * entry and the final ones on exit; pi is the assignment of the last
 * iteration, so every stored centroid is the (rounded) mean of exactly the
 * tokens that point to it.  trace, if given, receives 2*iters objective
 * values: after each assignment and after each update. */
void ref_kmeans(const float* R, int64_t N, int d, int K, int iters, int dtype,
                float* C, uint8_t* pi, double* trace)
{
    int it;
    for (it = 0; it < iters; ++it) {
        ref_assign(R, N, d, C, K, pi);
        if (trace) trace[2 * it] = ref_objective(R, N, d, C, pi);
        ref_update(R, N, d, pi, K, dtype, C);
        if (trace) trace[2 * it + 1] = ref_objective(R, N, d, C, pi);
    }
}

/* Residual after a stage ([163] 三: subtract the group centroid):
 * R_out = round_S(R_in - C[pi]) with the subtraction in fp32. */
void ref_residual(const float* R, int64_t N, int d, const float* C,
                  const uint8_t* pi, int dtype, float* out)
{
    int64_t i;
    int j;
    for (i = 0; i < N; ++i)
        for (j = 0; j < d; ++j) {
            float diff = R[i * d + j] - C[(int64_t)pi[i] * d + j];
            out[i * d + j] = store_round((double)diff, dtype);
        }
}

/* ------------------------------------------------------------------ */
/* 2-bit group quantisation of the final residual ([163] 五, 六: INT2     */
/* values with FP8 E4M3 group scales).                                   */
/* READINGS: a group is G contiguous channels of one token; asymmetric   */
/* min/max quantisation with the zero point (the group minimum) stored   */
/* as a second E4M3 byte; codes q in {0..3} are packed four to a byte,   */
/* channel j at bits 2*(j mod 4).                                        */
/* ------------------------------------------------------------------ */
void ref_group_quant(const float* R, int64_t N, int d, int G,
                     uint8_t* codes, uint8_t* scale, uint8_t* zero)
{
    int64_t i;
    int g, j, ng = d / G;
    memset(codes, 0, (size_t)(N * (d / 4)));
    for (i = 0; i < N; ++i) {
        for (g = 0; g < ng; ++g) {
            const float* r = R + i * d + (int64_t)g * G;
            float lo = r[0], hi = r[0], m, s, span, sraw;
            uint8_t zc, sc;
            for (j = 1; j < G; ++j) {
                if (r[j] < lo) lo = r[j];
                if (r[j] > hi) hi = r[j];
            }
            /* READING: a minimum or maximum of -0 is taken as +0 (adding +0
             * maps -0 to +0 and leaves every other value unchanged), so the
             * stored bytes never depend on which of two equal zeros is met
             * first. */
            lo = lo + 0.0f;
            hi = hi + 0.0f;
            zc = ref_e4m3_encode(lo);
            m = ref_e4m3_decode(zc);
            span = hi - m;
            sraw = span / 3.0f;
            sc = ref_e4m3_encode(sraw);
            s = ref_e4m3_decode(sc);
            zero[i * ng + g] = zc;
            scale[i * ng + g] = sc;
            for (j = 0; j < G; ++j) {
                int ch = g * G + j, q = 0;
                if (s != 0.0f) {
                    float t = (r[j] - m) / s;
                    float rt = rintf(t);
                    if (rt < 0.0f) rt = 0.0f;
                    if (rt > 3.0f) rt = 3.0f;
                    q = (int)rt;
                }
                codes[i * (d / 4) + ch / 4] |= (uint8_t)(q << (2 * (ch % 4)));
            }
        }
    }
}

/* Symmetric variant: ONE FP8 E4M3 scale per group ([163] 五 names only
 * "FP8 E4M3 group scales"; with one byte per group the closed form gives the
 * 6.94-7.05x of [163] 六 at T = 1, G = 64, and the 6.40x of plain rounding at
 * G = 16, see ref_bits_per_element).  READING: standard symmetric signed
 * INT2, the scale being the group's largest magnitude over the largest
 * positive code (2^(b-1) - 1 = 1):
 *   s = E4M3(max |r|),  q = clamp(rint(r / s), -2, 1),  stored u = q + 2,
 * with an IEEE fp32 divide, ties to even, and q = 0 when s = 0.  The value
 * of u is s * (u - 2).  Codes are packed as in ref_group_quant. */
void ref_group_quant_sym(const float* R, int64_t N, int d, int G,
                         uint8_t* codes, uint8_t* scale)
{
    int64_t i;
    int g, j, ng = d / G;
    memset(codes, 0, (size_t)(N * (d / 4)));
    for (i = 0; i < N; ++i) {
        for (g = 0; g < ng; ++g) {
            const float* r = R + i * d + (int64_t)g * G;
            float amax = 0.0f, s;
            uint8_t sc;
            for (j = 0; j < G; ++j) {
                float a = fabsf(r[j]);
                if (a > amax) amax = a;
            }
            sc = ref_e4m3_encode(amax);
            s = ref_e4m3_decode(sc);
            scale[i * ng + g] = sc;
            for (j = 0; j < G; ++j) {
                int ch = g * G + j, q = 0;
                if (s != 0.0f) {
                    float t = r[j] / s;
                    float rt = rintf(t);
                    if (rt < -2.0f) rt = -2.0f;
                    if (rt > 1.0f) rt = 1.0f;
                    q = (int)rt;
                }
                codes[i * (d / 4) + ch / 4] |= (uint8_t)((q + 2) << (2 * (ch % 4)));
            }
        }
    }
}

/* ------------------------------------------------------------------ */
/* Whole codec.  Layouts (all row-major):                                */
/*   X          [H][N][d]   in S (bf16 bits or fp32)                      */
/*   init       [T][H][K][d] in S, or NULL for the cold start              */
/*   codes      [H][N][d/4]                                               */
/*   scale,zero [H][N][d/G] E4M3 bytes (zero unused, may be NULL, in the */
/*              symmetric mode: scale_mode = 1)                           */
/*   assign     [T][H][N]   uint8                                         */
/*   centroids  [T][H][K][d] in S                                         */
/* Progressive residual quantisation ([163] 四; [de] 2B; [pt] 2B):       */
/* R(0) = X; stage t runs semantic-aware smoothing on R(t-1) and gives    */
/* C(t), pi(t), R(t); only R(T) is quantised to 2 bits (READING: the      */
/* stages carry centroids and assignments, the low-bit step is on the     */
/* final residual, as [163] 四 describes it).  T = 0 is plain per-group   */
/* round-to-nearest on X (the RTN baseline of [163] 六).                  */
/* Cold start takes the first K tokens of the stage input as the initial  */
/* centroids (READING).                                                   */
/* Returns 0 on success, -1 on invalid arguments.                          */
/* ------------------------------------------------------------------ */
int ref_quantize_ex(int K, int T, int G, int iters, int warm_iters, int warm_stages, int dtype,
                    int scale_mode, const void* X, int64_t N, int H, int d, const void* init,
                    uint8_t* codes, uint8_t* scale, uint8_t* zero, uint8_t* assign, void* centroids);

int ref_quantize(int K, int T, int G, int iters, int dtype, int scale_mode,
                 const void* X, int64_t N, int H, int d, const void* init,
                 uint8_t* codes, uint8_t* scale, uint8_t* zero,
                 uint8_t* assign, void* centroids)
{
    /* every stage warm-started from init when it is given, cold otherwise */
    return ref_quantize_ex(K, T, G, iters, iters, init ? T : 0, dtype, scale_mode, X, N, H, d, init,
                           codes, scale, zero, assign, centroids);
}

/* The codec with the first warm_stages stages started from init[t] (the
 * previous chunk's tables, [163] 五) and run for warm_iters Lloyd
 * iterations, the other stages started cold from the first K tokens of their
 * input and run for iters. */
int ref_quantize_ex(int K, int T, int G, int iters, int warm_iters, int warm_stages, int dtype,
                    int scale_mode, const void* X, int64_t N, int H, int d, const void* init,
                    uint8_t* codes, uint8_t* scale, uint8_t* zero, uint8_t* assign, void* centroids)
{
    int64_t esz = dtype == REF_FP32 ? 4 : 2;
    int h, t;
    float *R, *R2, *C;
    if (K < 1 || K > 256 || T < 0 || G < 4 || G % 4 || d % G || d % 4 || N < 1 || H < 1 || iters < 0)
        return -1;
    if (scale_mode != 0 && scale_mode != 1) return -1;
    if (warm_stages < 0 || warm_stages > T || (warm_stages > 0 && init == NULL)) return -1;
    if (T > warm_stages && iters < 1) return -1;   /* assignments need one assign step */
    if (warm_stages > 0 && warm_iters < 1) return -1;
    if (T > warm_stages && N < K) return -1;
    R = (float*)malloc((size_t)(N * d) * sizeof(float));
    R2 = (float*)malloc((size_t)(N * d) * sizeof(float));
    C = (float*)malloc((size_t)K * d * sizeof(float));
    for (h = 0; h < H; ++h) {
        load_values((const char*)X + (int64_t)h * N * d * esz, dtype, N * d, R);
        for (t = 0; t < T; ++t) {
            int64_t tab = ((int64_t)t * H + h) * K * d;
            uint8_t* pi = assign + ((int64_t)t * H + h) * N;
            float* tmp;
            if (t < warm_stages) load_values((const char*)init + tab * esz, dtype, (int64_t)K * d, C);
            else memcpy(C, R, (size_t)K * d * sizeof(float));
            ref_kmeans(R, N, d, K, t < warm_stages ? warm_iters : iters, dtype, C, pi, NULL);
            store_values(C, dtype, (int64_t)K * d, (char*)centroids + tab * esz);
            ref_residual(R, N, d, C, pi, dtype, R2);
            tmp = R; R = R2; R2 = tmp;
        }
        if (scale_mode == 1)
            ref_group_quant_sym(R, N, d, G, codes + (int64_t)h * N * (d / 4),
                                scale + (int64_t)h * N * (d / G));
        else
            ref_group_quant(R, N, d, G, codes + (int64_t)h * N * (d / 4),
                            scale + (int64_t)h * N * (d / G), zero + (int64_t)h * N * (d / G));
    }
    free(R);
    free(R2);
    free(C);
    return 0;
}

/* Reconstruction in reverse order ([163] 四, 五; [de] 2B "Rekonstruktion"):
 * y = s*q + m (symmetric mode: y = s*(u - 2)), then the centroid of stage
 * T, T-1, ..., 1 is added, each an fp32 add, and the sum is rounded once to
 * S.  The first value is exact in fp32: s and m are E4M3 values (4
 * significant bits, bits between 2^-9 and 2^8) and q <= 3, so it spans fewer
 * than 24 bits. */
int ref_dequantize(int K, int T, int G, int dtype, int scale_mode, const uint8_t* codes,
                   const uint8_t* scale, const uint8_t* zero,
                   const uint8_t* assign, const void* centroids,
                   int64_t N, int H, int d, void* Y)
{
    int64_t esz = dtype == REF_FP32 ? 4 : 2, i;
    int h, j, t, ng;
    float* C;
    float* row;
    if (K < 1 || K > 256 || T < 0 || G < 4 || G % 4 || d % G || d % 4 || N < 0 || H < 1) return -1;
    if (scale_mode != 0 && scale_mode != 1) return -1;
    ng = d / G;
    C = (float*)malloc((size_t)(T > 0 ? T : 1) * K * d * sizeof(float));
    row = (float*)malloc((size_t)d * sizeof(float));
    for (h = 0; h < H; ++h) {
        for (t = 0; t < T; ++t)
            load_values((const char*)centroids + ((int64_t)t * H + h) * K * d * esz, dtype,
                        (int64_t)K * d, C + (int64_t)t * K * d);
        for (i = 0; i < N; ++i) {
            int64_t tok = (int64_t)h * N + i;
            for (j = 0; j < d; ++j) {
                int q = (codes[tok * (d / 4) + j / 4] >> (2 * (j % 4))) & 3;
                float s = ref_e4m3_decode(scale[tok * ng + j / G]);
                float y;
                if (scale_mode == 1) {
                    y = (float)((double)s * (double)(q - 2));
                } else {
                    float m = ref_e4m3_decode(zero[tok * ng + j / G]);
                    y = (float)((double)s * (double)q + (double)m);
                }
                for (t = T - 1; t >= 0; --t) {
                    int k = assign[((int64_t)t * H + h) * N + i];
                    y = y + C[((int64_t)t * K + k) * d + j];
                }
                row[j] = y;
            }
            store_values(row, dtype, d, (char*)Y + tok * d * esz);
        }
    }
    free(C);
    free(row);
    return 0;
}

/* ------------------------------------------------------------------ */
/* Closed forms.                                                         */
/* ------------------------------------------------------------------ */

/* KV-cache bytes for a model with L layers and hidden size `hidden`
 * storing `tokens` latent tokens (H x W x T_frames): 2 (K and V) x L x
 * tokens x hidden x bytes per value ([163] 一). */
double ref_kv_cache_bytes(int64_t L, int64_t tokens, int64_t hidden, int64_t bytes)
{
    return 2.0 * (double)L * (double)tokens * (double)hidden * (double)bytes;
}

/* Bits per cached element of the codec: b code bits, two E4M3 bytes per
 * group of G (one in the symmetric mode), one uint8 assignment per token per
 * stage (8T/d per element), and T centroid tables of K x d values in S
 * amortised over the N tokens of a block. */
double ref_bits_per_element(int K, int T, int G, int bits, int64_t N, int d, int dtype, int scale_mode)
{
    double sc = dtype == REF_FP32 ? 32.0 : 16.0;
    double per_group = scale_mode == 1 ? 8.0 : 16.0;
    return (double)bits + per_group / G + 8.0 * T / d + sc * T * K / (double)N;
}

/* Bytes of the packed stream for H blocks of N tokens, summed array by
 * array over the layouts above. */
int64_t ref_packed_bytes(int K, int T, int G, int bits, int64_t N, int H, int d, int dtype, int scale_mode)
{
    int64_t esz = dtype == REF_FP32 ? 4 : 2;
    int64_t codes = (int64_t)H * N * d * bits / 8;
    int64_t scales = (scale_mode == 1 ? 1 : 2) * (int64_t)H * N * (d / G);
    int64_t assign = (int64_t)T * H * N;
    int64_t cents = (int64_t)T * H * K * d * esz;
    return codes + scales + assign + cents;
}

/* ------------------------------------------------------------------ */
/* Attention over the reconstructed cache ([163] 五: keys are cached     */
/* before the rotary position embedding, which is applied after         */
/* dequantisation; the fused kernel feeds the reconstruction to          */
/* attention without writing it out; [de] 2C "Fused Kernel").            */
/* READINGS (the pages give no formula for either step):                */
/*   rotary embedding in the RoFormer form: channel pair (2i, 2i+1) of a  */
/*   token at position p is rotated by the angle p * base^(-2i/d);       */
/*   softmax attention with scale 1/sqrt(d) and no mask: every query     */
/*   sees every cached token.                                            */
/* Everything in fp64, exact positions; cos and sin from libm.          */
/* ------------------------------------------------------------------ */

/* out[n][d] = rotary embedding of x[n][d] (token i at position pos[i]). */
void ref_rope(const float* x, int64_t n, int d, const int64_t* pos, double base, double* out)
{
    int64_t t;
    int i;
    for (t = 0; t < n; ++t) {
        for (i = 0; i < d / 2; ++i) {
            const double theta = pow(base, -2.0 * i / (double)d);
            const double a = (double)pos[t] * theta;
            const double c = cos(a), s = sin(a);
            const double x0 = x[t * d + 2 * i], x1 = x[t * d + 2 * i + 1];
            out[t * d + 2 * i] = x0 * c - x1 * s;
            out[t * d + 2 * i + 1] = x0 * s + x1 * c;
        }
    }
}

/* O[nq][d] = softmax(rope(Q) rope(K)^T / sqrt(d)) V for one head, with Q at
 * positions qpos and the cached keys at positions 0 .. nk-1 (cache order).
 * K and V are the reconstructed cache (the dequantised values).  Returns 0,
 * or -1 for invalid sizes. */
int ref_attention(const float* Q, const int64_t* qpos, int64_t nq, const float* K, const float* V,
                  int64_t nk, int d, double base, double* O)
{
    double *qr, *kr, *s;
    int64_t* kpos;
    int64_t i, j;
    int c;
    if (nq < 1 || nk < 1 || d < 2 || d % 2) return -1;
    qr = (double*)malloc((size_t)(nq * d) * sizeof(double));
    kr = (double*)malloc((size_t)(nk * d) * sizeof(double));
    kpos = (int64_t*)malloc((size_t)nk * sizeof(int64_t));
    for (j = 0; j < nk; ++j) kpos[j] = j;
    ref_rope(Q, nq, d, qpos, base, qr);
    ref_rope(K, nk, d, kpos, base, kr);
#pragma omp parallel for schedule(static) private(j, c, s)
    for (i = 0; i < nq; ++i) {
        double m = -INFINITY, l = 0.0;
        s = (double*)malloc((size_t)nk * sizeof(double));
        for (j = 0; j < nk; ++j) {
            double dot = 0.0;
            for (c = 0; c < d; ++c) dot += qr[i * d + c] * kr[j * d + c];
            s[j] = dot / sqrt((double)d);
            if (s[j] > m) m = s[j];
        }
        for (c = 0; c < d; ++c) O[i * d + c] = 0.0;
        for (j = 0; j < nk; ++j) {
            const double p = exp(s[j] - m);
            l += p;
            for (c = 0; c < d; ++c) O[i * d + c] += p * (double)V[j * d + c];
        }
        for (c = 0; c < d; ++c) O[i * d + c] /= l;
        free(s);
    }
    free(qr);
    free(kr);
    free(kpos);
    return 0;
}

/* ------------------------------------------------------------------ */
/* Adaptive per-chunk settings on the streaming path ([163] 九: adapt the */
/* compression parameters to the content; [163] 五: the streaming        */
/* centroid cache).  The pages give no rule; READINGS:                    */
/*   statistic of a chunk: over every block, token and group of           */
/*     probe_group channels, the sum of the E4M3 codes of the group's     */
/*     range fl32(max - min) (the code grows with the range, about eight  */
/*     codes per binade);                                                  */
/*   level: the number of ascending thresholds theta_j (in sixteenths of */
/*     a code) with 16 * S > theta_j * (number of groups), so a chunk of  */
/*     wider ranges takes a later, more expensive setting of the ladder;  */
/*   centroid reuse: chunk c > 0 starts stage t from chunk c-1's C(t) for */
/*     t < min(T of c-1, T of c), every other stage cold (first K tokens);*/
/*     every refresh_every-th chunk (when > 0) starts all stages cold.     */
/* ------------------------------------------------------------------ */
uint64_t ref_range_stat(const void* X, int dtype, int64_t N, int H, int d, int G)
{
    int64_t esz = dtype == REF_FP32 ? 4 : 2, i;
    uint64_t S = 0;
    int h, g, j;
    float* row = (float*)malloc((size_t)d * sizeof(float));
    for (h = 0; h < H; ++h)
        for (i = 0; i < N; ++i) {
            load_values((const char*)X + ((int64_t)h * N + i) * d * esz, dtype, d, row);
            for (g = 0; g < d / G; ++g) {
                float lo = row[g * G], hi = row[g * G];
                for (j = 1; j < G; ++j) {
                    if (row[g * G + j] < lo) lo = row[g * G + j];
                    if (row[g * G + j] > hi) hi = row[g * G + j];
                }
                S += ref_e4m3_encode(hi - lo);
            }
        }
    free(row);
    return S;
}

/* Level of a chunk from its statistic: the count of thresholds it exceeds. */
int ref_adaptive_level(uint64_t S, int64_t n_groups, const int* thresholds, int levels)
{
    int lvl = 0, j;
    for (j = 0; j + 1 < levels; ++j)
        if ((double)S * 16.0 > (double)thresholds[j] * (double)n_groups) lvl = j + 1;
    return lvl;
}

/* Stages of chunk `chunk` (with T_cur stages) started from the previous
 * chunk's tables (which had T_prev stages). */
int ref_adaptive_warm_stages(int chunk, int T_prev, int T_cur, int refresh_every)
{
    if (chunk == 0) return 0;
    if (refresh_every > 0 && chunk % refresh_every == 0) return 0;
    return T_prev < T_cur ? T_prev : T_cur;
}
