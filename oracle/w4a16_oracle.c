/*
 * CPU oracle for the W4A16 group-quantised linear layer.  TEST INFRASTRUCTURE
 * ONLY: tests, the smoke check and the benchmark's CPU-baseline leg use it to
 * judge the CUDA library; no product code path calls it.
 *
 * What it computes (plain definition, no blocking, fusion or reordering):
 *
 *   "PerfXLLM on Snapdragon 8 Gen2", section 3.1 (low-precision quantisation):
 *   weights only are quantised, to int4, with group_size 128 and a scale and a
 *   zero parameter per group.  Reading taken: for row m and group g the
 *   weight is  w[m,k] = fp16_RN( (q[m,k] - z[m,g]) * s[m,g] ),  k in group g,
 *   with q and z unsigned 4-bit integers and s an fp16 scale.
 *
 *   Same page, section 3.3 item 1 (GEMM definition): A[m,k] . B[k,n] = C[m,n]
 *   with A the weights and n the number of tokens; item 2: GEMV is the n = 1
 *   case.  Storage order taken: activations token-major x[n][k], output
 *   token-major y[n][m].  Every sum runs in fp64 in ascending k, so the result
 *   does not depend on the number of OpenMP threads (rows are split, never k).
 *
 * fp16 handling is written here from the IEEE 754 binary16 definition
 * (1 sign, 5 exponent bits with bias 15, 10 fraction bits, subnormals,
 * round-to-nearest-even, overflow to infinity).  No CUDA or compiler half
 * type is used.
 */
#include <math.h>
#include <stdint.h>
#include <stddef.h>
#include <stdlib.h>
#ifdef _OPENMP
#include <omp.h>
#endif

/* ---------------------------------------------------------------- fp16 ---- */

double w4o_fp16_to_double(uint16_t h)
{
    int sign = (h >> 15) & 1;
    int e = (h >> 10) & 0x1f;
    int f = h & 0x3ff;
    double v;
    if (e == 0) {
        v = ldexp((double)f, -24);                 /* subnormal: f * 2^-24 */
    } else if (e == 31) {
        v = f ? NAN : INFINITY;
    } else {
        v = ldexp((double)(1024 + f), e - 25);     /* (1 + f/1024) * 2^(e-15) */
    }
    return sign ? -v : v;
}

/* Round a non-negative double that is below 2^53 to the nearest integer,
 * ties to even.  All steps are exact in double precision. */
static double round_half_even(double v)
{
    double fl = floor(v);
    double r = v - fl;
    if (r > 0.5) return fl + 1.0;
    if (r < 0.5) return fl;
    return (fmod(fl, 2.0) == 0.0) ? fl : fl + 1.0;
}

uint16_t w4o_fp16_from_double(double x)
{
    if (isnan(x)) return 0x7e00;
    uint16_t sign = signbit(x) ? 0x8000 : 0;
    double a = fabs(x);
    if (isinf(a)) return sign | 0x7c00;
    if (a < ldexp(1.0, -14)) {
        /* subnormal range: quantum 2^-24; n == 1024 encodes the smallest
         * normal number, which the bit pattern below yields directly */
        double n = round_half_even(ldexp(a, 24));
        return sign | (uint16_t)n;
    }
    int e2;
    frexp(a, &e2);                 /* a = f * 2^e2, f in [0.5, 1) */
    int E = e2 - 1;                /* a in [2^E, 2^(E+1)) */
    double n = round_half_even(ldexp(a, 10 - E));   /* in [1024, 2048] */
    if (n == 2048.0) { n = 1024.0; E += 1; }
    if (E + 15 >= 31) return sign | 0x7c00;         /* overflow -> inf */
    return sign | (uint16_t)(((E + 15) << 10) | ((int)n - 1024));
}

void w4o_fp16_from_double_array(const double* x, uint16_t* out, int64_t n)
{
    for (int64_t i = 0; i < n; ++i) out[i] = w4o_fp16_from_double(x[i]);
}

void w4o_fp16_to_double_array(const uint16_t* h, double* out, int64_t n)
{
    for (int64_t i = 0; i < n; ++i) out[i] = w4o_fp16_to_double(h[i]);
}

/* ------------------------------------------------------------- threads ---- */

void w4o_set_threads(int n)
{
#ifdef _OPENMP
    if (n > 0) omp_set_num_threads(n);
#else
    (void)n;
#endif
}

int w4o_get_threads(void)
{
#ifdef _OPENMP
    return omp_get_max_threads();
#else
    return 1;
#endif
}

/* ------------------------------------------------------------- dequant ---- */

static int check_shape(int64_t M, int64_t K, int64_t G)
{
    if (M <= 0 || K <= 0 || G <= 0) return 1;
    if (K % G) return 2;
    return 0;
}

/* One weight: w = fp16_RN((q - z) * s).  The product of an integer in
 * [-15, 15] and an fp16 value has at most 16 significant bits, so the double
 * product is exact and the fp16 rounding is the only rounding. */
static uint16_t dequant_one(uint8_t q, uint8_t z, uint16_t s)
{
    int d = (int)q - (int)z;
    return w4o_fp16_from_double((double)d * w4o_fp16_to_double(s));
}

/* W[m][k] (fp16 bits) for the whole M x K weight. */
int w4o_dequant(const uint8_t* q, const uint8_t* zeros, const uint16_t* scales,
                int64_t M, int64_t K, int64_t G, uint16_t* W)
{
    int rc = check_shape(M, K, G);
    if (rc) return rc;
    int64_t kg = K / G;
    #pragma omp parallel for schedule(static)
    for (int64_t m = 0; m < M; ++m) {
        for (int64_t k = 0; k < K; ++k) {
            int64_t g = k / G;
            W[m * K + k] = dequant_one(q[m * K + k], zeros[m * kg + g],
                                       scales[m * kg + g]);
        }
    }
    return 0;
}

/* -------------------------------------------------------------- product ---- */

/* y[n][j] = sum_k w[rows[j], k] * x[n][k] in fp64, ascending k.
 * rows == NULL means every row, j == m.  y has N x ny entries. */
static int gemm_rows(const uint8_t* q, const uint8_t* zeros, const uint16_t* scales,
                     const uint16_t* x, int64_t M, int64_t K, int64_t N, int64_t G,
                     const int64_t* rows, int64_t ny, double* y)
{
    int rc = check_shape(M, K, G);
    if (rc) return rc;
    if (N < 0) return 1;
    int64_t kg = K / G;
    for (int64_t j = 0; rows && j < ny; ++j)
        if (rows[j] < 0 || rows[j] >= M) return 1;

    /* x widened once to fp64 (exact), shared by every thread */
    double* xd = (double*)malloc((size_t)(N * K > 0 ? N * K : 1) * sizeof(double));
    if (!xd) return 3;
    for (int64_t i = 0; i < N * K; ++i) xd[i] = w4o_fp16_to_double(x[i]);
    int failed = 0;

    #pragma omp parallel
    {
        /* per-thread row of the dequantised weight, in fp64 (exact) */
        double* wrow = (double*)malloc((size_t)K * sizeof(double));
        if (!wrow) {
            #pragma omp atomic write
            failed = 1;
        }
        #pragma omp for schedule(static)
        for (int64_t j = 0; j < ny; ++j) {
            if (!wrow) continue;
            int64_t m = rows ? rows[j] : j;
            for (int64_t k = 0; k < K; ++k) {
                int64_t g = k / G;
                wrow[k] = w4o_fp16_to_double(
                    dequant_one(q[m * K + k], zeros[m * kg + g], scales[m * kg + g]));
            }
            for (int64_t n = 0; n < N; ++n) {
                const double* xn = xd + n * K;
                double acc = 0.0;
                for (int64_t k = 0; k < K; ++k) acc += wrow[k] * xn[k];
                y[n * ny + j] = acc;
            }
        }
        free(wrow);
    }
    free(xd);
    return failed ? 3 : 0;
}

/* Full product: y is [N][M]. */
int w4o_gemm(const uint8_t* q, const uint8_t* zeros, const uint16_t* scales,
             const uint16_t* x, int64_t M, int64_t K, int64_t N, int64_t G, double* y)
{
    return gemm_rows(q, zeros, scales, x, M, K, N, G, NULL, M, y);
}

/* Selected output rows only: y is [N][nrows], column j is weight row rows[j]. */
int w4o_gemm_rows(const uint8_t* q, const uint8_t* zeros, const uint16_t* scales,
                  const uint16_t* x, int64_t M, int64_t K, int64_t N, int64_t G,
                  const int64_t* rows, int64_t nrows, double* y)
{
    return gemm_rows(q, zeros, scales, x, M, K, N, G, rows, nrows, y);
}

/* ------------------------------------------------------------ quantiser ---- */

/*
 * Group quantiser, fp16 W -> (q, s, z): the step before the layer's packing
 * ("PerfXLLM on Snapdragon 8 Gen2", section 3.1: int4 weights, group_size
 * 128, one scale and one zero per group).  The page names no rounding rule;
 * reading taken: min-max asymmetric, with 0 always inside the range, every
 * decision in IEEE fp32 (round to nearest even) so that a GPU can take the
 * same decisions:
 *
 *   lo = min(0, min w), hi = max(0, max w) over the group (exact in fp32);
 *   r  = hi - lo, raised to 2^-14 if smaller;
 *   s  = fp16_RN(r / 15);            f = 1 / float(s);
 *   z  = clamp(rint(-lo * f), 0, 15);
 *   q  = clamp(rint(w * f) + z, 0, 15)   for each w of the group.
 *
 * Each line is one fp32 operation; this file is compiled without
 * floating-point contraction.
 */
int w4o_quantize(const uint16_t* W, int64_t M, int64_t K, int64_t G,
                 uint8_t* q, uint16_t* scales, uint8_t* zeros)
{
    if (check_shape(M, K, G)) return 1;
    const int64_t kg = K / G;
#pragma omp parallel for schedule(static)
    for (int64_t m = 0; m < M; ++m) {
        for (int64_t g = 0; g < kg; ++g) {
            const uint16_t* w = W + m * K + g * G;
            float lo = 0.0f, hi = 0.0f;
            for (int64_t i = 0; i < G; ++i) {
                const float v = (float)w4o_fp16_to_double(w[i]);
                if (v < lo) lo = v;
                if (v > hi) hi = v;
            }
            float r = hi - lo;
            const float r_min = 6.103515625e-05f;          /* 2^-14 */
            if (!(r >= r_min)) r = r_min;
            const float s32 = r / 15.0f;
            const uint16_t s16 = w4o_fp16_from_double((double)s32);
            const float f = 1.0f / (float)w4o_fp16_to_double(s16);
            const float zneg = -lo;
            const float zt = zneg * f;
            float zf = rintf(zt);
            if (zf < 0.0f) zf = 0.0f;
            if (zf > 15.0f) zf = 15.0f;
            for (int64_t i = 0; i < G; ++i) {
                const float v = (float)w4o_fp16_to_double(w[i]);
                const float t = v * f;
                float qf = rintf(t) + zf;
                if (qf < 0.0f) qf = 0.0f;
                if (qf > 15.0f) qf = 15.0f;
                q[m * K + g * G + i] = (uint8_t)qf;
            }
            scales[m * kg + g] = s16;
            zeros[m * kg + g] = (uint8_t)zf;
        }
    }
    return 0;
}

/* ------------------------------------------------ residual add + norm ---- */

/*
 * Residual add and RMS normalisation, the operator that produces the
 * layer's input X.  "PerfXLLM on Snapdragon 8 Gen2", section 3.2, first
 * fusion: the residual connection's addition and the normalisation become
 * one operator, so their intermediate does not travel through global memory.
 * The page names the two operations only; reading taken, per token row n of
 * K channels:
 *
 *   r[k] = fp16_RN(h[k] + d[k])        (d absent: r[k] = h[k]), the new residual
 *   x[k] = r[k] * gamma[k] / sqrt(eps + (1/K) * sum_j r[j]^2)
 *
 * h, d and gamma are fp16.  The sum of two fp16 values is exact in double, so
 * r has one rounding.  The sum of squares runs in fp64 in ascending k; x is
 * returned in fp64, unrounded.
 */
int w4o_add_rmsnorm(const uint16_t* h, const uint16_t* d, const uint16_t* gamma, double eps,
                    int64_t N, int64_t K, uint16_t* r_out, double* x_out)
{
    if (N < 0 || K <= 0 || !(eps >= 0.0)) return 1;
#pragma omp parallel for schedule(static)
    for (int64_t n = 0; n < N; ++n) {
        uint16_t* r = r_out + n * K;
        double ss = 0.0;
        for (int64_t k = 0; k < K; ++k) {
            double v = w4o_fp16_to_double(h[n * K + k]);
            if (d) v += w4o_fp16_to_double(d[n * K + k]);
            r[k] = w4o_fp16_from_double(v);
            const double rv = w4o_fp16_to_double(r[k]);
            ss += rv * rv;
        }
        const double rms = sqrt(ss / (double)K + eps);
        for (int64_t k = 0; k < K; ++k)
            x_out[n * K + k] = w4o_fp16_to_double(r[k]) * w4o_fp16_to_double(gamma[k]) / rms;
    }
    return 0;
}
