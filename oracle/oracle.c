/*
 * oracle.c -- plain, slow, fp64 CPU reference for the small-M decode GEMM
 *
 *     Y[m, n] = sum_k X[m, k] * W[n, k]        (X: [M, K], W: [N, K], Y: [M, N])
 *
 * TEST INFRASTRUCTURE ONLY.  Nothing in the product path may call, link or
 * load this file; only the tests, the package smoke check and the benchmark's
 * CPU-baseline leg use it.  It shares no code, header, table or constant with
 * the CUDA library.
 *
 * What it follows:
 *   - The decode GEMM regime (small M, K and N in the thousands) of
 *     "AMD: ROCm Low-Latency-GEMM-Kernel beschleunigen LLM-Inferenz bis zu
 *     1,79x auf Instinct MI355X", section "Was ist GEMM und die Decode-Phase".
 *   - The linear layers being the whole cost of decode, and their shapes
 *     (d = 4096, d_ff = 12288), from "Fleet: Hierarchical Task-based
 *     Abstraction for Megakernels on Multi-Die GPUs" (reading notes),
 *     Summary and section 1 "System Scope".
 *   The pages never define the arithmetic.  The reading used here is the
 *   plain definition of the product: each output is the exact dot product of a
 *   row of X with a row of W, accumulated in fp64 in increasing k over
 *   bf16 inputs widened exactly to fp64, then rounded once (round to nearest,
 *   ties to even) to bf16.
 *
 * bf16 is the upper 16 bits of an IEEE-754 binary32 value: 1 sign bit,
 * 8 exponent bits, 7 fraction bits.
 */
#include <math.h>
#include <stdint.h>
#include <string.h>
#include <stddef.h>

#ifdef _OPENMP
#include <omp.h>
#endif

/* bf16 bit pattern -> fp64 value.  Exact: every bf16 value is a binary32
 * value, and every binary32 value is a binary64 value. */
double wsmo_bf16_to_f64(uint16_t h)
{
    uint32_t bits = (uint32_t)h << 16;
    float f;
    memcpy(&f, &bits, sizeof f);
    return (double)f;
}

/* fp64 value -> nearest bf16 bit pattern, ties to even, written from the
 * IEEE-754 definition of rounding to a format with p = 8 significand bits,
 * emin = -126 and emax = 127:
 *   - NaN maps to a quiet NaN with the input's sign;
 *   - magnitudes at or above (2 - 2^-8) * 2^127, the midpoint between the
 *     largest finite bf16 and 2^128, round to infinity (that midpoint's
 *     neighbours are the odd-significand max finite and the even 2^128);
 *   - otherwise the quantum of the binade of |y| (clamped at the subnormal
 *     quantum 2^-133) divides |y|, the quotient is rounded to the nearest
 *     integer with ties to even, and the product with the quantum is the
 *     result, which is exactly representable in bf16 (and binary32). */
uint16_t wsmo_f64_to_bf16(double y)
{
    uint16_t sign = signbit(y) ? 0x8000u : 0u;
    double a = fabs(y);
    if (isnan(y))
        return (uint16_t)(sign | 0x7FC0u);
    const double overflow_mid = (2.0 - ldexp(1.0, -8)) * ldexp(1.0, 127);
    if (a >= overflow_mid)
        return (uint16_t)(sign | 0x7F80u);
    if (a == 0.0)
        return sign;
    int e2;
    (void)frexp(a, &e2);          /* a = f * 2^e2 with f in [0.5, 1) */
    int e = e2 - 1;               /* a in [2^e, 2^(e+1)) */
    if (e < -126)
        e = -126;                 /* subnormal range shares the quantum 2^-133 */
    double q = ldexp(1.0, e - 7); /* spacing of bf16 values in this binade */
    double r = a / q;             /* exact: division by a power of two */
    double n = floor(r);
    double frac = r - n;          /* exact */
    if (frac > 0.5 || (frac == 0.5 && fmod(n, 2.0) != 0.0))
        n += 1.0;
    double v = n * q;             /* exact, and representable in bf16 */
    float vf = (float)v;          /* exact */
    uint32_t bits;
    memcpy(&bits, &vf, sizeof bits);
    return (uint16_t)(sign | (uint16_t)(bits >> 16));
}

void wsmo_round_bf16(const double *y, int64_t count, uint16_t *out)
{
    for (int64_t i = 0; i < count; ++i)
        out[i] = wsmo_f64_to_bf16(y[i]);
}

/* Full product.  Y_ref and S (= sum_k |X[m,k] * W[n,k]|, the scale the
 * acceptance bound is stated in) are [M, N] row-major fp64.  Each output is an
 * independent loop over k in increasing order, so the thread count changes
 * nothing in the result. */
void wsmo_gemm(const uint16_t *X, const uint16_t *W, int M, int N, int K,
               double *Y_ref, double *S)
{
    int64_t total = (int64_t)M * N;
#pragma omp parallel for schedule(static)
    for (int64_t idx = 0; idx < total; ++idx) {
        int m = (int)(idx / N);
        int n = (int)(idx % N);
        const uint16_t *xr = X + (size_t)m * K;
        const uint16_t *wr = W + (size_t)n * K;
        double acc = 0.0, sabs = 0.0;
        for (int k = 0; k < K; ++k) {
            double p = wsmo_bf16_to_f64(xr[k]) * wsmo_bf16_to_f64(wr[k]);
            acc += p;
            sabs += fabs(p);
        }
        Y_ref[idx] = acc;
        if (S)
            S[idx] = sabs;
    }
}

/* The same definition evaluated only at `count` sampled output positions
 * (ms[i], ns[i]); used where the full product is too large for the CPU. */
void wsmo_gemm_sampled(const uint16_t *X, const uint16_t *W, int M, int N, int K,
                       const int32_t *ms, const int32_t *ns, int64_t count,
                       double *Y_ref, double *S)
{
    (void)M;
    (void)N;
#pragma omp parallel for schedule(static)
    for (int64_t i = 0; i < count; ++i) {
        const uint16_t *xr = X + (size_t)ms[i] * K;
        const uint16_t *wr = W + (size_t)ns[i] * K;
        double acc = 0.0, sabs = 0.0;
        for (int k = 0; k < K; ++k) {
            double p = wsmo_bf16_to_f64(xr[k]) * wsmo_bf16_to_f64(wr[k]);
            acc += p;
            sabs += fabs(p);
        }
        Y_ref[i] = acc;
        if (S)
            S[i] = sabs;
    }
}

/* Thread control for the timed CPU baseline; returns the count in effect. */
int wsmo_set_threads(int n)
{
#ifdef _OPENMP
    if (n > 0)
        omp_set_num_threads(n);
    return omp_get_max_threads();
#else
    (void)n;
    return 1;
#endif
}
