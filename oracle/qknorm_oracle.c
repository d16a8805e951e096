/*
 * qknorm_oracle.c -- plain fp64 CPU oracle for QK-Norm and FlashNorm.
 *
 * TEST INFRASTRUCTURE ONLY.  Only the tests, the package smoke check and the
 * benchmark's CPU-baseline leg may load this library; the CUDA library never
 * does, and the two share no code, headers or constants.
 *
 * Everything is computed in double precision from inputs that the caller has
 * widened exactly (fp32 and bf16 values are exact doubles).  Rows are
 * independent, so OpenMP splits work over rows only; the arithmetic inside a
 * row is a plain left-to-right loop whose order does not depend on the number
 * of threads.  Build without -ffast-math and with -ffp-contract=off.
 *
 * What each function restates (the pages give the method in words, not in
 * formulas; the formula below is the standard RMSNorm definition):
 *
 *   SwiftQK, abstract: layerwise QK-Norm is an RMSNorm of each token's full
 *   query vector and full key vector; under tensor parallelism each shard
 *   contributes a scalar partial sum of squares and only those scalars are
 *   exchanged, which leaves the normalisation itself unchanged.
 *     RMSNorm(x)_i = x_i / sqrt(mean_i(x_i^2) + eps) * w_i
 *
 *   FlashNorm (Graef), abstract, items (i) and (ii): the weights w are folded
 *   into the next linear layer, W' = diag(w) W, and the 1/rms scaling is
 *   applied to the matmul output:  y = (x W') / rms(x), an exact
 *   reformulation of RMSNorm(x) W.
 */
#include <math.h>
#include <stdint.h>
#include <string.h>
#include <stdlib.h>
#ifdef _OPENMP
#include <omp.h>
#endif

/* Number of threads the oracle's parallel loops use. */
int oracle_threads(void)
{
#ifdef _OPENMP
    return omp_get_max_threads();
#else
    return 1;
#endif
}

/* Sum of squares of n consecutive values, left to right. */
static double sum_sq(const double *x, int64_t n)
{
    double s = 0.0;
    for (int64_t i = 0; i < n; ++i)
        s += x[i] * x[i];
    return s;
}

/*
 * SwiftQK, abstract (QK-Norm = RMSNorm over the full vector):
 *   y[r][i] = x[r][i] / sqrt(S_r / d + eps) * w[i],   S_r = sum_i x[r][i]^2.
 * x: rows x d with leading dimension ld; y: rows x d, contiguous.
 */
void oracle_rmsnorm(const double *x, int64_t rows, int64_t d, int64_t ld,
                    const double *w, double eps, double *y)
{
#pragma omp parallel for schedule(static)
    for (int64_t r = 0; r < rows; ++r) {
        const double *xr = x + r * ld;
        double *yr = y + r * d;
        double S = sum_sq(xr, d);
        double rms = sqrt(S / (double)d + eps);
        for (int64_t i = 0; i < d; ++i)
            yr[i] = xr[i] / rms * w[i];
    }
}

/*
 * SwiftQK, abstract (scalar partial sums): split each row into n_seg
 * contiguous equal segments -- the slices the n_seg tensor-parallel shards
 * would hold -- and return each segment's sum of squares.
 *   partial[r][j] = sum_{i in [j*d/n_seg, (j+1)*d/n_seg)} x[r][i]^2
 * Requires d % n_seg == 0 (returns -1 otherwise, 0 on success).
 */
int oracle_segment_partials(const double *x, int64_t rows, int64_t d, int64_t ld,
                            int64_t n_seg, double *partial)
{
    if (n_seg <= 0 || d % n_seg != 0)
        return -1;
    int64_t len = d / n_seg;
#pragma omp parallel for schedule(static)
    for (int64_t r = 0; r < rows; ++r)
        for (int64_t j = 0; j < n_seg; ++j)
            partial[r * n_seg + j] = sum_sq(x + r * ld + j * len, len);
    return 0;
}

/*
 * SwiftQK, abstract: the exchanged scalars are combined into the full-row
 * statistic; here in a fixed left-to-right order, S = ((S_0 + S_1) + ...).
 */
void oracle_combine_partials(const double *partial, int64_t rows, int64_t n_seg,
                             double *S)
{
    for (int64_t r = 0; r < rows; ++r) {
        double s = 0.0;
        for (int64_t j = 0; j < n_seg; ++j)
            s += partial[r * n_seg + j];
        S[r] = s;
    }
}

/* 1/rms of each row: inv[r] = 1 / sqrt(S_r / d + eps). */
void oracle_inv_rms(const double *x, int64_t rows, int64_t d, int64_t ld,
                    double eps, double *inv)
{
#pragma omp parallel for schedule(static)
    for (int64_t r = 0; r < rows; ++r)
        inv[r] = 1.0 / sqrt(sum_sq(x + r * ld, d) / (double)d + eps);
}

/* FlashNorm, abstract item (i): W'[k][n] = w[k] * W[k][n]; W is K x N. */
void oracle_fold_weights(const double *w, const double *W, int64_t K, int64_t N,
                         double *Wf)
{
#pragma omp parallel for schedule(static)
    for (int64_t k = 0; k < K; ++k)
        for (int64_t n = 0; n < N; ++n)
            Wf[k * N + n] = w[k] * W[k * N + n];
}

/*
 * Reference semantics that FlashNorm reformulates: RMSNorm(x) followed by the
 * linear layer, Y = RMSNorm(x; w, eps) W.  x: M x K, W: K x N, Y: M x N.
 */
void oracle_norm_then_project(const double *x, int64_t M, int64_t K,
                              const double *w, const double *W, int64_t N,
                              double eps, double *Y)
{
#pragma omp parallel for schedule(static)
    for (int64_t m = 0; m < M; ++m) {
        const double *xm = x + m * K;
        double rms = sqrt(sum_sq(xm, K) / (double)K + eps);
        double *Ym = Y + m * N;
        for (int64_t n = 0; n < N; ++n)
            Ym[n] = 0.0;
        for (int64_t k = 0; k < K; ++k) {
            double a = xm[k] / rms * w[k];
            const double *Wk = W + k * N;
            for (int64_t n = 0; n < N; ++n)
                Ym[n] += a * Wk[n];
        }
    }
}

/*
 * FlashNorm, abstract item (ii): the matmul runs on the raw x with the folded
 * weights and the scalar 1/rms(x) is applied to its output,
 *   Y[m][n] = (sum_k x[m][k] * Wf[k][n]) / rms(x_m).
 */
void oracle_flashnorm_deferred(const double *x, int64_t M, int64_t K,
                               const double *Wf, int64_t N, double eps, double *Y)
{
#pragma omp parallel for schedule(static)
    for (int64_t m = 0; m < M; ++m) {
        const double *xm = x + m * K;
        double *Ym = Y + m * N;
        for (int64_t n = 0; n < N; ++n)
            Ym[n] = 0.0;
        for (int64_t k = 0; k < K; ++k) {
            double a = xm[k];
            const double *Wk = Wf + k * N;
            for (int64_t n = 0; n < N; ++n)
                Ym[n] += a * Wk[n];
        }
        double rms = sqrt(sum_sq(xm, K) / (double)K + eps);
        for (int64_t n = 0; n < N; ++n)
            Ym[n] = Ym[n] / rms;
    }
}

/*
 * Round a double to bfloat16 (1 sign, 8 exponent, 7 fraction bits, the
 * exponent range of binary32) with round-to-nearest, ties to even, directly
 * from the double -- no intermediate rounding to binary32.  Returns the
 * 16-bit pattern.  NaN maps to a quiet NaN with the input's sign.
 *
 * Method: inside a binade [2^E, 2^(E+1)) the representable values are the
 * multiples of 2^(E-7) (for E >= -126; below that the subnormal spacing
 * 2^-133 applies).  Divide by that spacing (exact: a power of two), round to
 * the nearest integer with ties to even, multiply back.  The result is then a
 * bfloat16 value, which is also a binary32 value, and its pattern is the top
 * half of the binary32 pattern.
 */
static uint16_t bf16_rne_one(double v)
{
    uint16_t sign = signbit(v) ? 0x8000u : 0u;
    if (isnan(v))
        return (uint16_t)(sign | 0x7FC0u);
    double a = fabs(v);
    if (isinf(a))
        return (uint16_t)(sign | 0x7F80u);
    if (a == 0.0)
        return sign;
    int ex;
    (void)frexp(a, &ex);            /* a = f * 2^ex, f in [0.5, 1) */
    int E = ex - 1;                 /* a in [2^E, 2^(E+1)) */
    if (E < -126)
        E = -126;                   /* subnormal range: fixed spacing */
    double spacing = ldexp(1.0, E - 7);
    double n = nearbyint(a / spacing);   /* default mode: nearest, ties even */
    double r = n * spacing;
    if (r >= ldexp(1.0, 128))
        return (uint16_t)(sign | 0x7F80u);
    float f = (float)r;             /* exact */
    uint32_t bits;
    memcpy(&bits, &f, sizeof bits);
    return (uint16_t)(sign | (uint16_t)((bits >> 16) & 0x7FFFu));
}

void oracle_round_bf16(const double *v, int64_t n, uint16_t *out)
{
#pragma omp parallel for schedule(static)
    for (int64_t i = 0; i < n; ++i)
        out[i] = bf16_rne_one(v[i]);
}
