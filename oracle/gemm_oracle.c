/*
 * CPU oracle for the fp16 GEMM (+bias+ReLU) path.  TEST INFRASTRUCTURE ONLY:
 * the tests, the smoke check and the benchmark's CPU-baseline leg use it; the
 * CUDA library never does, and the two share no code.
 *
 * What it computes is the plain definition, written out with no blocking,
 * fusion or reordering:
 *
 *   ref[i][j] = sum_{k=0}^{K-1} dec(A[i][k]) * dec(B[k][j])          (fp64)
 *   bias+ReLU variant: ref[i][j] = max(ref[i][j] + dec(bias[j]), 0)
 *
 * Sources, by page and section:
 *   - the GEMM C = A.B on an fp16 MxK row-major A and an fp16 KxN row-major B
 *     with an fp32 accumulator: "tilelang operator-compilation walkthrough"
 *     (lqnn.cn/news/222844) sections 2.1 and 4.2; the fp32-output form:
 *     "TileLang Python DSL practice" (codechina.net/.../126997) section 3.2.
 *   - the fused epilogue, bias indexed by the output column and added before
 *     the ReLU: "domestic-GPU TileLang adoption" (xdnf.cn/news/333523)
 *     section 4.2; the same page's section 4.1 names fusing an activation
 *     and a residual connection into the GEMM, written here as
 *     ref = act(A.B + bias[j]) + R[i][j] with act = none, ReLU, GELU, SiLU
 *     or GELU's tanh form.  The pages give no activation formulas; each is
 *     its standard definition (oracle_activation below).
 *
 * The accumulation is fp64 (every fp16 x fp16 product is exact in fp64), so
 * the result is the exact sum up to fp64 rounding.  The k order is ascending
 * in both the full and the sampled routine, so the two agree bit for bit.
 *
 * Every function here is pinned by the CPU tests against something other than
 * itself (numpy's float16 for the codec, numpy's fp64 matmul, math.fsum,
 * closed forms and hand-worked fixtures); no function is "parity unpinned".
 */
#include <math.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>

#ifdef _OPENMP
#include <omp.h>
#endif

/* IEEE 754 binary16: 1 sign bit, 5 exponent bits (bias 15), 10 fraction bits. */
double oracle_f16_decode(uint16_t h)
{
    const int sign = (h >> 15) & 1;
    const int e = (h >> 10) & 0x1f;
    const int f = h & 0x3ff;
    double v;
    if (e == 0)
        v = ldexp((double)f, -24); /* zero or subnormal: f * 2^-24 */
    else if (e == 31)
        v = f ? NAN : INFINITY;
    else
        v = ldexp((double)(1024 + f), e - 25); /* (1 + f/1024) * 2^(e-15) */
    return sign ? -v : v;
}

/* Round a double to binary16, round-to-nearest, ties to even; overflow gives inf. */
uint16_t oracle_f16_encode_rne(double x)
{
    const uint16_t sign = signbit(x) ? 0x8000u : 0u;
    if (isnan(x))
        return 0x7e00u;
    double a = fabs(x);
    if (a == 0.0)
        return sign;
    if (isinf(a))
        return (uint16_t)(sign | 0x7c00u);
    int e2;
    (void)frexp(a, &e2); /* a = m * 2^e2, m in [0.5, 1) */
    int E = e2 - 1;      /* a = m' * 2^E,  m' in [1, 2) */
    if (E < -14) {
        /* subnormal range: the spacing is 2^-24 */
        double n = nearbyint(ldexp(a, 24)); /* ties to even under the default rounding mode */
        return (uint16_t)(sign | (uint16_t)n); /* n == 1024 lands on the smallest normal */
    }
    double n = nearbyint(ldexp(a, 10 - E)); /* in [1024, 2048] */
    if (n == 2048.0) {
        n = 1024.0;
        E += 1;
    }
    if (E > 15)
        return (uint16_t)(sign | 0x7c00u);
    return (uint16_t)(sign | (uint16_t)((E + 15) << 10) | (uint16_t)((int)n - 1024));
}

void oracle_f16_decode_array(const uint16_t *h, double *out, int64_t n)
{
    for (int64_t i = 0; i < n; ++i)
        out[i] = oracle_f16_decode(h[i]);
}

void oracle_f16_encode_array(const double *x, uint16_t *out, int64_t n)
{
    for (int64_t i = 0; i < n; ++i)
        out[i] = oracle_f16_encode_rne(x[i]);
}

/* Activation codes shared by the fused routines below. */
enum {
    ORACLE_ACT_NONE = 0,
    ORACLE_ACT_RELU = 1,
    ORACLE_ACT_GELU = 2,
    ORACLE_ACT_SILU = 3,
    ORACLE_ACT_GELU_TANH = 4
};

/*
 * The activations by their standard definitions (the pages name activation
 * fusion but print no formulas):
 *   ReLU  max(x, 0)
 *   GELU  x * Phi(x) = x/2 * (1 + erf(x / sqrt 2))
 *   SiLU  x * sigmoid(x) = x / (1 + exp(-x))
 *   GELU, tanh form  x/2 * (1 + tanh(sqrt(2/pi) * (x + 0.044715 x^3)))
 */
double oracle_activation(double x, int act)
{
    if (act == ORACLE_ACT_RELU)
        return x > 0.0 ? x : 0.0;
    if (act == ORACLE_ACT_GELU)
        return 0.5 * x * (1.0 + erf(x / sqrt(2.0)));
    if (act == ORACLE_ACT_SILU)
        return x / (1.0 + exp(-x));
    if (act == ORACLE_ACT_GELU_TANH) {
        const double pi = 3.14159265358979323846;
        return 0.5 * x * (1.0 + tanh(sqrt(2.0 / pi) * (x + 0.044715 * x * x * x)));
    }
    return x;
}

/*
 * Full product with the fused epilogue:
 *   C[i][j] = act(sum_k A[i][k] B[k][j] + bias[j]) + R[i][j]
 * bias (N fp16 bits) may be NULL.  R holds the residual's values (M x N
 * doubles, row stride ldr: the residual has the output's type, fp16 or fp32,
 * and either converts to fp64 exactly) and may be NULL.
 * Returns 0, or -1 if the decoded copy of B cannot be allocated.
 */
int oracle_gemm_fused(int64_t M, int64_t N, int64_t K,
                      const uint16_t *A, int64_t lda,
                      const uint16_t *B, int64_t ldb,
                      const uint16_t *bias, int act,
                      const double *R, int64_t ldr,
                      double *C, int64_t ldc, int nthreads)
{
    double *Bd = (double *)malloc((size_t)(K * N > 0 ? K * N : 1) * sizeof(double));
    if (!Bd)
        return -1;
    for (int64_t k = 0; k < K; ++k)
        for (int64_t j = 0; j < N; ++j)
            Bd[k * N + j] = oracle_f16_decode(B[k * ldb + j]);
    if (nthreads < 1)
        nthreads = 1;

#pragma omp parallel for num_threads(nthreads) schedule(static)
    for (int64_t i = 0; i < M; ++i) {
        double *c = C + i * ldc;
        for (int64_t j = 0; j < N; ++j)
            c[j] = 0.0;
        for (int64_t k = 0; k < K; ++k) {
            const double a = oracle_f16_decode(A[i * lda + k]);
            const double *b = Bd + k * N;
            for (int64_t j = 0; j < N; ++j)
                c[j] += a * b[j];
        }
        for (int64_t j = 0; j < N; ++j) {
            double v = c[j];
            if (bias)
                v += oracle_f16_decode(bias[j]);
            v = oracle_activation(v, act);
            if (R)
                v += R[i * ldr + j];
            c[j] = v;
        }
    }
    free(Bd);
    return 0;
}

/*
 * Full product.  A: M x K fp16 bits, row stride lda; B: K x N, row stride ldb;
 * bias: N fp16 bits or NULL; C: M x N doubles, row stride ldc.
 * relu != 0 applies max(., 0) after the bias.  Rows are split over nthreads
 * OpenMP threads; each output keeps its own ascending-k sum.
 * Returns 0, or -1 if the decoded copy of B cannot be allocated.
 */
int oracle_gemm(int64_t M, int64_t N, int64_t K,
                const uint16_t *A, int64_t lda,
                const uint16_t *B, int64_t ldb,
                const uint16_t *bias, int relu,
                double *C, int64_t ldc, int nthreads)
{
    /* decode B once (an elementwise step; no reordering of the sums) */
    double *Bd = (double *)malloc((size_t)(K * N > 0 ? K * N : 1) * sizeof(double));
    if (!Bd)
        return -1;
    for (int64_t k = 0; k < K; ++k)
        for (int64_t j = 0; j < N; ++j)
            Bd[k * N + j] = oracle_f16_decode(B[k * ldb + j]);
    if (nthreads < 1)
        nthreads = 1;

#pragma omp parallel for num_threads(nthreads) schedule(static)
    for (int64_t i = 0; i < M; ++i) {
        double *c = C + i * ldc;
        for (int64_t j = 0; j < N; ++j)
            c[j] = 0.0;
        for (int64_t k = 0; k < K; ++k) {
            const double a = oracle_f16_decode(A[i * lda + k]);
            const double *b = Bd + k * N;
            for (int64_t j = 0; j < N; ++j)
                c[j] += a * b[j];
        }
        if (bias)
            for (int64_t j = 0; j < N; ++j)
                c[j] += oracle_f16_decode(bias[j]);
        if (relu)
            for (int64_t j = 0; j < N; ++j)
                c[j] = c[j] > 0.0 ? c[j] : 0.0;
    }
    free(Bd);
    return 0;
}

/*
 * Selected outputs only: out[s] = ref[rows[s]][cols[s]], each a length-K
 * dot product in ascending k, then bias, activation and residual as above.
 */
void oracle_gemm_at_fused(int64_t K,
                          const uint16_t *A, int64_t lda,
                          const uint16_t *B, int64_t ldb,
                          const uint16_t *bias, int act,
                          const double *R, int64_t ldr,
                          const int64_t *rows, const int64_t *cols, int64_t count,
                          double *out, int nthreads)
{
    if (nthreads < 1)
        nthreads = 1;
#pragma omp parallel for num_threads(nthreads) schedule(static)
    for (int64_t s = 0; s < count; ++s) {
        const int64_t i = rows[s], j = cols[s];
        double acc = 0.0;
        for (int64_t k = 0; k < K; ++k)
            acc += oracle_f16_decode(A[i * lda + k]) * oracle_f16_decode(B[k * ldb + j]);
        if (bias)
            acc += oracle_f16_decode(bias[j]);
        acc = oracle_activation(acc, act);
        if (R)
            acc += R[i * ldr + j];
        out[s] = acc;
    }
}

void oracle_gemm_at(int64_t K,
                    const uint16_t *A, int64_t lda,
                    const uint16_t *B, int64_t ldb,
                    const uint16_t *bias, int relu,
                    const int64_t *rows, const int64_t *cols, int64_t count,
                    double *out, int nthreads)
{
    oracle_gemm_at_fused(K, A, lda, B, ldb, bias, relu ? ORACLE_ACT_RELU : ORACLE_ACT_NONE,
                         NULL, 0, rows, cols, count, out, nthreads);
}

int oracle_openmp_enabled(void)
{
#ifdef _OPENMP
    return 1;
#else
    return 0;
#endif
}
