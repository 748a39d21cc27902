/*
 * gemm_oracle.c -- the CPU oracle for the dense GEMM path.
 *
 * TEST INFRASTRUCTURE ONLY.  Nothing in the product library links, loads or
 * calls this file; only the tests, the smoke check and the bench's CPU
 * baseline leg do.  It shares no code, header, table or helper with the CUDA
 * path.
 *
 * What it computes is the plain definition of the tiled GEMM that the pages
 * describe ("用Triton跨芯片优化GEMM", sections 2.1 and 3.4; "Triton 学习笔记",
 * section 2.1 on fp32 accumulation; the Gluon/Triton page, section
 * "示例：编写高性能矩阵乘法内核"):
 *
 *     C[i,j] = act( sum_{k<K} A[i,k] * B[k,j]  +  bias[j] )
 *
 * where A and B hold IEEE binary16 or bfloat16 values, the sum is taken in
 * double precision with k ascending (the pages require an accumulator at
 * least as wide as fp32; fp64 makes the oracle's own rounding negligible),
 * bias is optional and act is either the identity or ReLU, max(x, 0).  The
 * result is kept in double and never rounded to the output type: the
 * comparison tolerance absorbs the output cast.
 *
 * Tiling, pipelining, rasterisation and the output cast are properties of the
 * kernels, not of the result, so none of them appears here.  The only steps
 * are: decode the 16-bit inputs to double (own bit-level decoders, written
 * from the IEEE 754 binary16 format and from bfloat16 = the upper half of an
 * IEEE binary32), form the K products per output, add them in order, add the
 * bias, apply ReLU.
 *
 * Layouts (the pages pass a stride pair per operand; here a leading
 * dimension plus one layout flag for B):
 *   A[i,k] = A[i*lda + k]                     (row-major, M x K)
 *   B[k,j] = B[k*ldb + j]     if b_colmajor==0 (row-major, K x N)
 *   B[k,j] = B[j*ldb + k]     if b_colmajor!=0 (column-major, stored N x K)
 *   out[i,j] = out[i*ldo + j] (double, row-major)
 *
 * fp32 inputs (oracle_gemm_f32) follow the same definition; each value
 * converts to double exactly.
 *
 * Grouped variant (the MoE layer's per-expert GEMMs, "用Triton跨芯片优化GEMM"
 * section 2.3): rows of A are sorted by group; group g owns rows
 * [r_g, r_g + rows[g]) with r_g = sum_{h<g} rows[h], and uses the g-th B
 * matrix at B + g*strideB and the g-th bias at bias + g*N.
 *
 * Build: gcc -O2 -fopenmp -shared -fPIC (no -ffast-math, so the fp64 sum is
 * evaluated exactly in the order written).
 */
#include <math.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>

#ifdef _OPENMP
#include <omp.h>
#endif

#define ORACLE_F16 0
#define ORACLE_BF16 1

/* IEEE 754 binary16: 1 sign bit, 5 exponent bits (bias 15), 10 fraction bits.
 * Normal:    (1024 + f) * 2^(e - 25)
 * Subnormal: f * 2^-24
 * e == 31:   infinity (f == 0) or NaN. */
double oracle_decode_f16(uint16_t h)
{
    int s = (h >> 15) & 1;
    int e = (h >> 10) & 0x1f;
    int f = h & 0x3ff;
    double v;
    if (e == 0)
        v = ldexp((double)f, -24);
    else if (e == 31)
        v = f ? NAN : INFINITY;
    else
        v = ldexp((double)(1024 + f), e - 25);
    return s ? -v : v;
}

/* bfloat16: the upper 16 bits of an IEEE binary32 -- 1 sign bit, 8 exponent
 * bits (bias 127), 7 fraction bits.
 * Normal:    (128 + f) * 2^(e - 134)
 * Subnormal: f * 2^-133
 * e == 255:  infinity (f == 0) or NaN. */
double oracle_decode_bf16(uint16_t h)
{
    int s = (h >> 15) & 1;
    int e = (h >> 7) & 0xff;
    int f = h & 0x7f;
    double v;
    if (e == 0)
        v = ldexp((double)f, -133);
    else if (e == 255)
        v = f ? NAN : INFINITY;
    else
        v = ldexp((double)(128 + f), e - 134);
    return s ? -v : v;
}

static double decode(uint16_t h, int dtype)
{
    return dtype == ORACLE_BF16 ? oracle_decode_bf16(h) : oracle_decode_f16(h);
}

int oracle_decode_array(const uint16_t *src, int64_t n, int dtype, double *dst)
{
    if (n < 0 || (n > 0 && (!src || !dst)))
        return -1;
    for (int64_t i = 0; i < n; ++i)
        dst[i] = decode(src[i], dtype);
    return 0;
}

/* The definition itself, on already-decoded operands (double in, double out).
 * Exposed so that properties such as linearity can be checked without the
 * rounding a 16-bit encoding would add. */
int oracle_gemm_f64(int M, int N, int K,
                    const double *A, int64_t lda,
                    const double *B, int64_t ldb, int b_colmajor,
                    const double *bias, int relu,
                    double *out, int64_t ldo, int nthreads)
{
    if (M < 0 || N < 0 || K < 0)
        return -1;
    if (M == 0 || N == 0)
        return 0;
    if (!out || (K > 0 && (!A || !B)))
        return -1;
    if (nthreads < 1)
        nthreads = 1;
    (void)nthreads;
#pragma omp parallel for num_threads(nthreads) schedule(static)
    for (int i = 0; i < M; ++i) {
        for (int j = 0; j < N; ++j) {
            double s = 0.0;
            for (int k = 0; k < K; ++k) {
                double a = A[(int64_t)i * lda + k];
                double b = b_colmajor ? B[(int64_t)j * ldb + k]
                                      : B[(int64_t)k * ldb + j];
                s += a * b;
            }
            if (bias)
                s += bias[j];
            if (relu && s < 0.0)
                s = 0.0;
            out[(int64_t)i * ldo + j] = s;
        }
    }
    return 0;
}

/* Decode a strided 16-bit matrix (rows x cols, leading dimension ld) into a
 * dense double matrix with leading dimension cols. */
static double *decode_matrix(const uint16_t *src, int rows, int cols,
                             int64_t ld, int dtype)
{
    size_t n = (size_t)rows * (size_t)cols;
    double *d = (double *)malloc((n ? n : 1) * sizeof(double));
    if (!d)
        return NULL;
    for (int r = 0; r < rows; ++r)
        for (int c = 0; c < cols; ++c)
            d[(size_t)r * cols + c] = decode(src[(int64_t)r * ld + c], dtype);
    return d;
}

/* Dense GEMM on 16-bit inputs: decode, then the definition above. */
int oracle_gemm(int M, int N, int K,
                const uint16_t *A, int64_t lda,
                const uint16_t *B, int64_t ldb, int b_colmajor,
                const uint16_t *bias, int relu, int dtype,
                double *out, int64_t ldo, int nthreads)
{
    if (M < 0 || N < 0 || K < 0 || (dtype != ORACLE_F16 && dtype != ORACLE_BF16))
        return -1;
    if (M == 0 || N == 0)
        return 0;
    if (!out || (K > 0 && (!A || !B)))
        return -1;
    double *a = K ? decode_matrix(A, M, K, lda, dtype) : NULL;
    /* B decoded in its stored orientation, so the layout flag is honoured by
     * the definition exactly as for the caller's buffer. */
    double *b = NULL;
    if (K) {
        b = b_colmajor ? decode_matrix(B, N, K, ldb, dtype)
                       : decode_matrix(B, K, N, ldb, dtype);
    }
    double *bs = NULL;
    if (bias) {
        bs = (double *)malloc((size_t)N * sizeof(double));
        if (bs)
            oracle_decode_array(bias, N, dtype, bs);
    }
    int rc = -2;
    if ((!K || (a && b)) && (!bias || bs))
        rc = oracle_gemm_f64(M, N, K, a, K, b, b_colmajor ? K : N, b_colmajor,
                             bs, relu, out, ldo, nthreads);
    free(a);
    free(b);
    free(bs);
    return rc;
}

/* Dense GEMM on IEEE binary32 inputs (each value is exactly representable in
 * double, so the conversion is exact): the same definition as above.  This
 * is what an fp32-input GEMM computes before any reduced-precision multiply
 * (tf32) rounds its inputs. */
int oracle_gemm_f32(int M, int N, int K,
                    const float *A, int64_t lda,
                    const float *B, int64_t ldb, int b_colmajor,
                    const float *bias, int relu,
                    double *out, int64_t ldo, int nthreads)
{
    if (M < 0 || N < 0 || K < 0)
        return -1;
    if (M == 0 || N == 0)
        return 0;
    if (!out || (K > 0 && (!A || !B)))
        return -1;
    size_t na = (size_t)M * (size_t)K;
    size_t nb = (size_t)K * (size_t)N;
    double *a = (double *)malloc((na ? na : 1) * sizeof(double));
    double *b = (double *)malloc((nb ? nb : 1) * sizeof(double));
    double *bs = bias ? (double *)malloc((size_t)N * sizeof(double)) : NULL;
    int rc = -2;
    if (a && b && (!bias || bs)) {
        for (int i = 0; i < M; ++i)
            for (int k = 0; k < K; ++k)
                a[(size_t)i * K + k] = (double)A[(int64_t)i * lda + k];
        /* B kept in its stored orientation */
        int rows = b_colmajor ? N : K, cols = b_colmajor ? K : N;
        for (int r = 0; r < rows; ++r)
            for (int c = 0; c < cols; ++c)
                b[(size_t)r * cols + c] = (double)B[(int64_t)r * ldb + c];
        for (int j = 0; bias && j < N; ++j)
            bs[j] = (double)bias[j];
        rc = oracle_gemm_f64(M, N, K, a, K, b, cols, b_colmajor, bs, relu, out, ldo, nthreads);
    }
    free(a);
    free(b);
    free(bs);
    return rc;
}

/* Single output element C[i,j] straight from the 16-bit buffers. */
static double element(int i, int j, int K,
                      const uint16_t *A, int64_t lda,
                      const uint16_t *B, int64_t ldb, int b_colmajor,
                      const uint16_t *bias, int relu, int dtype)
{
    double s = 0.0;
    for (int k = 0; k < K; ++k) {
        double a = decode(A[(int64_t)i * lda + k], dtype);
        double b = decode(b_colmajor ? B[(int64_t)j * ldb + k]
                                     : B[(int64_t)k * ldb + j], dtype);
        s += a * b;
    }
    if (bias)
        s += decode(bias[j], dtype);
    if (relu && s < 0.0)
        s = 0.0;
    return s;
}

/* Sampled dense GEMM: out[t] = C[rows[t], cols[t]] for t < n. */
int oracle_gemm_at(int M, int N, int K,
                   const uint16_t *A, int64_t lda,
                   const uint16_t *B, int64_t ldb, int b_colmajor,
                   const uint16_t *bias, int relu, int dtype,
                   int64_t n, const int64_t *rows, const int64_t *cols,
                   double *out, int nthreads)
{
    if (M < 0 || N < 0 || K < 0 || n < 0 || (dtype != ORACLE_F16 && dtype != ORACLE_BF16))
        return -1;
    if (n == 0)
        return 0;
    if (!rows || !cols || !out || (K > 0 && (!A || !B)))
        return -1;
    for (int64_t t = 0; t < n; ++t)
        if (rows[t] < 0 || rows[t] >= M || cols[t] < 0 || cols[t] >= N)
            return -1;
    if (nthreads < 1)
        nthreads = 1;
    (void)nthreads;
#pragma omp parallel for num_threads(nthreads) schedule(static)
    for (int64_t t = 0; t < n; ++t)
        out[t] = element((int)rows[t], (int)cols[t], K, A, lda, B, ldb,
                         b_colmajor, bias, relu, dtype);
    return 0;
}

/* 2-D convolution, NHWC activations, straight from its definition ("FlagOS
 * 众智跨芯算子优化实践" section 5.3 names convolution as the first operator
 * to reuse the GEMM: it is the same sum of products over a sliding window):
 *
 *   y[n][oh][ow][co] = act( sum_{kh,kw,ci} x[n][ih][iw][ci] * w[kh][kw][ci][co]
 *                           + bias[co] ),  ih = oh*sh - ph + kh*dh,
 *                                          iw = ow*sw - pw + kw*dw,
 *
 * with x taken as 0 outside [0,H) x [0,W) (zero padding).  x is
 * [batch][H][W][cin], w is [KH][KW][cin][cout], y is [batch][OH][OW][cout]
 * (double), OH = (H + 2ph - dh(KH-1) - 1)/sh + 1, OW likewise.  The sum runs
 * kh, kw, ci ascending in fp64. */
int oracle_conv2d_nhwc(int batch, int H, int W, int cin, int cout, int KH, int KW,
                       int sh, int sw, int ph, int pw, int dh, int dw,
                       const uint16_t *x, const uint16_t *w, const uint16_t *bias,
                       int relu, int dtype, double *y, int nthreads)
{
    if (batch < 0 || H < 1 || W < 1 || cin < 1 || cout < 1 || KH < 1 || KW < 1 ||
        sh < 1 || sw < 1 || ph < 0 || pw < 0 || dh < 1 || dw < 1 ||
        (dtype != ORACLE_F16 && dtype != ORACLE_BF16))
        return -1;
    const int OH = (H + 2 * ph - dh * (KH - 1) - 1) / sh + 1;
    const int OW = (W + 2 * pw - dw * (KW - 1) - 1) / sw + 1;
    if (OH < 1 || OW < 1)
        return -1;
    if (!x || !w || !y)
        return -1;
    if (nthreads < 1)
        nthreads = 1;
    (void)nthreads;
    const int64_t rows = (int64_t)batch * OH * OW;
#pragma omp parallel for num_threads(nthreads) schedule(static)
    for (int64_t r = 0; r < rows; ++r) {
        const int n = (int)(r / ((int64_t)OH * OW));
        const int oh = (int)((r / OW) % OH);
        const int ow = (int)(r % OW);
        for (int co = 0; co < cout; ++co) {
            double s = 0.0;
            for (int kh = 0; kh < KH; ++kh) {
                const int ih = oh * sh - ph + kh * dh;
                for (int kw = 0; kw < KW; ++kw) {
                    const int iw = ow * sw - pw + kw * dw;
                    if (ih < 0 || ih >= H || iw < 0 || iw >= W)
                        continue;  /* zero padding contributes nothing */
                    for (int ci = 0; ci < cin; ++ci) {
                        double a = decode(x[(((int64_t)n * H + ih) * W + iw) * cin + ci], dtype);
                        double b = decode(w[(((int64_t)kh * KW + kw) * cin + ci) * cout + co], dtype);
                        s += a * b;
                    }
                }
            }
            if (bias)
                s += decode(bias[co], dtype);
            if (relu && s < 0.0)
                s = 0.0;
            y[r * cout + co] = s;
        }
    }
    return 0;
}

/* Group that owns global row r, and that group's first row; -1 if none. */
static int group_of_row(int G, const int32_t *group_rows, int64_t r,
                        int64_t *first)
{
    int64_t start = 0;
    for (int g = 0; g < G; ++g) {
        if (r >= start && r < start + group_rows[g]) {
            *first = start;
            return g;
        }
        start += group_rows[g];
    }
    return -1;
}

static int check_groups(int G, const int32_t *group_rows, int64_t *total)
{
    if (G < 0 || (G > 0 && !group_rows))
        return -1;
    int64_t t = 0;
    for (int g = 0; g < G; ++g) {
        if (group_rows[g] < 0)
            return -1;
        t += group_rows[g];
    }
    *total = t;
    return 0;
}

/* Grouped GEMM, full output: for every group g and every row r it owns,
 * out[r, :] = act(A[r, :] . B_g + bias_g). */
int oracle_grouped_gemm(int G, const int32_t *group_rows, int N, int K,
                        const uint16_t *A, int64_t lda,
                        const uint16_t *B, int64_t ldb, int64_t strideB,
                        int b_colmajor,
                        const uint16_t *bias, int relu, int dtype,
                        double *out, int64_t ldo, int nthreads)
{
    int64_t total = 0;
    if (N < 0 || K < 0 || check_groups(G, group_rows, &total) ||
        (dtype != ORACLE_F16 && dtype != ORACLE_BF16))
        return -1;
    int64_t row0 = 0;
    for (int g = 0; g < G; ++g) {
        int m = group_rows[g];
        if (m > 0) {
            int rc = oracle_gemm(m, N, K, A ? A + row0 * lda : NULL, lda,
                                 B ? B + (int64_t)g * strideB : NULL, ldb,
                                 b_colmajor, bias ? bias + (int64_t)g * N : NULL,
                                 relu, dtype, out + row0 * ldo, ldo, nthreads);
            if (rc)
                return rc;
        }
        row0 += m;
    }
    return 0;
}

/* Grouped GEMM, sampled: out[t] = C[rows[t], cols[t]] with rows[t] a global
 * row index (it selects its group). */
int oracle_grouped_gemm_at(int G, const int32_t *group_rows, int N, int K,
                           const uint16_t *A, int64_t lda,
                           const uint16_t *B, int64_t ldb, int64_t strideB,
                           int b_colmajor,
                           const uint16_t *bias, int relu, int dtype,
                           int64_t n, const int64_t *rows, const int64_t *cols,
                           double *out, int nthreads)
{
    int64_t total = 0;
    if (N < 0 || K < 0 || n < 0 || check_groups(G, group_rows, &total) ||
        (dtype != ORACLE_F16 && dtype != ORACLE_BF16))
        return -1;
    if (n == 0)
        return 0;
    if (!rows || !cols || !out || (K > 0 && (!A || !B)))
        return -1;
    for (int64_t t = 0; t < n; ++t)
        if (rows[t] < 0 || rows[t] >= total || cols[t] < 0 || cols[t] >= N)
            return -1;
    if (nthreads < 1)
        nthreads = 1;
    (void)nthreads;
#pragma omp parallel for num_threads(nthreads) schedule(static)
    for (int64_t t = 0; t < n; ++t) {
        int64_t first = 0;
        int g = group_of_row(G, group_rows, rows[t], &first);
        out[t] = element((int)rows[t], (int)cols[t], K, A, lda,
                         B + (int64_t)g * strideB, ldb, b_colmajor,
                         bias ? bias + (int64_t)g * N : NULL, relu, dtype);
    }
    return 0;
}

/* Threads an OpenMP region of nthreads actually gets (1 without OpenMP). */
int oracle_threads_used(int nthreads)
{
    int used = 1;
#ifdef _OPENMP
    if (nthreads < 1)
        nthreads = 1;
#pragma omp parallel num_threads(nthreads)
    {
#pragma omp single
        used = omp_get_num_threads();
    }
#else
    (void)nthreads;
#endif
    return used;
}
