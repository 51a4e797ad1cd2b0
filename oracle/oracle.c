/*
 * oracle.c -- the CPU oracle for the tiled dense GEMM library.
 *
 * TEST INFRASTRUCTURE ONLY.  Nothing on the product path links, loads or
 * calls this file; only the tests, the smoke check and the benchmark's CPU
 * baseline leg do.  It shares no code, header, table or helper with the CUDA
 * library under tiled_dense_gemm_tma_b200/csrc.
 *
 * What it computes is the plain definition of the operation the pages build
 * kernels for:
 *
 *     C[i][j] = epi( sum_{k<K} A[i][k] * B[k][j] )
 *
 *   - the scalar triple loop written out on "TileLang: 用Python DSL简化GPU算子
 *     开发与FlashAttention实现" (gtnt.cn), section 1.1, and the tiling
 *     rationale on "TileLang ... 高效 GEMM 内核" (mhpq.cn), section 2.1, which
 *     states C = A x B for row-major A (M x K) and B (K x N);
 *   - epi is the identity or ReLU, the output post-processing named on
 *     "使用 Tilelang DSL 开发 GPU/CPU/加速器高性能内核" (blog.hotdry.top),
 *     landing checklist item 2;
 *   - the dequantize GEMM (same blog page, last paragraphs: "Dequant GEMM")
 *     multiplies by an explicitly dequantised weight W[k][n] = q[k][n] *
 *     s[k / 128][n].  The pages give no storage format; the one used here is
 *     the library's documented reading: signed 4-bit q packed two per byte,
 *     even column in the low nibble, fp16 scales per 128 rows of K.
 *
 *   - the FP4-weight ("WFP4") GEMM named in the performance section of
 *     "TileLang架构深度剖析" (test.krestaai.com.au) likewise multiplies by an
 *     explicitly dequantised weight.  The pages give no FP4 format; the
 *     library's reading is MXFP4 from the OCP Microscaling Formats (MX)
 *     specification v1.0: E2M1 elements (sign, 2 exponent bits with bias 1,
 *     1 mantissa bit) sharing one E8M0 scale 2^(E - 127) per 32 consecutive
 *     k of a column, with bf16 activations.
 *
 * Every stored input value is widened exactly to double, products and sums
 * are taken in double, and ReLU is applied in double.  No blocking, no
 * reordering beyond the i-k-j loop order, no fusion.  Rows of C are spread
 * over OpenMP threads; each C element is still one sequential sum over k in
 * increasing order.
 *
 * Rounding helpers turn a double into the stored output type with
 * round-to-nearest-even, for bit-exact comparisons on integer-valued inputs.
 */
#include <stdint.h>
#include <string.h>
#include <math.h>
#include <stdlib.h>
#ifdef _OPENMP
#include <omp.h>
#endif

/* ------------------------------------------------------------------------ */
/* Decoding of stored values (independent of any generator or GPU code).    */
/* ------------------------------------------------------------------------ */

/* IEEE binary16 bit pattern -> double (exact). */
double oracle_f16_to_f64(uint16_t h)
{
    int sign = (h >> 15) & 1;
    int expo = (h >> 10) & 0x1f;
    int mant = h & 0x3ff;
    double v;
    if (expo == 0) {
        v = ldexp((double)mant, -24);                 /* subnormal: m * 2^-24 */
    } else if (expo == 31) {
        v = mant ? NAN : INFINITY;
    } else {
        v = ldexp((double)(mant | 0x400), expo - 25); /* (1.m) * 2^(e-15) */
    }
    return sign ? -v : v;
}

/* bfloat16 bit pattern -> double (exact): the upper half of a binary32. */
double oracle_bf16_to_f64(uint16_t b)
{
    uint32_t u = (uint32_t)b << 16;
    float f;
    memcpy(&f, &u, sizeof f);
    return (double)f;
}

/* Signed 4-bit value of column n in a packed row (two's complement). */
static int oracle_nibble(const uint8_t *row, int64_t n)
{
    uint8_t byte = row[n >> 1];
    int v = (n & 1) ? (byte >> 4) : (byte & 0x0f);
    return v >= 8 ? v - 16 : v;
}

/* Unsigned 4-bit code of column n in a packed row (low nibble = even column). */
static int oracle_code4(const uint8_t *row, int64_t n)
{
    uint8_t byte = row[n >> 1];
    return (n & 1) ? (byte >> 4) : (byte & 0x0f);
}

/* FP4 E2M1 element -> double (exact).  Bit 3 is the sign, bits 2-1 the
 * exponent e (bias 1), bit 0 the mantissa m.  e = 0 encodes 0 and the one
 * subnormal magnitude 0.5 (m * 2^(1-1) / 2); otherwise the value is
 * 2^(e-1) * (1 + m/2).  The format has no infinity or NaN. */
double oracle_e2m1_to_f64(uint8_t code)
{
    int sign = (code >> 3) & 1;
    int e = (code >> 1) & 3;
    int m = code & 1;
    double mag = (e == 0) ? 0.5 * m : ldexp(1.0 + 0.5 * m, e - 1);
    return sign ? -mag : mag;
}

/* E8M0 shared scale -> double: 2^(E - 127); E = 255 encodes NaN. */
double oracle_e8m0_to_f64(uint8_t e)
{
    return e == 255 ? NAN : ldexp(1.0, (int)e - 127);
}

/* ------------------------------------------------------------------------ */
/* Rounding of a double to the stored output types (round to nearest even). */
/* ------------------------------------------------------------------------ */

float oracle_round_f32(double x)
{
    return (float)x;  /* C conversion in the default rounding mode: RNE */
}

/* Round |x| (finite, non-negative) to an integer multiple of 2^e, ties to
 * even multiple.  Exact in double for the ranges used here. */
static double round_to_multiple(double x, int e)
{
    double scaled = ldexp(x, -e);
    double fl = floor(scaled);
    double rem = scaled - fl;
    if (rem > 0.5 || (rem == 0.5 && fmod(fl, 2.0) != 0.0)) fl += 1.0;
    return ldexp(fl, e);
}

/* double -> binary16 bit pattern, round to nearest even, overflow to inf. */
uint16_t oracle_round_f16(double x)
{
    if (isnan(x)) return 0x7e00;
    uint16_t sign = signbit(x) ? 0x8000 : 0;
    double a = fabs(x);
    if (a == 0.0) return sign;
    int e;
    frexp(a, &e);                  /* a = f * 2^e, f in [0.5, 1) */
    int unbiased = e - 1;          /* a in [2^unbiased, 2^(unbiased+1)) */
    if (unbiased < -14) unbiased = -14;     /* subnormal spacing 2^-24 */
    double r = round_to_multiple(a, unbiased - 10);
    if (r >= 65536.0) return sign | 0x7c00;  /* rounds past the largest */
    if (r < ldexp(1.0, -14)) {               /* subnormal or zero */
        return sign | (uint16_t)ldexp(r, 24);
    }
    int re;
    double f = frexp(r, &re);                /* r = f * 2^re */
    int expo = re - 1 + 15;
    uint16_t mant = (uint16_t)(ldexp(f, 11) - 1024.0);
    return sign | (uint16_t)(expo << 10) | mant;
}

/* double -> bfloat16 bit pattern, round to nearest even, overflow to inf. */
uint16_t oracle_round_bf16(double x)
{
    if (isnan(x)) return 0x7fc0;
    uint16_t sign = signbit(x) ? 0x8000 : 0;
    double a = fabs(x);
    if (a == 0.0) return sign;
    int e;
    frexp(a, &e);
    int unbiased = e - 1;
    if (unbiased < -126) unbiased = -126;    /* subnormal spacing 2^-133 */
    double r = round_to_multiple(a, unbiased - 7);
    /* largest finite bf16 is (2 - 2^-7) * 2^127; the next step is 2^128 */
    if (r >= ldexp(1.0, 128)) return sign | 0x7f80;
    if (r < ldexp(1.0, -126)) {
        return sign | (uint16_t)ldexp(r, 133);
    }
    int re;
    double f = frexp(r, &re);
    int expo = re - 1 + 127;
    uint16_t mant = (uint16_t)(ldexp(f, 8) - 128.0);
    return sign | (uint16_t)(expo << 7) | mant;
}

/* ------------------------------------------------------------------------ */
/* The GEMM definition.  One generic i-k-j loop over exact double operands. */
/* ------------------------------------------------------------------------ */

/* Loaders that widen one stored element of A or B to double. */
typedef double (*load_fn)(const void *base, int64_t row, int64_t col, int64_t ld);

static double load_f32(const void *p, int64_t r, int64_t c, int64_t ld)
{
    return (double)((const float *)p)[r * ld + c];
}
static double load_f16(const void *p, int64_t r, int64_t c, int64_t ld)
{
    return oracle_f16_to_f64(((const uint16_t *)p)[r * ld + c]);
}
static double load_bf16(const void *p, int64_t r, int64_t c, int64_t ld)
{
    return oracle_bf16_to_f64(((const uint16_t *)p)[r * ld + c]);
}

/*
 * C[i][j] = epi(sum_k A[i][k] B[k][j]) in double.  For each row i the row of
 * B values is streamed in order k = 0..K-1 and added into a double row
 * accumulator, so each C[i][j] is the sum in increasing k.  relu != 0 clamps
 * negatives to zero after the sum.
 */
static void gemm_generic(int64_t M, int64_t N, int64_t K,
                         const void *A, int64_t lda, load_fn la,
                         const void *B, int64_t ldb, load_fn lb,
                         double *C, int64_t ldc, int relu)
{
    /* Widen B once; a plain copy, not a reordering of the arithmetic. */
    double *Bd = (double *)malloc(sizeof(double) * (size_t)(K > 0 ? K : 1) * (size_t)(N > 0 ? N : 1));
    for (int64_t k = 0; k < K; ++k)
        for (int64_t j = 0; j < N; ++j)
            Bd[k * N + j] = lb(B, k, j, ldb);

    #pragma omp parallel for schedule(dynamic, 1)
    for (int64_t i = 0; i < M; ++i) {
        double *acc = C + i * ldc;
        for (int64_t j = 0; j < N; ++j) acc[j] = 0.0;
        for (int64_t k = 0; k < K; ++k) {
            double a = la(A, i, k, lda);
            const double *brow = Bd + k * N;
            for (int64_t j = 0; j < N; ++j) acc[j] += a * brow[j];
        }
        if (relu)
            for (int64_t j = 0; j < N; ++j)
                if (acc[j] < 0.0) acc[j] = 0.0;
    }
    free(Bd);
}

/* fp32 operands. */
void oracle_gemm_f32(int64_t M, int64_t N, int64_t K,
                     const float *A, int64_t lda, const float *B, int64_t ldb,
                     double *C, int64_t ldc, int relu)
{
    gemm_generic(M, N, K, A, lda, load_f32, B, ldb, load_f32, C, ldc, relu);
}

/* fp16 operands, given as binary16 bit patterns. */
void oracle_gemm_f16(int64_t M, int64_t N, int64_t K,
                     const uint16_t *A, int64_t lda, const uint16_t *B, int64_t ldb,
                     double *C, int64_t ldc, int relu)
{
    gemm_generic(M, N, K, A, lda, load_f16, B, ldb, load_f16, C, ldc, relu);
}

/* bf16 operands, given as bfloat16 bit patterns. */
void oracle_gemm_bf16(int64_t M, int64_t N, int64_t K,
                      const uint16_t *A, int64_t lda, const uint16_t *B, int64_t ldb,
                      double *C, int64_t ldc, int relu)
{
    gemm_generic(M, N, K, A, lda, load_bf16, B, ldb, load_bf16, C, ldc, relu);
}

/*
 * Explicit dequantisation: W[k][n] = q[k][n] * s[k / group][n], in double
 * (exact: a 4-bit integer times an fp16 value).  Bq is K rows of ldbq bytes;
 * column n of row k sits in byte n/2, low nibble for even n, high nibble for
 * odd n.  scales is (K / group) rows of lds fp16 bit patterns.
 */
void oracle_dequant_w4(int64_t K, int64_t N, const uint8_t *Bq, int64_t ldbq,
                       const uint16_t *scales, int64_t lds, int64_t group,
                       double *W, int64_t ldw)
{
    for (int64_t k = 0; k < K; ++k) {
        const uint8_t *row = Bq + k * ldbq;
        const uint16_t *srow = scales + (k / group) * lds;
        for (int64_t n = 0; n < N; ++n)
            W[k * ldw + n] = (double)oracle_nibble(row, n) * oracle_f16_to_f64(srow[n]);
    }
}

static double load_f64(const void *p, int64_t r, int64_t c, int64_t ld)
{
    return ((const double *)p)[r * ld + c];
}

/* Dequantise, then the plain GEMM with fp16 activations A (M x K). */
void oracle_gemm_w4a16(int64_t M, int64_t N, int64_t K,
                       const uint16_t *A, int64_t lda,
                       const uint8_t *Bq, int64_t ldbq,
                       const uint16_t *scales, int64_t lds, int64_t group,
                       double *C, int64_t ldc, int relu)
{
    double *W = (double *)malloc(sizeof(double) * (size_t)(K > 0 ? K : 1) * (size_t)(N > 0 ? N : 1));
    oracle_dequant_w4(K, N, Bq, ldbq, scales, lds, group, W, N);
    gemm_generic(M, N, K, A, lda, load_f16, W, N, load_f64, C, ldc, relu);
    free(W);
}

/*
 * Explicit dequantisation of FP4 weights: W[k][n] = e2m1(code[k][n]) *
 * e8m0(E[k / block][n]), in double (exact: a 2-significant-bit value times a
 * power of two).  Bq is K rows of ldbq bytes, column n of row k in byte n/2,
 * low nibble for even n.  scales is (K / block) rows of lds E8M0 bytes.
 */
void oracle_dequant_fp4(int64_t K, int64_t N, const uint8_t *Bq, int64_t ldbq,
                        const uint8_t *scales, int64_t lds, int64_t block,
                        double *W, int64_t ldw)
{
    for (int64_t k = 0; k < K; ++k) {
        const uint8_t *row = Bq + k * ldbq;
        const uint8_t *srow = scales + (k / block) * lds;
        for (int64_t n = 0; n < N; ++n)
            W[k * ldw + n] = oracle_e2m1_to_f64((uint8_t)oracle_code4(row, n)) *
                             oracle_e8m0_to_f64(srow[n]);
    }
}

/* Dequantise, then the plain GEMM with bf16 activations A (M x K). */
void oracle_gemm_wfp4(int64_t M, int64_t N, int64_t K,
                      const uint16_t *A, int64_t lda,
                      const uint8_t *Bq, int64_t ldbq,
                      const uint8_t *scales, int64_t lds, int64_t block,
                      double *C, int64_t ldc, int relu)
{
    double *W = (double *)malloc(sizeof(double) * (size_t)(K > 0 ? K : 1) * (size_t)(N > 0 ? N : 1));
    oracle_dequant_fp4(K, N, Bq, ldbq, scales, lds, block, W, N);
    gemm_generic(M, N, K, A, lda, load_bf16, W, N, load_f64, C, ldc, relu);
    free(W);
}

/* Number of threads the OpenMP runtime will use for a parallel loop. */
int oracle_num_threads(void)
{
#ifdef _OPENMP
    return omp_get_max_threads();
#else
    return 1;
#endif
}

/* Array forms of the decode and rounding helpers (elementwise loops). */
void oracle_f16_to_f64_n(const uint16_t *in, double *out, int64_t n)
{
    for (int64_t i = 0; i < n; ++i) out[i] = oracle_f16_to_f64(in[i]);
}
void oracle_bf16_to_f64_n(const uint16_t *in, double *out, int64_t n)
{
    for (int64_t i = 0; i < n; ++i) out[i] = oracle_bf16_to_f64(in[i]);
}
void oracle_round_f16_n(const double *in, uint16_t *out, int64_t n)
{
    for (int64_t i = 0; i < n; ++i) out[i] = oracle_round_f16(in[i]);
}
void oracle_round_bf16_n(const double *in, uint16_t *out, int64_t n)
{
    for (int64_t i = 0; i < n; ++i) out[i] = oracle_round_bf16(in[i]);
}

/* ------------------------------------------------------------------------ */
/* 2:4 structured-sparse A.                                                  */
/* ------------------------------------------------------------------------ */

/*
 * The pages name a structured-sparse GEMM (T.gemm_sp, the 2:4 pattern, in the
 * monitoring-and-debugging paragraph of "使用 Tilelang DSL 开发 GPU/CPU/加速器
 * 高性能内核", blog.hotdry.top) and give no storage format; the library's
 * reading is the usual 2:4 compressed form of a row-major M x K matrix A:
 *   - each row is cut into chunks of 4 consecutive k (chunk c: k in
 *     [4c, 4c + 4)); at most two entries of a chunk are non-zero;
 *   - Ac (M x K/2) holds, for chunk c, its two kept values in positions
 *     2c and 2c + 1 (first, second);
 *   - E (M rows of K/8 bytes) holds a 4-bit code per chunk, chunk c in byte
 *     c / 2 (low nibble for even c, high nibble for odd c); bits 0-1 of the
 *     code give the position inside the chunk of the first kept value, bits
 *     2-3 that of the second.
 * Expansion to the dense matrix, in double: A[i][4c + idx_p] receives
 * Ac[i][2c + p] for p = 0, 1; every other entry is zero.  (A code naming one
 * position twice adds both values there: the plain reading.)  K is a
 * multiple of 4.
 */
void oracle_expand_sp24(int64_t M, int64_t K, const uint16_t *Ac, int64_t ldac,
                        const uint8_t *E, int64_t lde, int bf16, double *A, int64_t lda)
{
    for (int64_t i = 0; i < M; ++i) {
        double *arow = A + i * lda;
        for (int64_t k = 0; k < K; ++k) arow[k] = 0.0;
        for (int64_t c = 0; c < K / 4; ++c) {
            int code = oracle_code4(E + i * lde, c);
            for (int p = 0; p < 2; ++p) {
                int idx = (code >> (2 * p)) & 3;
                uint16_t bits = Ac[i * ldac + 2 * c + p];
                double v = bf16 ? oracle_bf16_to_f64(bits) : oracle_f16_to_f64(bits);
                arow[4 * c + idx] += v;
            }
        }
    }
}

/* Expand A, then the plain GEMM with B (K x N) of the same 16-bit type. */
void oracle_gemm_sp24(int64_t M, int64_t N, int64_t K,
                      const uint16_t *Ac, int64_t ldac, const uint8_t *E, int64_t lde,
                      const uint16_t *B, int64_t ldb, int bf16,
                      double *C, int64_t ldc, int relu)
{
    double *A = (double *)malloc(sizeof(double) * (size_t)(M > 0 ? M : 1) * (size_t)(K > 0 ? K : 1));
    oracle_expand_sp24(M, K, Ac, ldac, E, lde, bf16, A, K);
    gemm_generic(M, N, K, A, K, load_f64, B, ldb, bf16 ? load_bf16 : load_f16, C, ldc, relu);
    free(A);
}

