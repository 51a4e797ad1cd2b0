/*
 * tg_gemm.h -- C ABI of the tiled dense GEMM library for one NVIDIA B200.
 *
 * Operation (every entry point):
 *
 *     C[i][j] = epi( sum_{k<K} A[i][k] * B[k][j] ),   0 <= i < M, 0 <= j < N
 *
 * with A (M x K), B (K x N) and C (M x N) all ROW-MAJOR, i.e. element (r, c)
 * of a matrix with leading dimension ld lives at base[r * ld + c].  This is
 * the tiled matrix multiply of "TileLang ... 高效 GEMM 内核" (mhpq.cn),
 * section 3.2 (C = A x B, A M x K, B K x N, fp32, caller-allocated C) and
 * section 2.1 (tiling rationale); the row-major default is stated on the
 * gtnt.cn TileLang tutorial, section 4.3; epi is the identity or the ReLU
 * output post-processing of the blog.hotdry.top TileLang guide (landing
 * checklist, item 2).  C is overwritten (no alpha/beta, no accumulation).
 * Products are accumulated in fp32; the result is rounded once to C's type
 * with round-to-nearest-even after epi is applied.
 *
 * Conventions shared by all entry points
 * --------------------------------------
 * - Pointers are DEVICE pointers (cudaMalloc / torch CUDA memory) on the
 *   current CUDA device.  The caller owns every buffer.  C must not overlap
 *   A, B or the scales (not checked).
 * - Leading dimensions are in elements (in bytes for packed 4-bit weights,
 *   E8M0 scale bytes and 2:4 position codes), and must be >= the row length.
 * - stream is a cudaStream_t passed as void*; NULL means the legacy default
 *   stream.  Calls are asynchronous: they validate, enqueue and return.
 * - Sizes: M, N, K >= 0.  M == 0 or N == 0 -> TG_OK, nothing is launched.
 *   K == 0 -> C = epi(0) = 0 is written.  M, N, K above 2^31 - 1, or a row
 *   pitch (ld * sizeof(element)) of 2^40 bytes or more -> TG_ERR_UNSUPPORTED
 *   (the limits of the kernels' 32-bit indices and of a TMA stride).
 * - Alignment (the hardware tensor-copy engine, TMA, needs 16-byte aligned
 *   bases and row pitches): every base pointer 16-byte aligned and every
 *   ld * sizeof(element) a multiple of 16 bytes, else TG_ERR_ALIGNMENT.
 * - Errors are returned, never printed or thrown.  Validation happens
 *   before any CUDA call; on any error nothing is launched and C is untouched.
 * - The library allocates no per-call memory.  It keeps, per device and for
 *   the life of the process, a small status word (see
 *   tg_last_device_status), a cache of tensor-copy descriptors, and one
 *   split-K workspace per (device, stream): fp32 partials and tile tickets
 *   of the kernels that split K across CTAs through global memory (small M
 *   where the split does not run inside thread-block clusters, fp32 shapes
 *   with fewer 128 x 128 tiles than SMs, and 16-bit GEMMs on the CTA-pair
 *   kernel whose last wave of tiles is split along K).  It is allocated on
 *   the first such call on a stream (at least 8 MiB), grown when a larger
 *   call needs it (the regrow frees the old one, which synchronises the
 *   device), and reused.  Calls on one stream share it; calls on different
 *   streams get their own (cudaStreamPerThread counts as one stream per
 *   host thread).  A stream under CUDA graph capture never allocates it:
 *   there the 16-bit GEMM on the CTA-pair kernel runs its last wave of
 *   tiles whole, and the other users of the workspace return TG_ERR_CUDA
 *   unless one uncaptured call of the largest shape on that stream came
 *   first.  tg_gemm_bf16_small_m_static avoids it.
 * - Thread safety: calls from several host threads are allowed.  A thread
 *   needs no earlier CUDA call: on its first call the library makes the
 *   current device's primary context current on that thread.
 */
#ifndef TG_GEMM_H
#define TG_GEMM_H

#include <stdint.h>

#if defined(__GNUC__)
#define TG_API __attribute__((visibility("default")))
#else
#define TG_API
#endif

#ifdef __cplusplus
extern "C" {
#endif

typedef enum {
    TG_OK = 0,
    TG_ERR_INVALID_ARG = 1,  /* negative size, NULL pointer, ld < row length, bad flag */
    TG_ERR_ALIGNMENT = 2,    /* base not 16-byte aligned or row pitch not a multiple of 16 bytes */
    TG_ERR_UNSUPPORTED = 3,  /* 4-bit group / block size other than 128 / 32, K not a multiple of
                                the group, size limit */
    TG_ERR_CUDA = 4,         /* a CUDA runtime / driver call or the launch failed */
    TG_ERR_TIMEOUT = 5,      /* a kernel's bounded wait expired (reported by tg_last_device_status) */
    TG_ERR_NO_DEVICE = 6     /* no sm_100 device is current */
} tg_status;

/* Epilogue flags (the `epilogue` argument). */
enum { TG_EPI_NONE = 0, TG_EPI_RELU = 1 };

/* fp32 modes (the `mode` argument of tg_gemm_f32). */
enum {
    TG_F32_FFMA = 0,  /* exact fp32 products, fp32 FMA accumulation on CUDA cores */
    TG_F32_TF32 = 1   /* operands rounded to TF32 (10-bit mantissa) by the tensor
                         cores, fp32 accumulation in tensor memory; M > 128 on
                         CTA pairs (256 x 256 tiles), M <= 128 (or a refused
                         cluster launch) on one CTA per SM (128 x 256 tiles) */
};

/*
 * tg_gemm_f32 -- fp32 GEMM (mhpq.cn article, section 3.2: float32 A, B, C,
 * 128 x 128 x 32 tiles, 256 threads; section 3.3: float4 vector loads).
 *   A: M x K floats, row pitch lda (>= K, lda % 4 == 0)
 *   B: K x N floats, row pitch ldb (>= N, ldb % 4 == 0)
 *   C: M x N floats, row pitch ldc (>= N, ldc % 4 == 0); written
 *   epilogue: TG_EPI_NONE or TG_EPI_RELU; mode: TG_F32_FFMA or TG_F32_TF32
 */
TG_API tg_status tg_gemm_f32(int64_t M, int64_t N, int64_t K,
                      const float *A, int64_t lda,
                      const float *B, int64_t ldb,
                      float *C, int64_t ldc,
                      int epilogue, int mode, void *stream);

/*
 * tg_gemm_f16 -- fp16 operands and output, fp32 accumulation (explicit cast
 * to float16, gtnt.cn tutorial section 4.3; FP16 GEMM on the blog.hotdry.top
 * guide).  A, B, C hold IEEE binary16 values (e.g. __half or torch.float16);
 * every ld must be a multiple of 8 elements.  Other arguments as tg_gemm_f32.
 */
TG_API tg_status tg_gemm_f16(int64_t M, int64_t N, int64_t K,
                      const void *A, int64_t lda,
                      const void *B, int64_t ldb,
                      void *C, int64_t ldc,
                      int epilogue, void *stream);

/* tg_gemm_bf16 -- as tg_gemm_f16 with bfloat16 operands and output. */
TG_API tg_status tg_gemm_bf16(int64_t M, int64_t N, int64_t K,
                       const void *A, int64_t lda,
                       const void *B, int64_t ldb,
                       void *C, int64_t ldc,
                       int epilogue, void *stream);

/*
 * tg_gemm_f16_ex, tg_gemm_bf16_ex -- C = epi(op(A) . op(B)) with optionally
 * transposed operands, as the backward products of a linear layer need them
 * (dA = dC . B^T, dB = A^T . dC; the autograd wrapper of the mhpq.cn article,
 * section 3.4).  C is M x N row-major as in tg_gemm_f16.
 *   trans_a = 0: A is M x K, row pitch lda >= K;  trans_a = 1: A is stored
 *                K x M (op(A) = A^T), row pitch lda >= M.
 *   trans_b = 0: B is K x N, row pitch ldb >= N;  trans_b = 1: B is stored
 *                N x K (op(B) = B^T), row pitch ldb >= K.
 * trans flags other than 0 / 1 -> TG_ERR_INVALID_ARG.  With both flags 0
 * this is tg_gemm_f16 / tg_gemm_bf16.  A call with only B transposed takes
 * the kernel family that the plain call's tuning rule (tg_tune_rule, op
 * TG_OP_F16 / TG_OP_BF16) picks for its M and N: with M <= 128 and the
 * small-M or CUDA-core path, the weight-streaming small-M kernel on K-major
 * weight tiles; otherwise the CTA-pair kernel.  Every other transposed call
 * runs the CTA-pair tensor-core kernel.  A refused cluster launch of the
 * CTA-pair kernel returns TG_ERR_UNSUPPORTED.
 * Same alignment, status and ownership rules as tg_gemm_f16.
 */
TG_API tg_status tg_gemm_f16_ex(int64_t M, int64_t N, int64_t K,
                         const void *A, int64_t lda, int trans_a,
                         const void *B, int64_t ldb, int trans_b,
                         void *C, int64_t ldc,
                         int epilogue, void *stream);
TG_API tg_status tg_gemm_bf16_ex(int64_t M, int64_t N, int64_t K,
                          const void *A, int64_t lda, int trans_a,
                          const void *B, int64_t ldb, int trans_b,
                          void *C, int64_t ldc,
                          int epilogue, void *stream);

/*
 * tg_gemm_w4a16 -- dequantize GEMM (the "Dequant GEMM" workload of the
 * blog.hotdry.top TileLang guide; the pages give no format, this library
 * defines it):  C = epi(A . W) with
 *
 *     W[k][n] = fp16( q[k][n] * s[k / group_size][n] )
 *
 *   A:      M x K fp16 activations, row pitch lda (elements, % 8 == 0)
 *   Bq:     K rows of packed signed 4-bit weights q in [-8, 7], two's
 *           complement, two per byte: column 2j in bits 0-3 and column 2j+1
 *           in bits 4-7 of byte j of the row.  Row pitch ldbq in BYTES
 *           (>= ceil(N/2), % 16 == 0).
 *   scales: ceil(K / group_size) x N fp16 scales, row pitch lds (elements,
 *           % 8 == 0).
 *   group_size: must be 128, and K must be a multiple of it, else
 *           TG_ERR_UNSUPPORTED.
 *   C:      M x N fp16 output, row pitch ldc (elements, % 8 == 0).
 * The dequantised weight is formed as an fp32 product rounded once to fp16
 * (so it equals the exact product rounded to fp16), then used as an fp16
 * tensor-core operand with fp32 accumulation.
 */
TG_API tg_status tg_gemm_w4a16(int64_t M, int64_t N, int64_t K,
                        const void *A, int64_t lda,
                        const uint8_t *Bq, int64_t ldbq,
                        const void *scales, int64_t lds, int group_size,
                        void *C, int64_t ldc,
                        int epilogue, void *stream);

/*
 * tg_gemm_wfp4 -- FP4-weight GEMM ("WFP4", the low-precision GEMM of the
 * performance section, 性能表现与基准测试验证, of "TileLang架构深度剖析"
 * (test.krestaai.com.au); the pages give no format, this library reads it
 * as the MXFP4 weights of the OCP Microscaling Formats (MX) specification
 * v1.0 with bf16 activations):  C = epi(A . W) with
 *
 *     W[k][n] = e2m1(code[k][n]) * 2^(E[k / 32][n] - 127)
 *
 *   A:      M x K bf16 activations, row pitch lda (elements, % 8 == 0)
 *   Bq:     K rows of E2M1 codes, two per byte: column 2j in bits 0-3 and
 *           column 2j+1 in bits 4-7 of byte j.  A code is a sign (bit 3), a
 *           2-bit exponent with bias 1 (bits 2-1) and a mantissa bit (bit 0):
 *           magnitudes 0, 0.5, 1, 1.5, 2, 3, 4, 6.  Row pitch ldbq in BYTES
 *           (>= ceil(N/2), % 16 == 0).
 *   scales: ceil(K / 32) x N E8M0 bytes E (the scale 2^(E - 127); E = 255
 *           means NaN), row pitch lds in BYTES (>= N, % 16 == 0).
 *   block_size: must be 32 (k rows per scale), else TG_ERR_UNSUPPORTED.
 *   C:      M x N bf16 output, row pitch ldc (elements, % 8 == 0).
 * Any K >= 0.  For M > 4, W is formed exactly as a bf16 tensor-core
 * operand (for E <= 252; a larger E overflows bf16); for M <= 4 the CUDA-core
 * kernel multiplies the exact E2M1 values by the activations in fp32 and
 * applies each 32-row block's 2^(E - 127) once per block and column.  Either
 * way products accumulate in fp32 and the result is rounded once to bf16.
 * Same status and ownership rules as tg_gemm_w4a16.
 */
TG_API tg_status tg_gemm_wfp4(int64_t M, int64_t N, int64_t K,
                       const void *A, int64_t lda,
                       const uint8_t *Bq, int64_t ldbq,
                       const uint8_t *scales, int64_t lds, int block_size,
                       void *C, int64_t ldc,
                       int epilogue, void *stream);

/*
 * tg_gemm_sp24_f16, tg_gemm_sp24_bf16 -- 2:4 structured-sparse GEMM (the
 * structured-sparse T.gemm_sp with the 2:4 pattern of the blog.hotdry.top
 * TileLang guide, monitoring-and-debugging paragraph; the pages give no
 * format, this library defines it):  C = epi(A . B) where A (M x K) keeps at
 * most two non-zeros in every chunk of 4 consecutive k of a row and is
 * passed compressed:
 *   Ac:  M x K/2 fp16 / bf16 values, row pitch ldac (elements, % 8 == 0):
 *        the two kept values of chunk c (k in [4c, 4c + 4)) at columns 2c
 *        and 2c + 1, the first before the second.
 *   E:   M rows of ceil(K/8) code bytes, row pitch lde in BYTES (% 16 == 0):
 *        a 4-bit code per chunk, chunk c in byte c/2 (low nibble for even c);
 *        bits 0-1 give the position (0-3) inside the chunk of the first kept
 *        value, bits 2-3 that of the second.  Positions should be distinct
 *        (a chunk with fewer non-zeros keeps zeros at unused positions).
 *   B:   K x N dense, row pitch ldb (elements, % 8 == 0); C: M x N, ldc.
 * K must be a multiple of 4 (else TG_ERR_UNSUPPORTED).  Runs on the sparse
 * tensor cores (tcgen05.mma.sp) with fp32 accumulation and one rounding of
 * each result to C's type.  Same status and ownership rules as
 * tg_gemm_f16.
 */
TG_API tg_status tg_gemm_sp24_f16(int64_t M, int64_t N, int64_t K,
                           const void *Ac, int64_t ldac,
                           const uint8_t *E, int64_t lde,
                           const void *B, int64_t ldb,
                           void *C, int64_t ldc,
                           int epilogue, void *stream);
TG_API tg_status tg_gemm_sp24_bf16(int64_t M, int64_t N, int64_t K,
                            const void *Ac, int64_t ldac,
                            const uint8_t *E, int64_t lde,
                            const void *B, int64_t ldb,
                            void *C, int64_t ldc,
                            int epilogue, void *stream);

/*
 * tg_gemm_bf16_small_m_static -- tg_gemm_bf16 for M <= 128 that never
 * allocates device memory.  The pages have no counterpart: this entry point
 * exists for callers that may not call cudaMalloc / cudaFree where they run
 * the GEMM (a memory pool that already holds the device's free memory, or a
 * latency-critical loop that must stay out of the driver's allocator).
 *
 * Same arguments, semantics and alignment rules as tg_gemm_bf16; M must be
 * <= 128 (else TG_ERR_UNSUPPORTED).  It always runs the small-M tensor-core
 * kernel (tg_gemm_bf16 takes a CUDA-core kernel for M <= 4), with the same
 * plan as tg_gemm_bf16 on all SMs.  Shapes whose split-K runs inside
 * thread-block clusters need no scratch.  For the others the split-K
 * scratch lives in a fixed device array of 16 MiB of fp32 partials plus 4096
 * tile tickets that is part of the library image; shapes needing more return
 * TG_ERR_UNSUPPORTED.  Every call shares that array (tickets are cleared at
 * the start of each call): calls that overlap on the GPU, e.g. on two
 * streams, race and give wrong results -- serialise them.  The first call on
 * each device looks up the array's device address (cudaGetSymbolAddress) and
 * how many clusters of the kernel the device holds at once, and caches both;
 * make that first call before any stream capture.
 */
TG_API tg_status tg_gemm_bf16_small_m_static(int64_t M, int64_t N, int64_t K,
                                             const void *A, int64_t lda,
                                             const void *B, int64_t ldb,
                                             void *C, int64_t ldc,
                                             int epilogue, void *stream);

/*
 * Tuning table.  Every call picks its kernel family and launch shape from a
 * table of rules keyed by operation and by ranges of M and N, the kernels
 * being compiled ahead of time (this stands in for the parameter-space
 * search of the pages' autotuner: "TileLang架构深度剖析", 自动调优系统; the
 * tuning configuration of the gtnt.cn tutorial, section 3.3).  The built-in
 * rules are written by the offline sweep `python bench.py --sweep`, which
 * times the choices below on the device; rules installed with tg_tune_set
 * are consulted before them.  The first rule with the call's op whose
 * [m_lo, m_hi] holds M and [n_lo, n_hi] holds N applies; a field left 0
 * keeps the library's default.  Transposed-operand calls, the fp32 FFMA
 * kernel's tile shape and tg_gemm_bf16_small_m_static ignore the table.
 */
enum {
    TG_OP_BF16 = 0, TG_OP_F16 = 1, TG_OP_W4A16 = 2, TG_OP_WFP4 = 3,
    TG_OP_F32_FFMA = 4, TG_OP_F32_TF32 = 5
};
enum {
    TG_PATH_AUTO = 0,       /* the default choice by M */
    TG_PATH_CUDA_CORE = 1,  /* CUDA-core kernel: M <= 4 only; not for fp32 */
    TG_PATH_SMALL_M = 2,    /* weight-streaming tensor-core kernel: M <= 128 only */
    TG_PATH_CTA_PAIR = 3,   /* persistent CTA-pair tensor-core kernel (16-bit, 4-bit and
                               TF32 ops; 16-bit calls with M <= 128 run it with the
                               operands swapped, C^T = B^T A^T, and C written
                               transposed) */
    TG_PATH_ONE_CTA = 4     /* persistent one-CTA tensor-core kernel (not fp32 FFMA) */
};
typedef struct {
    int32_t op;             /* TG_OP_* */
    int32_t path;           /* TG_PATH_*; must serve op and every M of the rule */
    int64_t m_lo, m_hi;     /* inclusive range of M (>= 1) */
    int64_t n_lo, n_hi;     /* inclusive range of N (>= 1) */
    int32_t ctas;           /* persistent CTAs (CTA pairs for TG_PATH_CTA_PAIR); the
                               stream-K split of the small-M and CUDA-core kernels;
                               capped at the device's SMs; 0 = all */
    int32_t group_m;        /* raster band height in (pair) tiles, 1..256; 0 = default */
    int32_t splits;         /* TG_OP_F32_FFMA only: k ranges per output tile, 1..8 */
    int32_t stages;         /* 16-bit CTA-pair kernel with M > 128 only: ring depth, 4 or 6 */
} tg_tune_rule;

/* Replace the run-time rules with `count` rules (at most 64; 0 clears them).
 * A malformed rule -> TG_ERR_INVALID_ARG and the previous rules stay.  The
 * rules apply to calls made after this returns, from any thread. */
TG_API tg_status tg_tune_set(const tg_tune_rule *rules, int count);

/* Copy up to `capacity` built-in rules to `out`; returns how many exist. */
TG_API int tg_tune_builtin(tg_tune_rule *out, int capacity);

/* The rule a call of operation `op` with these M and N would use (a rule of
 * zero fields when none covers it); no CUDA call. */
TG_API tg_status tg_tune_query(int op, int64_t M, int64_t N, tg_tune_rule *out);

/* Human-readable name of a status code (static storage, never NULL). */
TG_API const char *tg_status_string(tg_status s);

/*
 * tg_last_device_status -- synchronises `stream`, then reads and clears the
 * current device's status word.  Kernels never spin forever: every wait on
 * a pipeline barrier has a time limit (4 s of device time by default), and a
 * kernel that hits it records TG_ERR_TIMEOUT there and returns early (C is
 * then incomplete).
 * Returns TG_OK, TG_ERR_TIMEOUT, or TG_ERR_CUDA if synchronising failed.
 */
TG_API tg_status tg_last_device_status(void *stream);

/*
 * tg_num_sms -- number of SMs of the current device (what the persistent
 * kernels size their grids by), or -1 on error.
 */
TG_API int tg_num_sms(void);

#ifdef __cplusplus
}
#endif

#endif /* TG_GEMM_H */
