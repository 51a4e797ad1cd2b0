// abi.cu -- the C ABI of include/tg_gemm.h: argument validation and dispatch.
//
// Every check here runs before any CUDA call, so a rejected call has no side
// effect.  The operation and its conventions are documented in the header.
#include "../../include/tg_gemm.h"
#include "launch.h"
#include "host.cuh"
#include "ptx.cuh"

#include <cuda_runtime.h>

#include <atomic>

namespace tg {

// Per-device status word written by kernels whose bounded wait expired.
__device__ int g_device_status = 0;

int* device_status_ptr() {
    static std::atomic<int*> ptrs[64] = {};
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64) return nullptr;
    int* q = ptrs[dev].load(std::memory_order_acquire);
    if (!q) {
        void* p = nullptr;
        if (cudaGetSymbolAddress(&p, g_device_status) != cudaSuccess) return nullptr;
        q = static_cast<int*>(p);
        ptrs[dev].store(q, std::memory_order_release);   // every thread finds the same address
    }
    return q;
}

}  // namespace tg

namespace {

constexpr int64_t kMaxDim = (1ll << 31) - 1;      // kernel indices and TMA coords are int32

bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

// A row pitch of ld elements of eb bytes that a tensor map can take: TMA
// strides stay below 2^40 bytes.  Checked before any ld * eb product.
bool pitch_ok(int64_t ld, int eb) { return ld < (1ll << 40) / eb; }

// Shared checks for a GEMM with element size `eb` (bytes).  With trans_a
// the stored A is K x M (rows of M), with trans_b the stored B is N x K.
tg_status check_gemm(int64_t M, int64_t N, int64_t K, const void* A, int64_t lda,
                     const void* B, int64_t ldb, const void* C, int64_t ldc,
                     int epilogue, int eb, int trans_a = 0, int trans_b = 0) {
    if (M < 0 || N < 0 || K < 0) return TG_ERR_INVALID_ARG;
    if (epilogue != TG_EPI_NONE && epilogue != TG_EPI_RELU) return TG_ERR_INVALID_ARG;
    if ((trans_a != 0 && trans_a != 1) || (trans_b != 0 && trans_b != 1)) return TG_ERR_INVALID_ARG;
    if (M == 0 || N == 0) return TG_OK;
    if (!C || ldc < N) return TG_ERR_INVALID_ARG;
    if (K > 0 && (!A || !B || lda < (trans_a ? M : K) || ldb < (trans_b ? K : N)))
        return TG_ERR_INVALID_ARG;
    if (M > kMaxDim || N > kMaxDim || K > kMaxDim) return TG_ERR_UNSUPPORTED;
    if (!pitch_ok(ldc, eb) || (K > 0 && (!pitch_ok(lda, eb) || !pitch_ok(ldb, eb))))
        return TG_ERR_UNSUPPORTED;
    if (!aligned16(C) || (ldc * eb) % 16 != 0) return TG_ERR_ALIGNMENT;
    if (K > 0 && (!aligned16(A) || !aligned16(B) || (lda * eb) % 16 != 0 || (ldb * eb) % 16 != 0))
        return TG_ERR_ALIGNMENT;
    return TG_OK;
}

// C = epi(0) = 0 when K == 0.
tg_status zero_fill(void* C, int64_t ldc, int64_t M, int64_t N, int eb, void* stream) {
    int dev;
    if (!tg::current_device(&dev)) return TG_ERR_NO_DEVICE;
    cudaError_t e = cudaMemset2DAsync(C, static_cast<size_t>(ldc * eb), 0,
                                      static_cast<size_t>(N * eb), static_cast<size_t>(M),
                                      static_cast<cudaStream_t>(stream));
    return e == cudaSuccess ? TG_OK : TG_ERR_CUDA;
}

tg::GemmArgs make_args(int64_t M, int64_t N, int64_t K, const void* A, int64_t lda,
                       const void* B, int64_t ldb, void* C, int64_t ldc, int epilogue,
                       void* stream) {
    tg::GemmArgs a;
    a.M = M; a.N = N; a.K = K;
    a.A = A; a.lda = lda; a.B = B; a.ldb = ldb; a.C = C; a.ldc = ldc;
    a.scales = nullptr; a.lds = 0; a.group = 0;
    a.relu = epilogue == TG_EPI_RELU;
    a.stream = stream;
    a.path = a.ctas = a.group_m = a.splits = a.stages = 0;
    return a;
}

}  // namespace

int tg::check_gemm_args(int64_t M, int64_t N, int64_t K, const void* A, int64_t lda,
                        const void* B, int64_t ldb, const void* C, int64_t ldc, int epilogue,
                        int eb) {
    return check_gemm(M, N, K, A, lda, B, ldb, C, ldc, epilogue, eb);
}

extern "C" {

tg_status tg_gemm_f32(int64_t M, int64_t N, int64_t K, const float* A, int64_t lda,
                      const float* B, int64_t ldb, float* C, int64_t ldc, int epilogue,
                      int mode, void* stream) {
    if (mode != TG_F32_FFMA && mode != TG_F32_TF32) return TG_ERR_INVALID_ARG;
    tg_status s = check_gemm(M, N, K, A, lda, B, ldb, C, ldc, epilogue, 4);
    if (s != TG_OK || M == 0 || N == 0) return s;
    if (K == 0) return zero_fill(C, ldc, M, N, 4, stream);
    const tg::GemmArgs a = tg::with_rule(make_args(M, N, K, A, lda, B, ldb, C, ldc, epilogue, stream),
                                         tg::tune_lookup(mode == TG_F32_TF32 ? tg::OP_F32_TF32
                                                                             : tg::OP_F32_FFMA, M, N));
    return static_cast<tg_status>(mode == TG_F32_TF32 ? tg::launch_tc_tf32(a)
                                                      : tg::launch_ffma_f32(a));
}

tg_status tg_gemm_f16(int64_t M, int64_t N, int64_t K, const void* A, int64_t lda,
                      const void* B, int64_t ldb, void* C, int64_t ldc, int epilogue,
                      void* stream) {
    tg_status s = check_gemm(M, N, K, A, lda, B, ldb, C, ldc, epilogue, 2);
    if (s != TG_OK || M == 0 || N == 0) return s;
    if (K == 0) return zero_fill(C, ldc, M, N, 2, stream);
    return static_cast<tg_status>(tg::launch_tc_f16(tg::with_rule(
        make_args(M, N, K, A, lda, B, ldb, C, ldc, epilogue, stream), tg::tune_lookup(tg::OP_F16, M, N))));
}

tg_status tg_gemm_f16_ex(int64_t M, int64_t N, int64_t K, const void* A, int64_t lda, int trans_a,
                         const void* B, int64_t ldb, int trans_b, void* C, int64_t ldc,
                         int epilogue, void* stream) {
    tg_status s = check_gemm(M, N, K, A, lda, B, ldb, C, ldc, epilogue, 2, trans_a, trans_b);
    if (s != TG_OK || M == 0 || N == 0) return s;
    if (K == 0) return zero_fill(C, ldc, M, N, 2, stream);
    tg::GemmArgs a = make_args(M, N, K, A, lda, B, ldb, C, ldc, epilogue, stream);
    if (!trans_a) a = tg::with_rule(a, tg::tune_lookup(tg::OP_F16, M, N));
    return static_cast<tg_status>(tg::launch_tc_trans(a, 0, trans_a, trans_b));
}

tg_status tg_gemm_bf16_ex(int64_t M, int64_t N, int64_t K, const void* A, int64_t lda, int trans_a,
                          const void* B, int64_t ldb, int trans_b, void* C, int64_t ldc,
                          int epilogue, void* stream) {
    tg_status s = check_gemm(M, N, K, A, lda, B, ldb, C, ldc, epilogue, 2, trans_a, trans_b);
    if (s != TG_OK || M == 0 || N == 0) return s;
    if (K == 0) return zero_fill(C, ldc, M, N, 2, stream);
    tg::GemmArgs a = make_args(M, N, K, A, lda, B, ldb, C, ldc, epilogue, stream);
    if (!trans_a) a = tg::with_rule(a, tg::tune_lookup(tg::OP_BF16, M, N));
    return static_cast<tg_status>(tg::launch_tc_trans(a, 1, trans_a, trans_b));
}

tg_status tg_gemm_bf16(int64_t M, int64_t N, int64_t K, const void* A, int64_t lda,
                       const void* B, int64_t ldb, void* C, int64_t ldc, int epilogue,
                       void* stream) {
    tg_status s = check_gemm(M, N, K, A, lda, B, ldb, C, ldc, epilogue, 2);
    if (s != TG_OK || M == 0 || N == 0) return s;
    if (K == 0) return zero_fill(C, ldc, M, N, 2, stream);
    return static_cast<tg_status>(tg::launch_tc_bf16(tg::with_rule(
        make_args(M, N, K, A, lda, B, ldb, C, ldc, epilogue, stream), tg::tune_lookup(tg::OP_BF16, M, N))));
}

tg_status tg_gemm_w4a16(int64_t M, int64_t N, int64_t K, const void* A, int64_t lda,
                        const uint8_t* Bq, int64_t ldbq, const void* scales, int64_t lds,
                        int group_size, void* C, int64_t ldc, int epilogue, void* stream) {
    if (M < 0 || N < 0 || K < 0) return TG_ERR_INVALID_ARG;
    if (epilogue != TG_EPI_NONE && epilogue != TG_EPI_RELU) return TG_ERR_INVALID_ARG;
    if (group_size != 128 || K % 128 != 0) return TG_ERR_UNSUPPORTED;
    if (M == 0 || N == 0) return TG_OK;
    if (!C || ldc < N) return TG_ERR_INVALID_ARG;
    if (K > 0 && (!A || !Bq || !scales || lda < K || ldbq < (N + 1) / 2 || lds < N))
        return TG_ERR_INVALID_ARG;
    if (M > kMaxDim || N > kMaxDim || K > kMaxDim) return TG_ERR_UNSUPPORTED;
    if (!pitch_ok(ldc, 2) ||
        (K > 0 && (!pitch_ok(lda, 2) || !pitch_ok(ldbq, 1) || !pitch_ok(lds, 2))))
        return TG_ERR_UNSUPPORTED;
    if (!aligned16(C) || (ldc * 2) % 16 != 0) return TG_ERR_ALIGNMENT;
    if (K > 0 && (!aligned16(A) || !aligned16(Bq) || !aligned16(scales) || (lda * 2) % 16 != 0 ||
                  ldbq % 16 != 0 || (lds * 2) % 16 != 0))
        return TG_ERR_ALIGNMENT;
    if (K == 0) return zero_fill(C, ldc, M, N, 2, stream);
    tg::GemmArgs a = tg::with_rule(make_args(M, N, K, A, lda, Bq, ldbq, C, ldc, epilogue, stream),
                                   tg::tune_lookup(tg::OP_W4A16, M, N));
    a.scales = scales;
    a.lds = lds;
    a.group = group_size;
    return static_cast<tg_status>(tg::launch_w4a16(a));
}

tg_status tg_gemm_wfp4(int64_t M, int64_t N, int64_t K, const void* A, int64_t lda,
                       const uint8_t* Bq, int64_t ldbq, const uint8_t* scales, int64_t lds,
                       int block_size, void* C, int64_t ldc, int epilogue, void* stream) {
    if (M < 0 || N < 0 || K < 0) return TG_ERR_INVALID_ARG;
    if (epilogue != TG_EPI_NONE && epilogue != TG_EPI_RELU) return TG_ERR_INVALID_ARG;
    if (block_size != 32) return TG_ERR_UNSUPPORTED;
    if (M == 0 || N == 0) return TG_OK;
    if (!C || ldc < N) return TG_ERR_INVALID_ARG;
    if (K > 0 && (!A || !Bq || !scales || lda < K || ldbq < (N + 1) / 2 || lds < N))
        return TG_ERR_INVALID_ARG;
    if (M > kMaxDim || N > kMaxDim || K > kMaxDim) return TG_ERR_UNSUPPORTED;
    if (!pitch_ok(ldc, 2) ||
        (K > 0 && (!pitch_ok(lda, 2) || !pitch_ok(ldbq, 1) || !pitch_ok(lds, 1))))
        return TG_ERR_UNSUPPORTED;
    if (!aligned16(C) || (ldc * 2) % 16 != 0) return TG_ERR_ALIGNMENT;
    if (K > 0 && (!aligned16(A) || !aligned16(Bq) || !aligned16(scales) || (lda * 2) % 16 != 0 ||
                  ldbq % 16 != 0 || lds % 16 != 0))
        return TG_ERR_ALIGNMENT;
    if (K == 0) return zero_fill(C, ldc, M, N, 2, stream);
    tg::GemmArgs a = tg::with_rule(make_args(M, N, K, A, lda, Bq, ldbq, C, ldc, epilogue, stream),
                                   tg::tune_lookup(tg::OP_WFP4, M, N));
    a.scales = scales;
    a.lds = lds;
    a.group = block_size;
    return static_cast<tg_status>(tg::launch_wfp4(a));
}

namespace {

// 2:4 sparse A: Ac (M x K/2 values), E (M x ceil(K/8) code bytes), B (K x N).
tg_status sp24(int64_t M, int64_t N, int64_t K, const void* Ac, int64_t ldac, const uint8_t* E,
               int64_t lde, const void* B, int64_t ldb, void* C, int64_t ldc, int epilogue,
               void* stream, int bf16) {
    if (M < 0 || N < 0 || K < 0) return TG_ERR_INVALID_ARG;
    if (epilogue != TG_EPI_NONE && epilogue != TG_EPI_RELU) return TG_ERR_INVALID_ARG;
    if (K % 4 != 0) return TG_ERR_UNSUPPORTED;
    if (M == 0 || N == 0) return TG_OK;
    if (!C || ldc < N) return TG_ERR_INVALID_ARG;
    if (K > 0 && (!Ac || !E || !B || ldac < K / 2 || lde < (K + 7) / 8 || ldb < N))
        return TG_ERR_INVALID_ARG;
    if (M > kMaxDim || N > kMaxDim || K > kMaxDim) return TG_ERR_UNSUPPORTED;
    if (!pitch_ok(ldc, 2) ||
        (K > 0 && (!pitch_ok(ldac, 2) || !pitch_ok(lde, 1) || !pitch_ok(ldb, 2))))
        return TG_ERR_UNSUPPORTED;
    if (!aligned16(C) || (ldc * 2) % 16 != 0) return TG_ERR_ALIGNMENT;
    if (K > 0 && (!aligned16(Ac) || !aligned16(E) || !aligned16(B) || (ldac * 2) % 16 != 0 ||
                  lde % 16 != 0 || (ldb * 2) % 16 != 0))
        return TG_ERR_ALIGNMENT;
    if (K == 0) return zero_fill(C, ldc, M, N, 2, stream);
    const tg::GemmArgs a = make_args(M, N, K, Ac, ldac, B, ldb, C, ldc, epilogue, stream);
    return static_cast<tg_status>(tg::launch_sp24(a, E, lde, bf16));
}

}  // namespace

tg_status tg_gemm_sp24_f16(int64_t M, int64_t N, int64_t K, const void* Ac, int64_t ldac,
                           const uint8_t* E, int64_t lde, const void* B, int64_t ldb, void* C,
                           int64_t ldc, int epilogue, void* stream) {
    return sp24(M, N, K, Ac, ldac, E, lde, B, ldb, C, ldc, epilogue, stream, 0);
}

tg_status tg_gemm_sp24_bf16(int64_t M, int64_t N, int64_t K, const void* Ac, int64_t ldac,
                            const uint8_t* E, int64_t lde, const void* B, int64_t ldb, void* C,
                            int64_t ldc, int epilogue, void* stream) {
    return sp24(M, N, K, Ac, ldac, E, lde, B, ldb, C, ldc, epilogue, stream, 1);
}

const char* tg_status_string(tg_status s) {
    switch (s) {
        case TG_OK: return "TG_OK";
        case TG_ERR_INVALID_ARG: return "TG_ERR_INVALID_ARG";
        case TG_ERR_ALIGNMENT: return "TG_ERR_ALIGNMENT";
        case TG_ERR_UNSUPPORTED: return "TG_ERR_UNSUPPORTED";
        case TG_ERR_CUDA: return "TG_ERR_CUDA";
        case TG_ERR_TIMEOUT: return "TG_ERR_TIMEOUT";
        case TG_ERR_NO_DEVICE: return "TG_ERR_NO_DEVICE";
    }
    return "TG_ERR_UNKNOWN";
}

tg_status tg_last_device_status(void* stream) {
    if (cudaStreamSynchronize(static_cast<cudaStream_t>(stream)) != cudaSuccess) return TG_ERR_CUDA;
    int v = 0;
    const int zero = 0;
    if (cudaMemcpyFromSymbol(&v, tg::g_device_status, sizeof v) != cudaSuccess) return TG_ERR_CUDA;
    if (v != 0 && cudaMemcpyToSymbol(tg::g_device_status, &zero, sizeof zero) != cudaSuccess)
        return TG_ERR_CUDA;
    if (v == TG_ERR_TIMEOUT) {
        int dev = 0;
        if (cudaGetDevice(&dev) == cudaSuccess) tg::mark_workspaces_dirty(dev);
    }
    return static_cast<tg_status>(v);
}

int tg_num_sms(void) {
    int dev;
    const tg::DeviceInfo* d = tg::current_device(&dev);
    return d ? d->num_sms : -1;
}

}  // extern "C"
