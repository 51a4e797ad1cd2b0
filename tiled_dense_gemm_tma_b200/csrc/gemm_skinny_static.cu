// gemm_skinny_static.cu -- tg_gemm_bf16_small_m_static: the small-M bf16 GEMM
// (the weight-streaming kernel of gemm_skinny.cuh) with its scratch memory in
// a fixed array of device memory that is part of the library image, so a call
// never allocates.  Shapes whose split-K runs inside clusters need no scratch
// at all; the others use the array for their stream-K partials.
//
// Who needs this: code that may not call cudaMalloc / cudaFree at the point
// where it runs the GEMM -- for example a program whose memory pool has
// already reserved the device's free memory (a new cudaMalloc there fails or
// steals from the pool), or a latency-critical loop that must not enter the
// driver's allocator (cudaMalloc can take milliseconds and cudaFree waits for
// the whole device).  The regular tg_gemm_bf16 allocates its workspace once
// per stream on first use; this entry point never does.
//
// Limits and sharing:
// - Scratch: kStaticPartialFloats fp32 partials (16 MiB) and kStaticTickets
//   (4096) tile tickets.  The CUDA runtime places the arrays in device memory
//   of every GPU on which this part of the library is loaded (at the latest
//   on the first call there) and keeps them until the process exits.  Shapes
//   that take stream-K and whose partials or tiles exceed that return
//   TG_ERR_UNSUPPORTED.
// - Every call uses the same array.  Tickets are cleared at the start of each
//   call; partials are overwritten before they are read.  Calls that overlap
//   on the GPU (different streams, or different host threads on one device)
//   race on the array and give wrong results: serialise them.
// - Set-up: the first call on each device looks up the array's device address
//   with cudaGetSymbolAddress (the array's name in host code is only a host
//   stand-in) and how many clusters of the kernel the device holds at once
//   (cudaOccupancyMaxActiveClusters), and caches both; make that first call
//   before any stream capture.
#include "gemm_skinny.cuh"
#include "host.cuh"
#include "launch.h"
#include "../../include/tg_gemm.h"

#include <cstring>
#include <mutex>

namespace tg {

namespace {

constexpr long long kStaticPartialFloats = 4ll << 20;     // 16 MiB of fp32 partials
constexpr long long kStaticTickets = 4096;

static __device__ __align__(256) float g_static_partials[kStaticPartialFloats];
static __device__ __align__(256) int g_static_tickets[kStaticTickets];

constexpr int kMaxDevs = 64;
float* g_part_ptr[kMaxDevs];
int* g_tick_ptr[kMaxDevs];
std::once_flag g_setup_once[kMaxDevs];
cudaError_t g_setup_err[kMaxDevs];

// Device addresses of the two arrays for device `dev` (which is current).
bool static_scratch(int dev, float** part, int** tick) {
    std::call_once(g_setup_once[dev], [dev] {
        void* p = nullptr;
        void* t = nullptr;
        cudaError_t e = cudaGetSymbolAddress(&p, g_static_partials);
        if (e == cudaSuccess) e = cudaGetSymbolAddress(&t, g_static_tickets);
        g_setup_err[dev] = e;
        g_part_ptr[dev] = static_cast<float*>(p);
        g_tick_ptr[dev] = static_cast<int*>(t);
    });
    if (g_setup_err[dev] != cudaSuccess || !g_part_ptr[dev] || !g_tick_ptr[dev]) return false;
    *part = g_part_ptr[dev];
    *tick = g_tick_ptr[dev];
    return true;
}

// A tensor map encoded directly (no cache insertion, so no host allocation).
typedef CUresult (*EncodeFn)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*,
                             const cuuint64_t*, const cuuint64_t*, const cuuint32_t*,
                             const cuuint32_t*, CUtensorMapInterleave, CUtensorMapSwizzle,
                             CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

bool encode_map(CUtensorMap* m, const void* base, uint64_t cols, uint64_t rows,
                uint64_t ld_bytes, uint32_t box_cols, uint32_t box_rows) {
    static EncodeFn fn = [] {
        void* f = nullptr;
        cudaDriverEntryPointQueryResult q;
        if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &f, cudaEnableDefault, &q) !=
                cudaSuccess || q != cudaDriverEntryPointSuccess)
            return static_cast<EncodeFn>(nullptr);
        return reinterpret_cast<EncodeFn>(f);
    }();
    if (!fn) return false;
    cuuint64_t dims[2] = {cols < 1 ? 1 : cols, rows < 1 ? 1 : rows};
    cuuint64_t strides[1] = {ld_bytes};
    cuuint32_t box[2] = {box_cols, box_rows};
    cuuint32_t estr[2] = {1, 1};
    std::memset(m, 0, sizeof *m);
    return fn(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, const_cast<void*>(base), dims, strides, box,
              estr, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
              CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) ==
           CUDA_SUCCESS;
}

template <int MPAD>
tg_status run_static(int64_t M, int64_t N, int64_t K, const void* A, int64_t lda,
                     const void* B, int64_t ldb, void* C, int64_t ldc, int relu,
                     void* stream, const DeviceInfo* di, int dev) {
    using Cfg = SkCfg<WKind::BF16, MPAD>;
    SkPlan pl;
    if (!sk_plan(N, K, Cfg::GN, Cfg::BK, di->num_sms, &pl)) return TG_ERR_UNSUPPORTED;
    auto kern = skinny_kernel<Cfg>;
    const int slot = 50 + (MPAD == 16 ? 0 : MPAD == 32 ? 1 : MPAD == 64 ? 2 : 3);
    if (set_smem_attr(reinterpret_cast<const void*>(kern), Cfg::SMEM_BYTES, slot) != cudaSuccess)
        return TG_ERR_CUDA;
    // the plan of tg_gemm_bf16 on all SMs: split-K inside clusters (no
    // scratch) where that fills the GPU, else stream-K over the fixed arrays
    const int S = skinny_cluster_split<Cfg>(pl.T, pl.KB, di->num_sms, di->num_sms, slot);
    const long long T = pl.T, KB = pl.KB, U = pl.U, J = pl.J;
    const long long G = S ? T * S : pl.G;
    float* part = nullptr;
    int* tick = nullptr;
    cudaStream_t s = static_cast<cudaStream_t>(stream);
    if (!S) {
        if (T > kStaticTickets || T * J * MPAD * Cfg::GN > kStaticPartialFloats)
            return TG_ERR_UNSUPPORTED;                 // beyond the fixed scratch size
        if (!static_scratch(dev, &part, &tick)) return TG_ERR_CUDA;
        if (cudaMemsetAsync(tick, 0, static_cast<size_t>(T) * sizeof(int), s) != cudaSuccess)
            return TG_ERR_CUDA;
    }
    CUtensorMap tW, tX;
    if (!encode_map(&tW, B, N, K, ldb * 2, 64, Cfg::BK)) return TG_ERR_CUDA;
    if (!encode_map(&tX, A, K, M, lda * 2, 64, MPAD)) return TG_ERR_CUDA;
    SkParams p;
    p.M = static_cast<int>(M);
    p.N = static_cast<int>(N);
    p.K = static_cast<int>(K);
    p.relu = relu;
    p.T = static_cast<int>(T);
    p.KB = static_cast<int>(KB);
    p.U = static_cast<int>(U);
    p.J = static_cast<int>(J);
    p.S = S;
    p.inject = 0;
    p.timeout_ns = wait_limit_ns();
    p.status = device_status_ptr();
    p.C = C;
    p.ldc = ldc;
    p.ws = part;
    p.tickets = tick;
    if (!p.status) return TG_ERR_CUDA;
    return skinny_launch<Cfg>(G, S, s, tW, tW, tX, p) == cudaSuccess ? TG_OK : TG_ERR_CUDA;
}

}  // namespace

}  // namespace tg

extern "C" tg_status tg_gemm_bf16_small_m_static(int64_t M, int64_t N, int64_t K, const void* A,
                                                 int64_t lda, const void* B, int64_t ldb, void* C,
                                                 int64_t ldc, int epilogue, void* stream) {
    // the checks of every other entry point (sizes, pointers, leading
    // dimensions, row-pitch bound, alignment), before any CUDA call
    const tg_status s = static_cast<tg_status>(
        tg::check_gemm_args(M, N, K, A, lda, B, ldb, C, ldc, epilogue, 2));
    if (s != TG_OK || M == 0 || N == 0) return s;
    if (M > 128) return TG_ERR_UNSUPPORTED;            // the small-M kernel's limit
    int dev = 0;
    const tg::DeviceInfo* di = tg::current_device(&dev);
    if (!di || dev >= tg::kMaxDevs) return TG_ERR_NO_DEVICE;
    if (K == 0)                                        // C = epi(0) = 0
        return cudaMemset2DAsync(C, static_cast<size_t>(ldc * 2), 0, static_cast<size_t>(N * 2),
                                 static_cast<size_t>(M), static_cast<cudaStream_t>(stream)) ==
                       cudaSuccess ? TG_OK : TG_ERR_CUDA;
    const int relu = epilogue == TG_EPI_RELU;
    if (M <= 16) return tg::run_static<16>(M, N, K, A, lda, B, ldb, C, ldc, relu, stream, di, dev);
    if (M <= 32) return tg::run_static<32>(M, N, K, A, lda, B, ldb, C, ldc, relu, stream, di, dev);
    if (M <= 64) return tg::run_static<64>(M, N, K, A, lda, B, ldb, C, ldc, relu, stream, di, dev);
    return tg::run_static<128>(M, N, K, A, lda, B, ldb, C, ldc, relu, stream, di, dev);
}
