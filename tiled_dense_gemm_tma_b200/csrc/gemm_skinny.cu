// gemm_skinny.cu -- launchers of the weight-streaming (small-M) kernel, for
// B stored K x N (the plain call) or N x K (a transposed-B call).  Split-K
// runs inside clusters where that fills the GPU; otherwise stream-K, whose
// partials and tile tickets live in the per-stream workspace (workspace.cu).
#include "gemm_skinny.cuh"
#include "host.cuh"
#include "launch.h"

namespace tg {

namespace {

template <WKind W, int MPAD, int WK>
int run(const GemmArgs& a) {
    using Cfg = SkCfg<W, MPAD, WK>;
    int dev = 0;
    const DeviceInfo* di = current_device(&dev);
    if (!di) return kNoDevice;
    const long long cap = persistent_grid(di->num_sms, di->num_sms, a.ctas);
    SkPlan pl;
    if (!sk_plan(a.N, a.K, Cfg::GN, Cfg::BK, static_cast<int>(cap), &pl)) return kUnsupported;
    auto kern = skinny_kernel<Cfg>;
    const int mi = MPAD == 16 ? 0 : MPAD == 32 ? 1 : MPAD == 64 ? 2 : 3;
    const int slot = W == WKind::FP4 ? 36 + mi
                   : WK ? 28 + static_cast<int>(W) * 4 + mi : 16 + static_cast<int>(W) * 4 + mi;
    if (set_smem_attr(reinterpret_cast<const void*>(kern), Cfg::SMEM_BYTES, slot) != cudaSuccess)
        return kCudaError;
    // split-K inside clusters where T groups x a small split fill the GPU
    // (no workspace, no tickets), else stream-K over the stream's workspace
    const int S = skinny_cluster_split<Cfg>(pl.T, pl.KB, cap, di->num_sms, slot);
    const long long T = pl.T, KB = pl.KB, U = pl.U, J = pl.J;
    const long long G = S ? T * S : pl.G;
    int* tickets = nullptr;
    float* ws = nullptr;
    if (!S && !stream_workspace(dev, a.stream, T, T * J * MPAD * Cfg::GN * 4, &tickets, &ws))
        return kCudaError;

    CUtensorMap tW, tS, tX;
    if constexpr (Cfg::Q4) {
        if (!tensor_map_2d(&tW, a.B, CU_TENSOR_MAP_DATA_TYPE_UINT8, 1, (a.N + 1) / 2, a.K, a.ldb,
                           Cfg::GN / 2, Cfg::BK, SWZ_128))
            return kCudaError;
        if constexpr (Cfg::FP4) {
            // E8M0 bytes: ceil(K / 32) rows of N; two rows (64 k) per unit
            if (!tensor_map_2d(&tS, a.scales, CU_TENSOR_MAP_DATA_TYPE_UINT8, 1, a.N, (a.K + 31) / 32,
                               a.lds, Cfg::GN, Cfg::BK / 32, SWZ_NONE))
                return kCudaError;
        } else {
            if (!tensor_map_2d(&tS, a.scales, CU_TENSOR_MAP_DATA_TYPE_FLOAT16, 2, a.N, a.K / 128,
                               a.lds * 2, Cfg::GN, 1, SWZ_NONE))
                return kCudaError;
        }
    } else if constexpr (WK) {
        // B stored N x K: boxes of 64 k x the tile's 128 stored rows
        const CUtensorMapDataType dt = W == WKind::BF16 ? CU_TENSOR_MAP_DATA_TYPE_BFLOAT16
                                                         : CU_TENSOR_MAP_DATA_TYPE_FLOAT16;
        if (!tensor_map_2d(&tW, a.B, dt, 2, a.K, a.N, a.ldb * 2, 64, Cfg::TN, SWZ_128))
            return kCudaError;
        tS = tW;                                   // unused
    } else {
        const CUtensorMapDataType dt = W == WKind::BF16 ? CU_TENSOR_MAP_DATA_TYPE_BFLOAT16
                                                         : CU_TENSOR_MAP_DATA_TYPE_FLOAT16;
        if (!tensor_map_2d(&tW, a.B, dt, 2, a.N, a.K, a.ldb * 2, 64, Cfg::BK, SWZ_128))
            return kCudaError;
        tS = tW;                                   // unused
    }
    const CUtensorMapDataType xt = Cfg::OUTW == WKind::BF16 ? CU_TENSOR_MAP_DATA_TYPE_BFLOAT16
                                                            : CU_TENSOR_MAP_DATA_TYPE_FLOAT16;
    if (!tensor_map_2d(&tX, a.A, xt, 2, a.K, a.M, a.lda * 2, 64, MPAD, SWZ_128))
        return kCudaError;

    SkParams p;
    p.M = static_cast<int>(a.M);
    p.N = static_cast<int>(a.N);
    p.K = static_cast<int>(a.K);
    p.relu = a.relu;
    p.T = static_cast<int>(T);
    p.KB = static_cast<int>(KB);
    p.U = static_cast<int>(U);
    p.J = static_cast<int>(J);
    p.S = S;
    p.inject = inject_mode();
    p.timeout_ns = wait_limit_ns();
    p.status = device_status_ptr();
    p.C = a.C;
    p.ldc = a.ldc;
    p.ws = ws;
    p.tickets = tickets;
    if (!p.status) return kCudaError;
    return skinny_launch<Cfg>(G, S, static_cast<cudaStream_t>(a.stream), tW, tS, tX, p) == cudaSuccess
               ? kOk : kCudaError;
}

template <WKind W, int WK = 0>
int dispatch(const GemmArgs& a) {
    if (a.M <= 16) return run<W, 16, WK>(a);
    if (a.M <= 32) return run<W, 32, WK>(a);
    if (a.M <= 64) return run<W, 64, WK>(a);
    return run<W, 128, WK>(a);
}

}  // namespace

int launch_skinny_bf16(const GemmArgs& a) { return dispatch<WKind::BF16>(a); }
int launch_skinny_f16(const GemmArgs& a) { return dispatch<WKind::F16>(a); }
int launch_skinny_w4a16(const GemmArgs& a) { return dispatch<WKind::INT4>(a); }
int launch_skinny_wfp4(const GemmArgs& a) { return dispatch<WKind::FP4>(a); }
int launch_skinny_trans_b(const GemmArgs& a, int bf16) {
    return bf16 ? dispatch<WKind::BF16, 1>(a) : dispatch<WKind::F16, 1>(a);
}

}  // namespace tg
