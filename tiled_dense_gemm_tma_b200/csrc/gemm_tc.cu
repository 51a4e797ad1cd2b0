// gemm_tc.cu -- launcher for the tensor-core GEMM (fp16, bf16, TF32 mode).
#include "gemm_tc.cuh"
#include "gemm_tc2.cuh"
#include "host.cuh"
#include "launch.h"

namespace tg {

namespace {

using CfgBF16 = TcCfg<2, 1, OutT::BF16, 256, 4>;
using CfgF16 = TcCfg<2, 0, OutT::F16, 256, 4>;
using CfgTF32 = TcCfg<4, 2, OutT::F32, 256, 4>;
using Cfg2BF16 = Tc2Cfg<1, OutT::BF16, 6>;
using Cfg2F16 = Tc2Cfg<0, OutT::F16, 6>;
// a 4-slot ring, one of the ring depths the tuning table can choose
using Cfg2BF16s4 = Tc2Cfg<1, OutT::BF16, 4>;
using Cfg2F16s4 = Tc2Cfg<0, OutT::F16, 4>;
// transposed operands (A stored K x M and/or B stored N x K)
template <int FMT, OutT OUT>
using Cfg2T10 = Tc2Cfg<FMT, OUT, 6, 1, 1>;
template <int FMT, OutT OUT>
using Cfg2T01 = Tc2Cfg<FMT, OUT, 6, 0, 0>;
template <int FMT, OutT OUT>
using Cfg2T11 = Tc2Cfg<FMT, OUT, 6, 1, 0>;
// Operand-swapped CTA pair for M <= 128 (C^T = B^T A^T, 128-column pair tiles,
// written transposed): B^T arrives from B stored K x N (MN-major) or N x K
// (K-major); A^T is A stored M x K, read K-major.
template <int FMT, OutT OUT>
using Cfg2S = Tc2Cfg<FMT, OUT, 6, 1, 0, 128, 1>;
template <int FMT, OutT OUT>
using Cfg2ST = Tc2Cfg<FMT, OUT, 6, 0, 0, 128, 1>;
// TF32 mode on CTA pairs (M > 128)
using Cfg2TF32 = Tc2Cfg<2, OutT::F32, 6>;

template <class Cfg>
int run(const GemmArgs& a, CUtensorMapDataType in_t, CUtensorMapDataType out_t, int slot) {
    int dev = 0;
    const DeviceInfo* di = current_device(&dev);
    if (!di) return kNoDevice;
    CUtensorMap tA, tB, tC;
    // A: K-major boxes of BK (128 B) x BM rows.
    if (!tensor_map_2d(&tA, a.A, in_t, Cfg::IN_BYTES, a.K, a.M, a.lda * Cfg::IN_BYTES,
                       Cfg::BK, Cfg::BM, SWZ_128))
        return kCudaError;
    // B: N-major boxes of CHUNK_N (128 B) x BK rows.
    if (!tensor_map_2d(&tB, a.B, in_t, Cfg::IN_BYTES, a.N, a.K, a.ldb * Cfg::IN_BYTES,
                       Cfg::CHUNK_N, Cfg::BK, Cfg::IN_BYTES == 4 ? SWZ_128_32B : SWZ_128))
        return kCudaError;
    // C: 32-row staging boxes of CW (128 B) columns.
    if (!tensor_map_2d(&tC, a.C, out_t, Cfg::OUT_BYTES, a.N, a.M, a.ldc * Cfg::OUT_BYTES,
                       Cfg::CW, 32, SWZ_128))
        return kCudaError;
    auto kern = tc_gemm_kernel<Cfg>;
    if (set_smem_attr(reinterpret_cast<const void*>(kern), Cfg::SMEM_BYTES, slot) != cudaSuccess)
        return kCudaError;
    const long long ntm = (a.M + Cfg::BM - 1) / Cfg::BM;
    const long long ntn = (a.N + Cfg::BN - 1) / Cfg::BN;
    const long long tiles = ntm * ntn;
    const int grid = static_cast<int>(persistent_grid(tiles, di->num_sms, a.ctas));
    TcParams p = {};
    p.M = static_cast<int>(a.M);
    p.N = static_cast<int>(a.N);
    p.K = static_cast<int>(a.K);
    p.relu = a.relu;
    p.group_m = a.group_m > 0 ? a.group_m : Cfg::GROUP_M;
    p.inject = inject_mode();
    p.timeout_ns = wait_limit_ns();
    p.status = device_status_ptr();
    p.C = a.C;
    p.ldc = a.ldc;
    p.tail_split = 1;
    p.dp_tiles = 0;
    p.tickets = nullptr;
    p.ws = nullptr;
    if (!p.status) return kCudaError;
    kern<<<grid, Cfg::THREADS, Cfg::SMEM_BYTES, static_cast<cudaStream_t>(a.stream)>>>(tA, tB, tC, p);
    return cudaGetLastError() == cudaSuccess ? kOk : kCudaError;
}

// CTA-pair kernel: 256 x 256 tiles on clusters of two CTAs.  Returns
// kUnsupported (nothing launched) if the device refuses the cluster launch.
template <class Cfg>
int run_pair(const GemmArgs& a, CUtensorMapDataType dt, int slot) {
    if (pair_kernels_disabled()) return kUnsupported;
    int dev = 0;
    const DeviceInfo* di = current_device(&dev);
    if (!di) return kNoDevice;
    CUtensorMap tA, tB, tC;
    constexpr int eb = Cfg::IN_BYTES, ob = Cfg::OUT_BYTES;
    const CUtensorMapDataType ot = Cfg::OUT == OutT::F32 ? CU_TENSOR_MAP_DATA_TYPE_FLOAT32 : dt;
    // A: row-major M x K -> K-major boxes of BK (128 B) x BM rows; stored
    // transposed (K x M) -> M-major boxes of 64 rows of A x BK.
    if (Cfg::A_MN ? !tensor_map_2d(&tA, a.A, dt, eb, a.M, a.K, a.lda * eb, 64, Cfg::BK, SWZ_128)
                  : !tensor_map_2d(&tA, a.A, dt, eb, a.K, a.M, a.lda * eb, Cfg::BK, Cfg::BM, SWZ_128))
        return kCudaError;
    // B: row-major K x N -> N-major boxes of CHUNK_N (128 B) columns x BK
    // (32-bit data with the 32-byte-unit swizzle); stored transposed (N x K)
    // -> K-major boxes of BK x HN columns.
    if (Cfg::B_MN ? !tensor_map_2d(&tB, a.B, dt, eb, a.N, a.K, a.ldb * eb, Cfg::CHUNK_N, Cfg::BK,
                                   eb == 4 ? SWZ_128_32B : SWZ_128)
                  : !tensor_map_2d(&tB, a.B, dt, eb, a.K, a.N, a.ldb * eb, Cfg::BK, Cfg::HN, SWZ_128))
        return kCudaError;
    // C: 128-byte x 32-row boxes of the tile; in the operand-swapped mode the
    // kernel's M x N is C^T, and C (a.N rows x a.M columns) takes unswizzled
    // boxes of 32 columns x 64 rows
    if (Cfg::TOUT ? !tensor_map_2d(&tC, a.C, ot, ob, a.M, a.N, a.ldc * ob, 32, 64, SWZ_NONE)
                  : !tensor_map_2d(&tC, a.C, ot, ob, a.N, a.M, a.ldc * ob, 128 / ob, 32, SWZ_128))
        return kCudaError;
    auto kern = tc2_gemm_kernel<Cfg>;
    if (set_smem_attr(reinterpret_cast<const void*>(kern), Cfg::SMEM_BYTES, slot) != cudaSuccess)
        return kCudaError;
    const long long tiles = ((a.M + Cfg::PM - 1) / Cfg::PM) * ((a.N + Cfg::BN - 1) / Cfg::BN);
    const int npairs = static_cast<int>(persistent_grid(tiles, di->num_sms / 2, a.ctas));
    // hybrid schedule: the tiles of a thin last wave split in two along K,
    // their halves meeting through the stream's workspace
    const int num_kb = static_cast<int>((a.K + Cfg::BK - 1) / Cfg::BK);
    int S = tiles < 0x7fffffffll ? tail_split(static_cast<int>(tiles), npairs, num_kb) : 1;
    int dp = tail_dp(static_cast<int>(tiles), npairs, S);
    int* tickets = nullptr;
    float* ws = nullptr;
    if (S > 1) {
        const long long R = tiles - dp;
        if (!stream_workspace(dev, a.stream, R * 4, R * 2 * Cfg::BM * Cfg::BN * 4, &tickets, &ws)) {
            // no workspace (a stream under graph capture that has none yet,
            // or no memory): the last wave runs whole tiles
            cudaGetLastError();
            S = 1;
            dp = static_cast<int>(tiles);
            tickets = nullptr;
            ws = nullptr;
        }
    }
    TcParams p;
    p.M = static_cast<int>(a.M);
    p.N = static_cast<int>(a.N);
    p.K = static_cast<int>(a.K);
    p.relu = a.relu;
    p.group_m = a.group_m > 0 ? a.group_m : Cfg::GROUP_M;
    p.inject = inject_mode();
    p.timeout_ns = wait_limit_ns();
    p.status = device_status_ptr();
    p.C = a.C;
    p.ldc = a.ldc;
    p.tail_split = S;
    p.dp_tiles = dp;
    p.tickets = tickets;
    p.ws = ws;
    if (!p.status) return kCudaError;
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3(2 * npairs, 1, 1);
    cfg.blockDim = dim3(Cfg::THREADS, 1, 1);
    cfg.dynamicSmemBytes = Cfg::SMEM_BYTES;
    cfg.stream = static_cast<cudaStream_t>(a.stream);
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeClusterDimension;
    attr[0].val.clusterDim.x = 2;
    attr[0].val.clusterDim.y = 1;
    attr[0].val.clusterDim.z = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    cudaError_t e = cudaLaunchKernelEx(&cfg, kern, tA, tB, tC, p);
    if (e != cudaSuccess) {
        cudaGetLastError();                       // clear; caller falls back
        return kUnsupported;
    }
    return kOk;
}

}  // namespace

// The CTA-pair kernel for M <= 128 with the operands swapped: the kernel's
// A is B^T (its M = N) and its B is A^T (its N = M); C is written transposed
// back.  trans_b: B is stored N x K.
template <int FMT, OutT OUT>
int run_pair_swapped(const GemmArgs& a, CUtensorMapDataType dt, int trans_b, int slot) {
    GemmArgs s = a;
    s.M = a.N;
    s.N = a.M;
    s.A = a.B;
    s.lda = a.ldb;
    s.B = a.A;
    s.ldb = a.lda;
    return trans_b ? run_pair<Cfg2ST<FMT, OUT>>(s, dt, slot + 1) : run_pair<Cfg2S<FMT, OUT>>(s, dt, slot);
}

// The tuning rule's path (a.path) wins; by default M <= 4 takes the CUDA-core
// kernel, M <= 128 the weight-streaming kernel, larger M the CTA-pair kernel
// (operand-swapped for M <= 128; the one-CTA kernel if a cluster launch is
// refused).
int launch_tc_bf16(const GemmArgs& a) {
    int path = a.path;
    if (path == PATH_AUTO)
        path = a.M <= kGemvMaxM ? PATH_CUDA_CORE : a.M <= kSkinnyMaxM ? PATH_SMALL_M : PATH_CTA_PAIR;
    if (path == PATH_CUDA_CORE) return launch_gemv_bf16(a);
    if (path == PATH_SMALL_M) return launch_skinny_bf16(a);
    if (path == PATH_CTA_PAIR) {
        const int r = a.M <= kSkinnyMaxM ? run_pair_swapped<1, OutT::BF16>(a, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 0, 64)
                    : a.stages == 4      ? run_pair<Cfg2BF16s4>(a, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 54)
                                         : run_pair<Cfg2BF16>(a, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3);
        if (r != kUnsupported) return r;
    }
    return run<CfgBF16>(a, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 0);
}
int launch_tc_f16(const GemmArgs& a) {
    int path = a.path;
    if (path == PATH_AUTO)
        path = a.M <= kGemvMaxM ? PATH_CUDA_CORE : a.M <= kSkinnyMaxM ? PATH_SMALL_M : PATH_CTA_PAIR;
    if (path == PATH_CUDA_CORE) return launch_gemv_f16(a);
    if (path == PATH_SMALL_M) return launch_skinny_f16(a);
    if (path == PATH_CTA_PAIR) {
        const int r = a.M <= kSkinnyMaxM ? run_pair_swapped<0, OutT::F16>(a, CU_TENSOR_MAP_DATA_TYPE_FLOAT16, 0, 66)
                    : a.stages == 4      ? run_pair<Cfg2F16s4>(a, CU_TENSOR_MAP_DATA_TYPE_FLOAT16, 55)
                                         : run_pair<Cfg2F16>(a, CU_TENSOR_MAP_DATA_TYPE_FLOAT16, 4);
        if (r != kUnsupported) return r;
    }
    return run<CfgF16>(a, CU_TENSOR_MAP_DATA_TYPE_FLOAT16, CU_TENSOR_MAP_DATA_TYPE_FLOAT16, 1);
}
// 16-bit GEMM with optionally transposed operands.  Only B transposed (the
// backward product dA = dC . B^T) follows the plain call's path choice: with
// M <= 128 and the small-M or CUDA-core path it runs the weight-streaming
// kernel on K-major weight tiles (there is no transposed CUDA-core kernel),
// with another path the operand-swapped CTA-pair kernel.  Every other
// transposed call runs the CTA-pair kernel (no one-CTA variant: a refused
// cluster launch reports kUnsupported).
int launch_tc_trans(const GemmArgs& a, int bf16, int trans_a, int trans_b) {
    if (!trans_a && !trans_b) return bf16 ? launch_tc_bf16(a) : launch_tc_f16(a);
    if (!trans_a && a.M <= kSkinnyMaxM && a.path != PATH_CTA_PAIR && a.path != PATH_ONE_CTA)
        return launch_skinny_trans_b(a, bf16);
    if (!trans_a && a.M <= kSkinnyMaxM)
        return bf16 ? run_pair_swapped<1, OutT::BF16>(a, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 1, 64)
                    : run_pair_swapped<0, OutT::F16>(a, CU_TENSOR_MAP_DATA_TYPE_FLOAT16, 1, 66);
    const CUtensorMapDataType dt = bf16 ? CU_TENSOR_MAP_DATA_TYPE_BFLOAT16 : CU_TENSOR_MAP_DATA_TYPE_FLOAT16;
    if (bf16) {
        if (trans_a && trans_b) return run_pair<Cfg2T11<1, OutT::BF16>>(a, dt, 11);
        return trans_a ? run_pair<Cfg2T10<1, OutT::BF16>>(a, dt, 12) : run_pair<Cfg2T01<1, OutT::BF16>>(a, dt, 13);
    }
    if (trans_a && trans_b) return run_pair<Cfg2T11<0, OutT::F16>>(a, dt, 14);
    return trans_a ? run_pair<Cfg2T10<0, OutT::F16>>(a, dt, 15) : run_pair<Cfg2T01<0, OutT::F16>>(a, dt, 5);
}

// TF32 mode: M > 128 on CTA pairs by default (the one-CTA kernel if a
// cluster launch is refused); M <= 128, or a one-CTA tuning rule, on the
// one-CTA kernel.
int launch_tc_tf32(const GemmArgs& a) {
    int path = a.path;
    if (path == PATH_AUTO) path = a.M <= kSkinnyMaxM ? PATH_ONE_CTA : PATH_CTA_PAIR;
    if (path == PATH_CTA_PAIR) {
        const int r = run_pair<Cfg2TF32>(a, CU_TENSOR_MAP_DATA_TYPE_FLOAT32, 68);
        if (r != kUnsupported) return r;
    }
    return run<CfgTF32>(a, CU_TENSOR_MAP_DATA_TYPE_FLOAT32, CU_TENSOR_MAP_DATA_TYPE_FLOAT32, 2);
}

}  // namespace tg
