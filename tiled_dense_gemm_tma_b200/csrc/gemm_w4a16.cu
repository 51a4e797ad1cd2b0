// gemm_w4a16.cu -- dequantize GEMM C = epi(A . W) with fp16 activations A
// (M x K, row-major) and 4-bit weights W = fp16(q * s) (see dequant.cuh),
// fp32 accumulation in tensor memory, fp16 output; and the same kernel for
// FP4 weights (E2M1 codes with E8M0 block scales, bf16 activations, W formed
// exactly in bf16, bf16 output).  One CTA per 128 x 256 tile: the large-M
// path when a CTA-pair launch is refused (gemm_w4a16_pair.cu is the default);
// small M goes to the weight-streaming kernel (gemm_skinny.cu).
//
// The unpack and group scale are fused into operand staging:
//   warp 0      TMA producer: per K slice (BK = 64) loads the A box (BM x 64
//               fp16, K-major, 128-byte swizzle), the packed weight box
//               (64 rows x BN/2 bytes) and the slice's scale row (BN fp16)
//               into a RAW_STAGES-deep ring.
//   warps 6-13  converters: expand the packed slice into the fp16 N-major
//               swizzled B tile of a B_STAGES-deep ring (dequant_slice).
//   warp 1      MMA issuer: tcgen05.mma kind::f16 from the A box and the
//               converted B tile into a double-buffered TMEM accumulator;
//               commits release the raw slot (with the converters'
//               arrivals) and the B tile.
//   warps 2-5   epilogue, as in the tensor-core GEMM, undoing the converter's
//               column order inside 8-column groups.
#include "gemm_tc.cuh"
#include "dequant.cuh"
#include "host.cuh"
#include "launch.h"

namespace tg {

namespace {

struct W4 {
    static constexpr int BM = 128, BN = 256, BK = 64;
    static constexpr int RAW_STAGES = 4, B_STAGES = 3;
    static constexpr int A_BYTES = BM * BK * 2;          // 16 KB
    static constexpr int Q_BYTES = BK * BN / 2;          // 8 KB
    static constexpr int S_BYTES = BN * 2;               // 512 B
    static constexpr int B_CHUNK = BK * 128;             // 8 KB: 64 columns x BK rows
    static constexpr int B_BYTES = (BN / 64) * B_CHUNK;  // 32 KB
    static constexpr int STG_BUF = 32 * 128;
    static constexpr int EPI_WARPS = 4, CONV_WARPS = 8;
    static constexpr int THREADS = 32 * (2 + EPI_WARPS + CONV_WARPS);
    static constexpr int TMEM_COLS = 2 * BN;
    static constexpr int GROUP_M = 16;
    // the scale ring is padded to 1 KB so the swizzled staging after it
    // stays 1024-byte aligned
    static constexpr int S_RING = (RAW_STAGES * S_BYTES + 1023) / 1024 * 1024;
    static constexpr int SMEM_DATA = RAW_STAGES * (A_BYTES + Q_BYTES) + S_RING +
                                     B_STAGES * B_BYTES + EPI_WARPS * STG_BUF;
    static constexpr int SMEM_BYTES = SMEM_DATA + 256 + 1024;
    // Layout guards: A, converted B and the staging (128-byte swizzle) and
    // the packed ring (its TMA boxes) start on 1024-byte boundaries; the
    // barriers, TMEM slot and abort flag fit their 256 bytes; one CTA fits
    // the 227 KB limit; the epilogue has one staging buffer per warp.
    static_assert(A_BYTES % 1024 == 0 && B_BYTES % 1024 == 0 && B_CHUNK % 1024 == 0, "swizzle");
    static_assert((RAW_STAGES * A_BYTES + B_STAGES * B_BYTES) % 1024 == 0, "packed ring alignment");
    static_assert((RAW_STAGES * Q_BYTES) % 1024 == 0 && S_RING % 1024 == 0, "staging alignment");
    static_assert((2 * RAW_STAGES + 2 * B_STAGES + 5) * 8 + 8 <= 256, "barrier area");
    static_assert(SMEM_BYTES <= 227 * 1024, "shared memory per CTA");
    static_assert(TMEM_COLS == 512, "TMEM: two 256-column accumulators");
};

// QFP4 = false: signed 4-bit weights with fp16 group scales, fp16
// activations and output; true: FP4 (E2M1) weights with E8M0 block scales,
// bf16 activations and output (dequant.cuh).
template <bool QFP4>
__global__ void __launch_bounds__(W4::THREADS, 1)
w4a16_gemm_kernel(const __grid_constant__ CUtensorMap tmA,
                  const __grid_constant__ CUtensorMap tmQ,
                  const __grid_constant__ CUtensorMap tmS,
                  const __grid_constant__ CUtensorMap tmC,
                  const TcParams p) {
    extern __shared__ uint8_t smem_raw[];
    const uint32_t raw_addr = smem_u32(smem_raw);
    uint8_t* smem = smem_raw + (((raw_addr + 1023u) & ~1023u) - raw_addr);
    uint8_t* smA = smem;
    uint8_t* smB = smA + W4::RAW_STAGES * W4::A_BYTES;
    uint8_t* smQ = smB + W4::B_STAGES * W4::B_BYTES;
    uint8_t* smS = smQ + W4::RAW_STAGES * W4::Q_BYTES;
    uint8_t* smStg = smS + W4::S_RING;
    uint64_t* bars = reinterpret_cast<uint64_t*>(smStg + W4::EPI_WARPS * W4::STG_BUF);
    uint64_t* full = bars;                               // [RAW_STAGES] TMA landed
    uint64_t* rempty = full + W4::RAW_STAGES;            // [RAW_STAGES] converters + MMA done
    uint64_t* bfull = rempty + W4::RAW_STAGES;           // [B_STAGES] converted
    uint64_t* bempty = bfull + W4::B_STAGES;             // [B_STAGES] MMA done
    uint64_t* tfull = bempty + W4::B_STAGES;             // [2]
    uint64_t* tempty = tfull + 2;                        // [2]
    uint64_t* drain = tempty + 2;
    uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(drain + 1);
    volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_slot + 1);

    const int warp = threadIdx.x >> 5;
    const int lane = threadIdx.x & 31;
    const int ntm = (p.M + W4::BM - 1) / W4::BM;
    const int ntn = (p.N + W4::BN - 1) / W4::BN;
    const int num_tiles = ntm * ntn;
    const int num_kb = (p.K + W4::BK - 1) / W4::BK;      // past K: zero-filled codes and activations
    const uint64_t limit = p.timeout_ns;

    if (threadIdx.x == 0) {
        for (int s = 0; s < W4::RAW_STAGES; ++s) {
            mbar_init(&full[s], 1);
            mbar_init(&rempty[s], W4::CONV_WARPS + 1);
        }
        for (int s = 0; s < W4::B_STAGES; ++s) {
            mbar_init(&bfull[s], W4::CONV_WARPS);
            mbar_init(&bempty[s], 1);
        }
        for (int a = 0; a < 2; ++a) { mbar_init(&tfull[a], 1); mbar_init(&tempty[a], W4::EPI_WARPS); }
        mbar_init(drain, 1);
        *abort_flag = 0;
        fence_mbar_init();
        fence_proxy_async_smem();
    }
    if (warp == 1) {
        tmem_alloc(tmem_slot, W4::TMEM_COLS);
        tmem_relinquish();
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem_base = *tmem_slot;

    if (warp == 0) {
        // ------------------------------------------------------ TMA producer
        if (elect_one()) {
            tma_prefetch_desc(&tmA);
            tma_prefetch_desc(&tmQ);
            tma_prefetch_desc(&tmS);
            tma_prefetch_desc(&tmC);
            uint32_t armed = 0, armed_par = 0, it = 0;
            bool ok = true;
            for (int t = blockIdx.x; t < num_tiles && ok; t += gridDim.x) {
                int tm, tn;
                tile_coords(t, ntm, ntn, p.group_m, tm, tn);
                for (int kb = 0; kb < num_kb; ++kb, ++it) {
                    const uint32_t s = it % W4::RAW_STAGES;
                    const uint32_t ph = (it / W4::RAW_STAGES) & 1;
                    if (!bounded_wait(&rempty[s], ph ^ 1, abort_flag, limit, p.status)) { ok = false; break; }
                    if (p.inject == 1 && it == 0 && blockIdx.x == 0) continue;   // debug: never arm slot 0
                    mbar_arrive_expect_tx(&full[s], W4::A_BYTES + W4::Q_BYTES + W4::S_BYTES);
                    armed |= 1u << s;
                    armed_par = (armed_par & ~(1u << s)) | (ph << s);
                    tma_load_2d(smA + s * W4::A_BYTES, &tmA, &full[s], kb * W4::BK, tm * W4::BM);
                    tma_load_2d(smQ + s * W4::Q_BYTES, &tmQ, &full[s], tn * (W4::BN / 2), kb * W4::BK);
                    tma_load_2d(smS + s * W4::S_BYTES, &tmS, &full[s], tn * W4::BN,
                                (kb * W4::BK) / (QFP4 ? 32 : 128));
                }
            }
            if (!ok) {
                for (int s = 0; s < W4::RAW_STAGES; ++s)
                    if (armed & (1u << s)) {
                        volatile int never = 0;
                        bounded_wait(&full[s], (armed_par >> s) & 1, &never, limit, p.status);
                    }
            }
        }
        __syncwarp();
    } else if (warp == 1) {
        // ------------------------------------------------------- MMA issuer
        if (elect_one()) {
            constexpr uint32_t idesc = make_idesc(QFP4 ? 1 : 0, W4::BM, W4::BN, 0, 1);
            uint32_t it = 0, tl = 0;
            bool ok = true;
            for (int t = blockIdx.x; t < num_tiles && ok; t += gridDim.x, ++tl) {
                const uint32_t acc = tl & 1;
                const uint32_t aph = (tl >> 1) & 1;
                if (!bounded_wait(&tempty[acc], aph ^ 1, abort_flag, limit, p.status)) { ok = false; break; }
                tc_fence_after();
                const uint32_t d_tmem = tmem_base + acc * W4::BN;
                for (int kb = 0; kb < num_kb; ++kb, ++it) {
                    const uint32_t s = it % W4::RAW_STAGES;
                    const uint32_t ph = (it / W4::RAW_STAGES) & 1;
                    const uint32_t b = it % W4::B_STAGES;
                    const uint32_t bph = (it / W4::B_STAGES) & 1;
                    if (!bounded_wait(&full[s], ph, abort_flag, limit, p.status) ||
                        !bounded_wait(&bfull[b], bph, abort_flag, limit, p.status)) { ok = false; break; }
                    tc_fence_after();
                    const uint32_t a_addr = smem_u32(smA + s * W4::A_BYTES);
                    const uint32_t b_addr = smem_u32(smB + b * W4::B_BYTES);
#pragma unroll
                    for (int k = 0; k < W4::BK / 16; ++k) {
                        const uint64_t ad = sw128_desc(a_addr + k * 32, 16, 1024);
                        const uint64_t bd = sw128_desc(b_addr + k * 16 * 128, W4::B_CHUNK, 1024);
                        mma_f16(d_tmem, ad, bd, idesc, (kb | k) != 0);
                    }
                    mma_commit(&rempty[s]);
                    mma_commit(&bempty[b]);
                }
                if (!ok) break;
                mma_commit(&tfull[acc]);
            }
            mma_commit(drain);
            volatile int never = 0;
            bounded_wait(drain, 0, &never, limit, p.status);
        }
        __syncwarp();
    } else if (warp < 2 + W4::EPI_WARPS) {
        // --------------------------------------------------------- epilogue
        const int q = warp & 3;
        uint8_t* stg0 = smStg + (warp - 2) * W4::STG_BUF;
        uint32_t tl = 0, nstore = 0;
        for (int t = blockIdx.x; t < num_tiles; t += gridDim.x, ++tl) {
            int tm, tn;
            tile_coords(t, ntm, ntn, p.group_m, tm, tn);
            const uint32_t acc = tl & 1;
            const uint32_t aph = (tl >> 1) & 1;
            if (!bounded_wait(&tfull[acc], aph, abort_flag, limit, p.status)) break;
            tc_fence_after();
            epilogue_tile<QFP4 ? OutT::BF16 : OutT::F16, W4::BN, true, 1>(&tmC, p, tmem_base + acc * W4::BN, q, lane,
                                                      tm * W4::BM + q * 32, tn * W4::BN, stg0,
                                                      nstore);
            tc_fence_before();
            __syncwarp();
            if (lane == 0) mbar_arrive(&tempty[acc]);
        }
        if (lane == 0) bulk_wait<0>();
        __syncwarp();
    } else {
        // ------------------------------------------------------- converters
        const int ctid = threadIdx.x - 32 * (2 + W4::EPI_WARPS);    // 0..255
        uint32_t it = 0;
        bool ok = true;
        for (int t = blockIdx.x; t < num_tiles && ok; t += gridDim.x) {
            for (int kb = 0; kb < num_kb; ++kb, ++it) {
                const uint32_t s = it % W4::RAW_STAGES;
                const uint32_t ph = (it / W4::RAW_STAGES) & 1;
                const uint32_t b = it % W4::B_STAGES;
                const uint32_t bph = (it / W4::B_STAGES) & 1;
                if (!bounded_wait(&full[s], ph, abort_flag, limit, p.status) ||
                    !bounded_wait(&bempty[b], bph ^ 1, abort_flag, limit, p.status)) { ok = false; break; }
                if constexpr (QFP4)
                    dequant_slice_fp4<W4::BK, W4::BN, 32 * W4::CONV_WARPS, W4::B_CHUNK>(
                        smQ + s * W4::Q_BYTES, smS + s * W4::S_BYTES, smB + b * W4::B_BYTES, ctid);
                else
                    dequant_slice<W4::BK, W4::BN, 32 * W4::CONV_WARPS, W4::B_CHUNK>(
                        smQ + s * W4::Q_BYTES, smS + s * W4::S_BYTES, smB + b * W4::B_BYTES, ctid);
                fence_proxy_async_smem();
                __syncwarp();
                if (lane == 0) {
                    mbar_arrive(&bfull[b]);
                    mbar_arrive(&rempty[s]);
                }
            }
        }
    }

    tc_fence_before();
    __syncthreads();
    if (warp == 1) {
        tc_fence_after();
        tmem_dealloc(tmem_base, W4::TMEM_COLS);
    }
}

template <bool QFP4>
int run_large(const GemmArgs& a) {
    int dev = 0;
    const DeviceInfo* di = current_device(&dev);
    if (!di) return kNoDevice;
    const CUtensorMapDataType at = QFP4 ? CU_TENSOR_MAP_DATA_TYPE_BFLOAT16 : CU_TENSOR_MAP_DATA_TYPE_FLOAT16;
    CUtensorMap tA, tQ, tS, tC;
    if (!tensor_map_2d(&tA, a.A, at, 2, a.K, a.M, a.lda * 2, W4::BK, W4::BM, SWZ_128))
        return kCudaError;
    if (!tensor_map_2d(&tQ, a.B, CU_TENSOR_MAP_DATA_TYPE_UINT8, 1, (a.N + 1) / 2, a.K, a.ldb,
                       W4::BN / 2, W4::BK, SWZ_128))
        return kCudaError;
    if (QFP4 ? !tensor_map_2d(&tS, a.scales, CU_TENSOR_MAP_DATA_TYPE_UINT8, 1, a.N, (a.K + 31) / 32,
                              a.lds, W4::BN, W4::BK / 32, SWZ_NONE)
             : !tensor_map_2d(&tS, a.scales, CU_TENSOR_MAP_DATA_TYPE_FLOAT16, 2, a.N, a.K / 128,
                              a.lds * 2, W4::BN, 1, SWZ_NONE))
        return kCudaError;
    if (!tensor_map_2d(&tC, a.C, at, 2, a.N, a.M, a.ldc * 2, 64, 32, SWZ_128))
        return kCudaError;
    auto kern = w4a16_gemm_kernel<QFP4>;
    if (set_smem_attr(reinterpret_cast<const void*>(kern), W4::SMEM_BYTES, QFP4 ? 6 : 9) !=
        cudaSuccess)
        return kCudaError;
    const long long tiles = ((a.M + W4::BM - 1) / W4::BM) * ((a.N + W4::BN - 1) / W4::BN);
    const int grid = static_cast<int>(persistent_grid(tiles, di->num_sms, a.ctas));
    TcParams p = {};
    p.M = static_cast<int>(a.M);
    p.N = static_cast<int>(a.N);
    p.K = static_cast<int>(a.K);
    p.relu = a.relu;
    p.inject = inject_mode();
    p.group_m = a.group_m > 0 ? a.group_m : W4::GROUP_M;
    p.timeout_ns = wait_limit_ns();
    p.status = device_status_ptr();
    p.C = a.C;
    p.ldc = a.ldc;
    if (!p.status) return kCudaError;
    kern<<<grid, W4::THREADS, W4::SMEM_BYTES, static_cast<cudaStream_t>(a.stream)>>>(
        tA, tQ, tS, tC, p);
    return cudaGetLastError() == cudaSuccess ? kOk : kCudaError;
}

}  // namespace

int launch_w4a16_large(const GemmArgs& a) { return run_large<false>(a); }
int launch_wfp4_large(const GemmArgs& a) { return run_large<true>(a); }

}  // namespace tg
