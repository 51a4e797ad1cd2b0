// gemm_w4a16_pair.cu -- the dequantize GEMM (fp16 activations x signed 4-bit
// weights with fp16 group scales, "W4A16" of the pages' dequantize-GEMM
// examples) for M > 128, on CTA pairs (tcgen05 cta_group::2); the same kernel
// serves FP4 weights (E2M1 codes with E8M0 block scales, bf16 activations,
// bf16 operand and output: the WFP4 GEMM).
//
// The one-CTA kernel (gemm_w4a16.cu) is bound by shared-memory bandwidth:
// per 128 x 256 x 64 step its MMAs read 48 KB of operands and its converter
// warps write 32 KB of fp16 weights and read the packed ones.  Here two CTAs
// on neighbouring SMs (a cluster of 2) share a 256 x 256 output tile, as in
// the 16-bit pair kernel (gemm_tc2.cuh): CTA rank r stages its own 128 rows
// of A by TMA and converts only its own 128 columns of the weight slice
// ([128 r, 128 r + 128) of the tile), so per SM and step the operand reads
// drop to 32 KB and the converted bytes to 16 KB for the same math.
//
// Roles (both CTAs unless noted):
//   warp 0      TMA producer: A rows into the A ring (completion on the
//               leader's full[s], as in the 16-bit pair kernel); the packed
//               weights (64 rows x 64 bytes) and their scale row into the raw
//               ring (rfull[s], local).
//   warp 1      MMA issuer (leader only): waits for A of both CTAs (full[s])
//               and the converted weights of both (bfull[b], 16 converter
//               warp arrivals from the pair), issues cta_group::2 MMAs with
//               M = 256, N = 256, commits stage releases to both CTAs.
//   warps 2-5   epilogue: TMEM -> ReLU -> fp16 -> TMA store of the CTA's
//               128 rows, undoing the converters' column order.
//   warps 6-13  converters: packed slice -> fp16(q * s) in the N-major
//               128-byte-swizzled operand layout (dequant.cuh); they fence
//               their stores to the async proxy and arrive on the leader's
//               bfull[b] (a plain arrive: one with release at cluster scope
//               stalled the converters on a memory barrier every step); the
//               MMA warp waits on it with acquire at cluster scope before the
//               tensor cores read both halves.
// Every wait is bounded; the CTAs meet on cluster barriers after set-up and
// before freeing TMEM.  Loads are plain tiled TMA copies of this GPU's
// memory (no multicast).
#include "dequant.cuh"
#include "gemm_tc.cuh"
#include "host.cuh"
#include "launch.h"

namespace tg {

namespace {

struct W4P {
    static constexpr int BM = 128, PM = 256, BN = 256, HN = 128, BK = 64;
    static constexpr int STAGES = 6, B_STAGES = 4;
    static constexpr int A_STAGE = BM * BK * 2;          // 16 KB
    static constexpr int Q_BYTES = BK * HN / 2;          // 4 KB packed
    static constexpr int S_BYTES = HN * 2;               // 256 B scales
    static constexpr int S_RING = (STAGES * S_BYTES + 1023) / 1024 * 1024;
    static constexpr int B_CHUNK = BK * 128;             // 8 KB: 64 columns x BK rows
    static constexpr int B_STAGE = (HN / 64) * B_CHUNK;  // 16 KB
    static constexpr int STG_BUF = 32 * 128;
    static constexpr int EPI_WARPS = 4, CONV_WARPS = 8;
    static constexpr int THREADS = 32 * (2 + EPI_WARPS + CONV_WARPS);
    static constexpr int TMEM_COLS = 2 * BN;             // double-buffered accumulator
    static constexpr int GROUP_M = 8;                    // pair-tile rows per raster band
    static constexpr int SMEM_DATA = STAGES * (A_STAGE + Q_BYTES) + S_RING + B_STAGES * B_STAGE +
                                     EPI_WARPS * 2 * STG_BUF;
    static constexpr int SMEM_BYTES = SMEM_DATA + 512 + 1024;
    // Layout guards: every 128-byte-swizzled buffer (A, converted B) starts
    // on a 1024-byte boundary, and so does the packed ring (64-byte swizzle)
    // and the staging after the scale ring; the barriers, TMEM slot and
    // abort flag fit their 512 bytes; one CTA fits the 227 KB limit.
    static_assert(A_STAGE % 1024 == 0 && B_STAGE % 1024 == 0 && B_CHUNK % 1024 == 0, "swizzle");
    static_assert((STAGES * A_STAGE + B_STAGES * B_STAGE) % 1024 == 0, "packed ring alignment");
    static_assert((STAGES * Q_BYTES) % 1024 == 0 && S_RING % 1024 == 0, "staging alignment");
    static_assert((4 * STAGES + 2 * B_STAGES + 5) * 8 + 8 <= 512, "barrier area");
    static_assert(SMEM_BYTES <= 227 * 1024, "shared memory per CTA");
    static_assert(TMEM_COLS == 512, "TMEM: two 256-column accumulators");
    static_assert(32 * CONV_WARPS == 256 && BK * HN / 2 == Q_BYTES, "converter split");
};

// mbarrier wait with acquire at cluster scope (the arrivals it waits for
// come from the peer CTA and publish its shared-memory writes).
__device__ __forceinline__ bool mbar_try_wait_cluster(uint64_t* bar, uint32_t parity) {
    uint32_t ok;
    asm volatile(
        "{\n\t.reg .pred p;\n\t"
        "mbarrier.try_wait.parity.acquire.cluster.shared::cta.b64 p, [%1], %2;\n\t"
        "selp.b32 %0, 1, 0, p;\n\t}"
        : "=r"(ok) : "r"(smem_u32(bar)), "r"(parity) : "memory");
    return ok != 0;
}

__device__ __forceinline__ bool bounded_wait_cluster(uint64_t* bar, uint32_t parity, volatile int* abort,
                                                     uint64_t limit_ns, int* status) {
    const uint64_t t0 = globaltimer_ns();
    for (;;) {
        if (mbar_try_wait_cluster(bar, parity)) return true;
        if (*abort) return false;
        if (globaltimer_ns() - t0 > limit_ns) {
            *abort = 1;
            atomicExch(status, ST_TIMEOUT);
            return false;
        }
    }
}


// QFP4 = false: signed 4-bit weights with fp16 group scales, fp16
// activations and output; true: FP4 (E2M1) weights with E8M0 block scales,
// bf16 activations and output (dequant.cuh).
template <bool QFP4>
__global__ void __launch_bounds__(W4P::THREADS, 1)
w4a16_pair_kernel(const __grid_constant__ CUtensorMap tmA,
                  const __grid_constant__ CUtensorMap tmQ,
                  const __grid_constant__ CUtensorMap tmS,
                  const __grid_constant__ CUtensorMap tmC,
                  const TcParams p) {
    extern __shared__ uint8_t smem_raw[];
    const uint32_t raw_addr = smem_u32(smem_raw);
    uint8_t* smem = smem_raw + (((raw_addr + 1023u) & ~1023u) - raw_addr);
    uint8_t* smA = smem;                                              // STAGES x 16 KB
    uint8_t* smB = smA + W4P::STAGES * W4P::A_STAGE;                  // B_STAGES x 16 KB
    uint8_t* smQ = smB + W4P::B_STAGES * W4P::B_STAGE;                // STAGES x 4 KB
    uint8_t* smS = smQ + W4P::STAGES * W4P::Q_BYTES;                  // STAGES x 256 B (padded)
    uint8_t* smStg = smS + W4P::S_RING;                               // epilogue staging
    uint64_t* bars = reinterpret_cast<uint64_t*>(smStg + W4P::EPI_WARPS * 2 * W4P::STG_BUF);
    uint64_t* full = bars;                                  // [STAGES] A of both (leader)
    uint64_t* empty = full + W4P::STAGES;                   // [STAGES] A stage free (MMA)
    uint64_t* rfull = empty + W4P::STAGES;                  // [STAGES] packed slice landed
    uint64_t* rempty = rfull + W4P::STAGES;                 // [STAGES] converters done with it
    uint64_t* bfull = rempty + W4P::STAGES;                 // [B_STAGES] converted, both (leader)
    uint64_t* bempty = bfull + W4P::B_STAGES;               // [B_STAGES] MMA done with it
    uint64_t* tfull = bempty + W4P::B_STAGES;               // [2]
    uint64_t* tempty = tfull + 2;                           // [2] (leader)
    uint64_t* drain = tempty + 2;
    uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(drain + 1);
    volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_slot + 1);

    const int warp = threadIdx.x >> 5;
    const int lane = threadIdx.x & 31;
    const uint32_t rank = cluster_ctarank();
    const int pair = blockIdx.x >> 1;
    const int npairs = gridDim.x >> 1;
    const int ntm = (p.M + W4P::PM - 1) / W4P::PM;
    const int ntn = (p.N + W4P::BN - 1) / W4P::BN;
    const int num_tiles = ntm * ntn;
    const int num_kb = (p.K + W4P::BK - 1) / W4P::BK;
    const uint64_t limit = p.timeout_ns;

    if (threadIdx.x == 0) {
        for (int s = 0; s < W4P::STAGES; ++s) {
            mbar_init(&full[s], 2);
            mbar_init(&empty[s], 1);
            mbar_init(&rfull[s], 1);
            mbar_init(&rempty[s], W4P::CONV_WARPS);
        }
        for (int b = 0; b < W4P::B_STAGES; ++b) {
            mbar_init(&bfull[b], 2 * W4P::CONV_WARPS);
            mbar_init(&bempty[b], 1);
        }
        for (int a = 0; a < 2; ++a) { mbar_init(&tfull[a], 1); mbar_init(&tempty[a], 2 * W4P::EPI_WARPS); }
        mbar_init(drain, 1);
        *abort_flag = 0;
        fence_mbar_init();
        fence_proxy_async_smem();
    }
    if (warp == 0 && lane == 0) {
        tma_prefetch_desc(&tmA);
        tma_prefetch_desc(&tmQ);
        tma_prefetch_desc(&tmS);
        tma_prefetch_desc(&tmC);
    }
    if (warp == 1) {
        tmem_alloc_pair(tmem_slot, W4P::TMEM_COLS);
        tmem_relinquish_pair();
    }
    tc_fence_before();
    __syncthreads();
    cluster_sync_all();          // peer barriers initialised before any remote use
    tc_fence_after();
    const uint32_t tmem_base = *tmem_slot;

    if (warp == 0) {
        // ------------------------------------------------ TMA producer (both)
        if (elect_one()) {
            uint32_t armed = 0, armed_par = 0, rarmed = 0, rarmed_par = 0, it = 0;
            bool ok = true;
            for (int t = pair; t < num_tiles && ok; t += npairs) {
                int tm, tn;
                tile_coords(t, ntm, ntn, p.group_m, tm, tn);
                const int m0 = tm * W4P::PM + rank * W4P::BM;
                const int n0 = tn * W4P::BN + rank * W4P::HN;
                // A rows entirely past M are not loaded (never stored); packed
                // slices past N read the copy engine's zero fill
                const bool a_live = m0 < p.M;
                for (int kb = 0; kb < num_kb; ++kb, ++it) {
                    const uint32_t s = it % W4P::STAGES;
                    const uint32_t ph = (it / W4P::STAGES) & 1;
                    if (!bounded_wait(&empty[s], ph ^ 1, abort_flag, limit, p.status) ||
                        !bounded_wait(&rempty[s], ph ^ 1, abort_flag, limit, p.status)) { ok = false; break; }
                    if (p.inject == 1 && it == 0 && pair == 0 && rank == 0) continue;   // debug: never arm slot 0
                    const uint32_t fbar = mapa_shared(smem_u32(&full[s]), 0);
                    mbar_arrive_expect_tx_cluster(fbar, a_live ? W4P::A_STAGE : 0);
                    armed |= 1u << s;
                    armed_par = (armed_par & ~(1u << s)) | (ph << s);
                    if (a_live) tma_load_2d_pair(smA + s * W4P::A_STAGE, &tmA, fbar, kb * W4P::BK, m0);
                    mbar_arrive_expect_tx(&rfull[s], W4P::Q_BYTES + W4P::S_BYTES);
                    rarmed |= 1u << s;
                    rarmed_par = (rarmed_par & ~(1u << s)) | (ph << s);
                    tma_load_2d(smQ + s * W4P::Q_BYTES, &tmQ, &rfull[s], n0 / 2, kb * W4P::BK);
                    tma_load_2d(smS + s * W4P::S_BYTES, &tmS, &rfull[s], n0,
                                (kb * W4P::BK) / (QFP4 ? 32 : 128));
                }
            }
            if (!ok) {
                // let this CTA's copies in flight land before it exits
                for (int s = 0; s < W4P::STAGES; ++s) {
                    volatile int never = 0;
                    if (rarmed & (1u << s))
                        bounded_wait(&rfull[s], (rarmed_par >> s) & 1, &never, limit, p.status);
                    if (rank == 0 && (armed & (1u << s)))
                        bounded_wait(&full[s], (armed_par >> s) & 1, &never, limit, p.status);
                }
                if (rank != 0) {
                    // A copies complete on the leader's barriers: give them 1 ms
                    const uint64_t t0 = globaltimer_ns();
                    while (globaltimer_ns() - t0 < 1000000ull) __nanosleep(10000);
                }
            }
        }
        __syncwarp();
    } else if (warp == 1) {
        // ------------------------------------------ MMA issuer (leader only)
        if (rank == 0 && elect_one()) {
            constexpr uint32_t idesc = make_idesc(QFP4 ? 1 : 0, W4P::PM, W4P::BN, 0, 1);
            uint32_t it = 0, tl = 0;
            bool ok = true;
            for (int t = pair; t < num_tiles && ok; t += npairs, ++tl) {
                const uint32_t acc = tl & 1;
                const uint32_t aph = (tl >> 1) & 1;
                if (!bounded_wait(&tempty[acc], aph ^ 1, abort_flag, limit, p.status)) { ok = false; break; }
                tc_fence_after();
                const uint32_t d_tmem = tmem_base + acc * W4P::BN;
                for (int kb = 0; kb < num_kb; ++kb, ++it) {
                    const uint32_t s = it % W4P::STAGES;
                    const uint32_t ph = (it / W4P::STAGES) & 1;
                    const uint32_t b = it % W4P::B_STAGES;
                    const uint32_t bph = (it / W4P::B_STAGES) & 1;
                    if (!bounded_wait(&full[s], ph, abort_flag, limit, p.status) ||
                        !bounded_wait_cluster(&bfull[b], bph, abort_flag, limit, p.status)) { ok = false; break; }
                    tc_fence_after();
                    const uint32_t a_addr = smem_u32(smA + s * W4P::A_STAGE);
                    const uint32_t b_addr = smem_u32(smB + b * W4P::B_STAGE);
#pragma unroll
                    for (int k = 0; k < W4P::BK / 16; ++k) {
                        const uint64_t ad = sw128_desc(a_addr + k * 32, 16, 1024);
                        const uint64_t bd = sw128_desc(b_addr + k * 16 * 128, W4P::B_CHUNK, 1024);
                        mma_f16_pair(d_tmem, ad, bd, idesc, (kb | k) != 0);
                    }
                    const uint32_t e_loc = smem_u32(&empty[s]);
                    const uint32_t be_loc = smem_u32(&bempty[b]);
                    mma_commit_pair(mapa_shared(e_loc, 0));       // both CTAs' A slots
                    mma_commit_pair(mapa_shared(e_loc, 1));
                    mma_commit_pair(mapa_shared(be_loc, 0));      // both CTAs' weight slots
                    mma_commit_pair(mapa_shared(be_loc, 1));
                }
                if (!ok) break;
                const uint32_t f_loc = smem_u32(&tfull[acc]);
                mma_commit_pair(mapa_shared(f_loc, 0));           // both CTAs' accumulators
                mma_commit_pair(mapa_shared(f_loc, 1));
            }
            mma_commit_pair(mapa_shared(smem_u32(drain), 0));
            volatile int never = 0;
            bounded_wait(drain, 0, &never, limit, p.status);
        }
        __syncwarp();
    } else if (warp < 2 + W4P::EPI_WARPS) {
        // --------------------------------------------------- epilogue (both)
        const int q = warp & 3;
        uint8_t* stg0 = smStg + (warp - 2) * 2 * W4P::STG_BUF;
        uint32_t tl = 0, nstore = 0;
        for (int t = pair; t < num_tiles; t += npairs, ++tl) {
            int tm, tn;
            tile_coords(t, ntm, ntn, p.group_m, tm, tn);
            const uint32_t acc = tl & 1;
            const uint32_t aph = (tl >> 1) & 1;
            if (!bounded_wait(&tfull[acc], aph, abort_flag, limit, p.status)) break;
            tc_fence_after();
            epilogue_tile<QFP4 ? OutT::BF16 : OutT::F16, W4P::BN, true, 2>(&tmC, p, tmem_base + acc * W4P::BN, q, lane,
                                                       tm * W4P::PM + rank * W4P::BM + q * 32,
                                                       tn * W4P::BN, stg0, nstore);
            tc_fence_before();
            __syncwarp();
            if (lane == 0) mbar_arrive_cluster(mapa_shared(smem_u32(&tempty[acc]), 0));
        }
        if (lane == 0) bulk_wait<0>();
        __syncwarp();
    } else {
        // ------------------------------------------------- converters (both)
        const int ctid = threadIdx.x - 32 * (2 + W4P::EPI_WARPS);    // 0..255
        uint32_t it = 0;
        bool ok = true;
        for (int t = pair; t < num_tiles && ok; t += npairs) {
            for (int kb = 0; kb < num_kb; ++kb, ++it) {
                const uint32_t s = it % W4P::STAGES;
                const uint32_t ph = (it / W4P::STAGES) & 1;
                const uint32_t b = it % W4P::B_STAGES;
                const uint32_t bph = (it / W4P::B_STAGES) & 1;
                if (!bounded_wait(&rfull[s], ph, abort_flag, limit, p.status) ||
                    !bounded_wait(&bempty[b], bph ^ 1, abort_flag, limit, p.status)) { ok = false; break; }
                if constexpr (QFP4)
                    dequant_slice_fp4<W4P::BK, W4P::HN, 32 * W4P::CONV_WARPS, W4P::B_CHUNK>(
                        smQ + s * W4P::Q_BYTES, smS + s * W4P::S_BYTES, smB + b * W4P::B_STAGE, ctid);
                else
                    dequant_slice<W4P::BK, W4P::HN, 32 * W4P::CONV_WARPS, W4P::B_CHUNK>(
                        smQ + s * W4P::Q_BYTES, smS + s * W4P::S_BYTES, smB + b * W4P::B_STAGE, ctid);
                fence_proxy_async_smem();
                __syncwarp();
                if (lane == 0) {
                    mbar_arrive(&rempty[s]);
                    mbar_arrive_cluster(mapa_shared(smem_u32(&bfull[b]), 0));
                }
            }
        }
    }

    tc_fence_before();
    __syncthreads();
    cluster_sync_all();          // the pair is done with each other's barriers and TMEM
    if (warp == 1) {
        tc_fence_after();
        tmem_dealloc_pair(tmem_base, W4P::TMEM_COLS);
    }
}

// Returns kUnsupported (nothing launched) when the pair launch is refused,
// so the caller can fall back to the one-CTA kernel.
template <bool QFP4>
int run_pair(const GemmArgs& a) {
    if (pair_kernels_disabled()) return kUnsupported;
    int dev = 0;
    const DeviceInfo* di = current_device(&dev);
    if (!di) return kNoDevice;
    const CUtensorMapDataType at = QFP4 ? CU_TENSOR_MAP_DATA_TYPE_BFLOAT16 : CU_TENSOR_MAP_DATA_TYPE_FLOAT16;
    CUtensorMap tA, tQ, tS, tC;
    if (!tensor_map_2d(&tA, a.A, at, 2, a.K, a.M, a.lda * 2, W4P::BK, W4P::BM, SWZ_128))
        return kCudaError;
    if (!tensor_map_2d(&tQ, a.B, CU_TENSOR_MAP_DATA_TYPE_UINT8, 1, (a.N + 1) / 2, a.K, a.ldb,
                       W4P::HN / 2, W4P::BK, SWZ_64))
        return kCudaError;
    if (QFP4 ? !tensor_map_2d(&tS, a.scales, CU_TENSOR_MAP_DATA_TYPE_UINT8, 1, a.N, (a.K + 31) / 32,
                              a.lds, W4P::HN, W4P::BK / 32, SWZ_NONE)
             : !tensor_map_2d(&tS, a.scales, CU_TENSOR_MAP_DATA_TYPE_FLOAT16, 2, a.N, a.K / 128,
                              a.lds * 2, W4P::HN, 1, SWZ_NONE))
        return kCudaError;
    if (!tensor_map_2d(&tC, a.C, at, 2, a.N, a.M, a.ldc * 2, 64, 32, SWZ_128))
        return kCudaError;
    auto kern = w4a16_pair_kernel<QFP4>;
    if (set_smem_attr(reinterpret_cast<const void*>(kern), W4P::SMEM_BYTES, QFP4 ? 7 : 10) !=
        cudaSuccess)
        return kCudaError;
    const long long tiles = ((a.M + W4P::PM - 1) / W4P::PM) * ((a.N + W4P::BN - 1) / W4P::BN);
    const int npairs = static_cast<int>(persistent_grid(tiles, di->num_sms / 2, a.ctas));
    TcParams p = {};
    p.M = static_cast<int>(a.M);
    p.N = static_cast<int>(a.N);
    p.K = static_cast<int>(a.K);
    p.relu = a.relu;
    p.inject = inject_mode();
    p.group_m = a.group_m > 0 ? a.group_m : W4P::GROUP_M;
    p.timeout_ns = wait_limit_ns();
    p.status = device_status_ptr();
    p.C = a.C;
    p.ldc = a.ldc;
    if (!p.status) return kCudaError;
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3(2 * npairs, 1, 1);
    cfg.blockDim = dim3(W4P::THREADS, 1, 1);
    cfg.dynamicSmemBytes = W4P::SMEM_BYTES;
    cfg.stream = static_cast<cudaStream_t>(a.stream);
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeClusterDimension;
    attr[0].val.clusterDim.x = 2;
    attr[0].val.clusterDim.y = 1;
    attr[0].val.clusterDim.z = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    if (cudaLaunchKernelEx(&cfg, kern, tA, tQ, tS, tC, p) != cudaSuccess) {
        cudaGetLastError();                       // clear; caller falls back
        return kUnsupported;
    }
    return kOk;
}

}  // namespace

int launch_w4a16_pair(const GemmArgs& a) { return run_pair<false>(a); }
int launch_wfp4_pair(const GemmArgs& a) { return run_pair<true>(a); }

}  // namespace tg
