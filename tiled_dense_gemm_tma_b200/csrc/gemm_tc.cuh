// gemm_tc.cuh -- persistent, warp-specialised tensor-core GEMM for sm_100a.
//
// C = epi(A . B), A row-major M x K, B row-major K x N, fp32 accumulation in
// tensor memory (TMEM).  Used for fp16, bf16 (tcgen05.mma kind::f16) and the
// TF32 mode of the fp32 path (kind::tf32).
//
// The design follows the tiling scheme of "TileLang ... 高效 GEMM 内核"
// (mhpq.cn), sections 2.1-3.3: each output tile's A and B strips are staged
// from global into shared memory slice by slice along K, multiplied into an
// on-chip accumulator, and the accumulator is written back once; loads of
// slice k+1 overlap the math on slice k (the num_stages pipelining of the
// blog.hotdry.top guide).  On B200 this becomes:
//
//   warp 0      TMA producer: one elected thread waits for a free ring slot
//               (empty[s]), arms full[s] with the slot's byte count and issues
//               cp.async.bulk.tensor loads of the A box (BM x 128 B, K-major)
//               and the B boxes (BK rows x 128 B each, N-major).  Out-of-range
//               rows / columns are zero-filled by the copy engine, which is
//               the boundary handling the mhpq.cn article, section 4.1, asks for.
//   warp 1      MMA issuer: allocates 2 x BN TMEM columns (double-buffered
//               accumulator), waits full[s], issues BK/MMA_K tcgen05.mma and
//               tcgen05.commit -> empty[s]; after the tile's last slice it
//               commits to tmem_full[acc].
//   warps 2-5   epilogue: wait tmem_full[acc], tcgen05.ld 32 rows each,
//               optional ReLU in fp32, round to the output type, write a
//               128-byte-swizzled 32-row staging box and TMA-store it (stores
//               are clipped at the matrix edge); then release tmem_empty[acc]
//               so the next tile's mainloop overlaps this epilogue.
//
// Tiles are visited in a grouped order (GROUP_M tile rows at a time) so that
// concurrently running CTAs share A and B strips in L2 (the swizzle for L2
// locality of the blog.hotdry.top guide).  The grid is one CTA per SM.
#pragma once
#include "ptx.cuh"
#include "tile_sched.h"     // tile_coords
#include <cuda_bf16.h>
#include <cuda_fp16.h>

namespace tg {

enum class OutT { F16, BF16, F32 };

template <int IN_BYTES_, int FMT_, OutT OUT_, int BN_, int STAGES_>
struct TcCfg {
    static constexpr int IN_BYTES = IN_BYTES_;          // 2 (f16/bf16) or 4 (tf32)
    static constexpr int FMT = FMT_;                    // idesc format: 0 f16, 1 bf16, 2 tf32
    static constexpr OutT OUT = OUT_;
    static constexpr int OUT_BYTES = OUT_ == OutT::F32 ? 4 : 2;
    static constexpr int BM = 128;
    static constexpr int BN = BN_;
    static constexpr int BK = 128 / IN_BYTES;           // one 128-byte swizzle row of K
    static constexpr int MMA_K = 32 / IN_BYTES;         // K per tcgen05.mma
    static constexpr int CHUNK_N = 128 / IN_BYTES;      // N columns per 128-byte B box row
    static constexpr int STAGES = STAGES_;
    static constexpr int A_STAGE = BM * 128;            // bytes
    static constexpr int B_CHUNK = BK * 128;            // bytes of one BK x CHUNK_N box
    static constexpr int B_STAGE = (BN / CHUNK_N) * B_CHUNK;
    static constexpr int STAGE_BYTES = A_STAGE + B_STAGE;
    // N-major B: tf32 needs the 32-byte-unit swizzle (4-row atom, 512 B).
    static constexpr uint32_t B_LAYOUT = IN_BYTES == 4 ? 1u : 2u;
    static constexpr uint32_t B_SBO = IN_BYTES == 4 ? 512u : 1024u;
    static constexpr int CW = 128 / OUT_BYTES;          // output columns per staging row
    static constexpr int STG_BUF = 32 * 128;            // one warp's 32-row staging box
    static constexpr int EPI_WARPS = 4;
    static constexpr int TMEM_COLS = 2 * BN;            // double-buffered accumulator
    static constexpr int THREADS = 64 + 32 * EPI_WARPS;
    static constexpr int GROUP_M = 16;
    static constexpr int SMEM_DATA = STAGES * STAGE_BYTES + EPI_WARPS * 2 * STG_BUF;
    static constexpr int SMEM_BYTES = SMEM_DATA + 256 + 1024;   // + barriers + alignment slack
    static_assert(TMEM_COLS == 256 || TMEM_COLS == 512, "TMEM allocation must be a power of 2");
    static_assert(BN % CHUNK_N == 0 && BN % CW == 0 && BN <= 256 && BN % 16 == 0, "bad BN");
};

struct TcParams {
    int M, N, K;
    int relu;
    int inject;               // debug: 1 = CTA 0's producer skips arming the first slot
    int group_m;              // raster band height in tiles (tile_coords)
    unsigned long long timeout_ns;
    int* status;              // device status word (ST_TIMEOUT on an expired wait)
    void* C;                  // output base and row pitch (elements), for the ragged
    long long ldc;            // last column chunk, which is stored without TMA
    // CTA-pair kernel only: hybrid schedule (tail_split / tail_dp of
    // tile_sched.h) and, when split, its workspace: per tail tile and rank a
    // check-in and a published word, and one 128 x 256 fp32 partial
    int tail_split;
    int dp_tiles;
    int* tickets;
    float* ws;
};

// Store the first `valid_bytes` (< 128) of one packed 128-byte output row
// segment with plain global stores.  The copy engine rounds a clipped store
// up to whole 16-byte units, so a row tail narrower than that is written here.
template <int OUT_BYTES>
__device__ __forceinline__ void store_row_tail(uint8_t* dst, const uint4* packed, int valid_bytes) {
#pragma unroll
    for (int j = 0; j < 8; ++j) {
        const int b0 = j * 16;
        if (b0 + 16 <= valid_bytes) {
            *reinterpret_cast<uint4*>(dst + b0) = packed[j];
        } else if (b0 < valid_bytes) {
            const uint32_t w[4] = {packed[j].x, packed[j].y, packed[j].z, packed[j].w};
#pragma unroll
            for (int e = 0; e < 16 / OUT_BYTES; ++e) {
                if (b0 + e * OUT_BYTES >= valid_bytes) break;
                if (OUT_BYTES == 4) {
                    *reinterpret_cast<uint32_t*>(dst + b0 + 4 * e) = w[e];
                } else {
                    *reinterpret_cast<uint16_t*>(dst + b0 + 2 * e) =
                        static_cast<uint16_t>(w[e >> 1] >> (16 * (e & 1)));
                }
            }
        }
    }
}

// Source position, inside an 8-column group, of output column q when the
// group's accumulator columns are stored in the order 0,2,4,6,1,3,5,7 (the
// order the 4-bit weight converter produces).
__device__ __forceinline__ constexpr int perm8_src(int q) { return (q >> 1) | ((q & 1) << 2); }

// 64 fp32 accumulators -> 64 fp16 / bf16 (8 x 16 B); 32 -> 32 fp32 (8 x 16 B).
// PERM8: undo the 0,2,4,6,1,3,5,7 column order inside each 8-column group.
template <OutT O, bool PERM8>
__device__ __forceinline__ void pack_row_chunk(const uint32_t* v, int relu, uint4* out) {
#pragma unroll
    for (int j = 0; j < 8; ++j) {
        uint32_t w[4];
#pragma unroll
        for (int h = 0; h < 4; ++h) {
            if constexpr (O == OutT::F32) {
                float x = __uint_as_float(v[j * 4 + h]);
                if (relu) x = fmaxf(x, 0.f);
                w[h] = __float_as_uint(x);
            } else {
                const int i0 = PERM8 ? perm8_src(2 * h) : 2 * h;
                const int i1 = PERM8 ? perm8_src(2 * h + 1) : 2 * h + 1;
                float x0 = __uint_as_float(v[j * 8 + i0]);
                float x1 = __uint_as_float(v[j * 8 + i1]);
                if (relu) { x0 = fmaxf(x0, 0.f); x1 = fmaxf(x1, 0.f); }
                if constexpr (O == OutT::BF16) {
                    __nv_bfloat162 pr = __floats2bfloat162_rn(x0, x1);
                    w[h] = *reinterpret_cast<uint32_t*>(&pr);
                } else {
                    __half2 pr = __floats2half2_rn(x0, x1);
                    w[h] = *reinterpret_cast<uint32_t*>(&pr);
                }
            }
        }
        out[j] = make_uint4(w[0], w[1], w[2], w[3]);
    }
}

// Epilogue of one output tile for the 32 rows of TMEM lane quarter q:
// tcgen05.ld the accumulator columns CW at a time, ReLU, round, write a
// 128-byte-swizzled 32-row staging box and TMA-store it; the ragged last
// chunk of a row (narrower than CW columns) is stored per lane instead.
// NBUF staging buffers of 4 KB per warp rotate through `nstore`.
template <OutT OUT, int BN, bool PERM8, int NBUF>
__device__ __forceinline__ void epilogue_tile(const CUtensorMap* tmC, const TcParams& p,
                                              uint32_t tmem_tile, int q, int lane,
                                              int row0, int n0, uint8_t* stg0,
                                              uint32_t& nstore) {
    constexpr int OUT_BYTES = OUT == OutT::F32 ? 4 : 2;
    constexpr int CW = 128 / OUT_BYTES;
    constexpr int STG_BUF = 32 * 128;
    if (row0 >= p.M) return;                               // warp-uniform
#pragma unroll 1
    for (int c = 0; c < BN / CW; ++c) {
        const int col0 = n0 + c * CW;
        if (col0 >= p.N) break;
        const uint32_t taddr = tmem_tile + (static_cast<uint32_t>(q * 32) << 16) + c * CW;
        uint32_t v[CW];
        tmem_ld_32x32b_x32(taddr, *reinterpret_cast<uint32_t(*)[32]>(&v[0]));
        if constexpr (CW == 64)
            tmem_ld_32x32b_x32(taddr + 32, *reinterpret_cast<uint32_t(*)[32]>(&v[32]));
        tmem_ld_wait();
        uint4 packed[8];
        pack_row_chunk<OUT, PERM8>(v, p.relu, packed);
        if (col0 + CW > p.N) {
            const int row = row0 + lane;
            if (row < p.M) {
                uint8_t* dst = static_cast<uint8_t*>(p.C) +
                    (static_cast<long long>(row) * p.ldc + col0) * OUT_BYTES;
                store_row_tail<OUT_BYTES>(dst, packed, (p.N - col0) * OUT_BYTES);
            }
            continue;
        }
        uint8_t* stg = stg0 + (nstore % NBUF) * STG_BUF;
        if (lane == 0) bulk_wait_read<NBUF - 1>();         // this buffer's last store has read it
        __syncwarp();
        uint8_t* row = stg + lane * 128;
#pragma unroll
        for (int j = 0; j < 8; ++j)
            *reinterpret_cast<uint4*>(row + ((j ^ (lane & 7)) << 4)) = packed[j];
        fence_proxy_async_smem();
        __syncwarp();
        if (lane == 0) {
            tma_store_2d(tmC, stg, col0, row0);
            bulk_commit();
        }
        ++nstore;
    }
}

template <class Cfg>
__global__ void __launch_bounds__(Cfg::THREADS, 1)
tc_gemm_kernel(const __grid_constant__ CUtensorMap tmA,
               const __grid_constant__ CUtensorMap tmB,
               const __grid_constant__ CUtensorMap tmC,
               const TcParams p) {
    extern __shared__ uint8_t smem_raw[];
    // 1024-byte alignment: the 128-byte swizzle pattern repeats every 8 rows.
    const uint32_t raw = smem_u32(smem_raw);
    uint8_t* smem = smem_raw + (((raw + 1023u) & ~1023u) - raw);
    uint8_t* smA = smem;                                        // STAGES x A_STAGE
    uint8_t* smB = smA + Cfg::STAGES * Cfg::A_STAGE;            // STAGES x B_STAGE
    uint8_t* smStg = smB + Cfg::STAGES * Cfg::B_STAGE;          // 4 warps x 2 x STG_BUF
    uint64_t* bars = reinterpret_cast<uint64_t*>(smStg + Cfg::EPI_WARPS * 2 * Cfg::STG_BUF);
    uint64_t* full = bars;                                      // [STAGES]
    uint64_t* empty = full + Cfg::STAGES;                       // [STAGES]
    uint64_t* tfull = empty + Cfg::STAGES;                      // [2]
    uint64_t* tempty = tfull + 2;                               // [2]
    uint64_t* drain = tempty + 2;                               // [1]
    uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(drain + 1);
    volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_slot + 1);

    const int warp = threadIdx.x >> 5;
    const int lane = threadIdx.x & 31;
    const int ntm = (p.M + Cfg::BM - 1) / Cfg::BM;
    const int ntn = (p.N + Cfg::BN - 1) / Cfg::BN;
    const int num_tiles = ntm * ntn;
    const int num_kb = (p.K + Cfg::BK - 1) / Cfg::BK;
    const uint64_t limit = p.timeout_ns;

    if (threadIdx.x == 0) {
        for (int s = 0; s < Cfg::STAGES; ++s) { mbar_init(&full[s], 1); mbar_init(&empty[s], 1); }
        for (int a = 0; a < 2; ++a) { mbar_init(&tfull[a], 1); mbar_init(&tempty[a], Cfg::EPI_WARPS); }
        mbar_init(drain, 1);
        *abort_flag = 0;
        fence_mbar_init();
        fence_proxy_async_smem();
    }
    if (warp == 0 && lane == 0) {
        tma_prefetch_desc(&tmA);
        tma_prefetch_desc(&tmB);
        tma_prefetch_desc(&tmC);
    }
    if (warp == 1) {
        tmem_alloc(tmem_slot, Cfg::TMEM_COLS);
        tmem_relinquish();
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem_base = *tmem_slot;

    if (warp == 0) {
        // ------------------------------------------------------ TMA producer
        if (elect_one()) {
            uint32_t armed = 0, armed_par = 0;     // per-slot: armed and its parity
            uint32_t it = 0;
            bool ok = true;
            for (int t = blockIdx.x; t < num_tiles && ok; t += gridDim.x) {
                int tm, tn;
                tile_coords(t, ntm, ntn, p.group_m, tm, tn);
                for (int kb = 0; kb < num_kb; ++kb, ++it) {
                    const uint32_t s = it % Cfg::STAGES;
                    const uint32_t ph = (it / Cfg::STAGES) & 1;
                    if (!bounded_wait(&empty[s], ph ^ 1, abort_flag, limit, p.status)) { ok = false; break; }
                    if (p.inject == 1 && it == 0 && blockIdx.x == 0) continue;   // debug: never arm slot 0
                    // B boxes that start past column N are not loaded: their
                    // columns only feed output columns >= N, which are never stored.
                    const int live_chunks = min(Cfg::BN / Cfg::CHUNK_N,
                                                (p.N - tn * Cfg::BN + Cfg::CHUNK_N - 1) / Cfg::CHUNK_N);
                    mbar_arrive_expect_tx(&full[s], Cfg::A_STAGE + live_chunks * Cfg::B_CHUNK);
                    armed |= 1u << s;
                    armed_par = (armed_par & ~(1u << s)) | (ph << s);
                    tma_load_2d(smA + s * Cfg::A_STAGE, &tmA, &full[s], kb * Cfg::BK, tm * Cfg::BM);
                    uint8_t* b_dst = smB + s * Cfg::B_STAGE;
                    for (int j = 0; j < live_chunks; ++j)
                        tma_load_2d(b_dst + j * Cfg::B_CHUNK, &tmB, &full[s],
                                    tn * Cfg::BN + j * Cfg::CHUNK_N, kb * Cfg::BK);
                }
            }
            if (!ok) {
                // Let copies already in flight land before the CTA exits.
                for (int s = 0; s < Cfg::STAGES; ++s)
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
            constexpr uint32_t idesc = make_idesc(Cfg::FMT, Cfg::BM, Cfg::BN, 0, 1);
            uint32_t it = 0, tl = 0;
            bool ok = true;
            for (int t = blockIdx.x; t < num_tiles && ok; t += gridDim.x, ++tl) {
                const uint32_t acc = tl & 1;
                const uint32_t aph = (tl >> 1) & 1;
                if (!bounded_wait(&tempty[acc], aph ^ 1, abort_flag, limit, p.status)) { ok = false; break; }
                tc_fence_after();
                const uint32_t d_tmem = tmem_base + acc * Cfg::BN;
                for (int kb = 0; kb < num_kb; ++kb, ++it) {
                    const uint32_t s = it % Cfg::STAGES;
                    const uint32_t ph = (it / Cfg::STAGES) & 1;
                    if (!bounded_wait(&full[s], ph, abort_flag, limit, p.status)) { ok = false; break; }
                    tc_fence_after();
                    const uint32_t a_addr = smem_u32(smA + s * Cfg::A_STAGE);
                    const uint32_t b_addr = smem_u32(smB + s * Cfg::B_STAGE);
#pragma unroll
                    for (int k = 0; k < Cfg::BK / Cfg::MMA_K; ++k) {
                        // A: K-major, advance 32 bytes of K inside the swizzle row.
                        const uint64_t ad = sw128_desc(a_addr + k * 32, 16, 1024);
                        // B: N-major, advance MMA_K rows of 128 bytes.  16-bit
                        // data uses the 8-row swizzle atom, tf32 the 4-row one.
                        const uint64_t bd = sw128_desc(b_addr + k * Cfg::MMA_K * 128,
                                                       Cfg::B_CHUNK, Cfg::B_SBO, Cfg::B_LAYOUT);
                        if (Cfg::FMT == 2) mma_tf32(d_tmem, ad, bd, idesc, (kb | k) != 0);
                        else               mma_f16(d_tmem, ad, bd, idesc, (kb | k) != 0);
                    }
                    mma_commit(&empty[s]);       // slot free once these MMAs have read it
                }
                if (!ok) break;
                mma_commit(&tfull[acc]);         // accumulator complete
            }
            // All issued MMAs must finish before TMEM is released.
            mma_commit(drain);
            volatile int never = 0;
            bounded_wait(drain, 0, &never, limit, p.status);
        }
        __syncwarp();
    } else {
        // --------------------------------------------------------- epilogue
        const int q = warp & 3;                  // TMEM lane quarter of this warp
        const int ew = warp - 2;                 // staging buffer owner index
        uint8_t* stg0 = smStg + ew * 2 * Cfg::STG_BUF;
        uint32_t tl = 0, nstore = 0;
        for (int t = blockIdx.x; t < num_tiles; t += gridDim.x, ++tl) {
            int tm, tn;
            tile_coords(t, ntm, ntn, p.group_m, tm, tn);
            const uint32_t acc = tl & 1;
            const uint32_t aph = (tl >> 1) & 1;
            if (!bounded_wait(&tfull[acc], aph, abort_flag, limit, p.status)) break;
            tc_fence_after();
            epilogue_tile<Cfg::OUT, Cfg::BN, false, 2>(&tmC, p, tmem_base + acc * Cfg::BN, q, lane,
                                                       tm * Cfg::BM + q * 32, tn * Cfg::BN,
                                                       stg0, nstore);
            tc_fence_before();
            __syncwarp();
            if (lane == 0) mbar_arrive(&tempty[acc]);
        }
        if (lane == 0) bulk_wait<0>();
        __syncwarp();
    }

    tc_fence_before();
    __syncthreads();
    if (warp == 1) {
        tc_fence_after();
        tmem_dealloc(tmem_base, Cfg::TMEM_COLS);
    }
}

}  // namespace tg
