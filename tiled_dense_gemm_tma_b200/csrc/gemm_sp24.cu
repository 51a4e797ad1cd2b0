// gemm_sp24.cu -- 2:4 structured-sparse GEMM on the sparse tensor cores:
// C = epi(A . B) with A (M x K) stored compressed -- the two kept values of
// every chunk of 4 consecutive k (Ac, M x K/2) and a 4-bit position code per
// chunk (E, M rows of K/8 bytes: bits 0-1 / 2-3 give the positions of the
// first / second kept value, even chunk in the low nibble) -- and a dense,
// row-major B (K x N); fp16 or bf16 operands and output, fp32 accumulation.
// (The structured-sparse GEMM, T.gemm_sp with the 2:4 pattern, of
// "使用 Tilelang DSL 开发 GPU/CPU/加速器高性能内核", blog.hotdry.top,
// monitoring-and-debugging paragraph; the storage format is this library's
// reading.)
//
// tcgen05.mma.sp kind::f16 multiplies a 128 x 32 (dense k) A tile, held as
// 128 x 16 compressed values in shared memory, by a 32 x N B tile; the
// positions come from tensor memory, one 32-bit column per instruction:
// lane L holds, in bits 0-15, the codes of row (L & ~8) for the 16 dense k
// of half (L >> 3) & 1 of the instruction's 32, and in bits 16-31 those of
// row (L & ~8) + 8 (four codes per half, increasing k from bit 0).  Four
// consecutive instructions use four consecutive columns; an instruction
// names the even column of its pair and selects the column in the
// instruction descriptor (bits 0-1), beside the sparse flag (bit 2).
//
// Roles of one persistent CTA per SM, 128 x 256 output tiles:
//   warp 0      TMA producer: per 64 dense k (a stage), Ac (128 rows x 32
//               values, 64-byte swizzle) and B (64 rows x 4 x 64 columns,
//               128-byte swizzle); per 128 dense k (a block), the rows' 16
//               code bytes (E ring).
//   warps 6-9   metadata writers: per block, read rows (L & ~8) and
//               (L & ~8) + 8 of the E slot, pair their 16-bit halves into the
//               lane layout above and store 4 TMEM columns (tcgen05.st).
//   warp 1      MMA issuer: two sparse MMAs (K = 32 each) per stage into one
//               256-column fp32 accumulator.
//   warps 2-5   epilogue (gemm_tc.cuh: epilogue_tile): TMEM -> ReLU ->
//               round -> swizzled staging -> TMA store.
// The accumulator is single-buffered (the other half of TMEM holds the
// metadata ring), so a tile's epilogue does not overlap the next tile's
// MMAs; the loads for the next tile still run ahead.  Every wait is bounded.
#include "gemm_tc.cuh"
#include "host.cuh"
#include "launch.h"

namespace tg {

namespace {

struct SP {
    static constexpr int BM = 128, BN = 256;
    static constexpr int BKD = 64;                       // dense k per stage
    static constexpr int BKC = BKD / 2;                  // compressed values per stage
    static constexpr int STAGES = 4;
    static constexpr int A_STAGE = BM * BKC * 2;         // 8 KB: rows of 64 bytes
    static constexpr int B_CHUNK = BKD * 128;            // 8 KB: 64 columns x 64 rows
    static constexpr int B_STAGE = (BN / 64) * B_CHUNK;  // 32 KB
    static constexpr int E_BLOCK = BM * 16;              // 2 KB: 128 dense k of codes per row
    static constexpr int E_SLOTS = 2;
    static constexpr int MT_SLOTS = 4;                   // metadata blocks in tensor memory
    static constexpr int ACC_COLS = BN;                  // 256
    static constexpr int META_COL = ACC_COLS;            // metadata ring after the accumulator
    static constexpr int TMEM_COLS = 512;
    static constexpr int STG_BUF = 32 * 128;
    static constexpr int EPI_WARPS = 4, META_WARPS = 4;
    static constexpr int THREADS = 32 * (2 + EPI_WARPS + META_WARPS);
    static constexpr int GROUP_M = 16;
    static constexpr int SMEM_DATA = STAGES * (A_STAGE + B_STAGE) + E_SLOTS * E_BLOCK +
                                     EPI_WARPS * 2 * STG_BUF;
    static constexpr int SMEM_BYTES = SMEM_DATA + 512 + 1024;
    // Layout guards: the swizzled A (64-byte pattern, 512-byte period) and B
    // tiles and the staging buffers start on 1024-byte boundaries; the TMEM
    // columns fit the allocation; barriers fit their 512 bytes; one CTA fits
    // the 227 KB limit.
    static_assert(A_STAGE % 1024 == 0 && B_STAGE % 1024 == 0 && B_CHUNK % 1024 == 0, "swizzle");
    static_assert((STAGES * (A_STAGE + B_STAGE) + E_SLOTS * E_BLOCK) % 1024 == 0, "staging");
    static_assert(META_COL + 4 * MT_SLOTS <= TMEM_COLS, "TMEM columns");
    static_assert((2 * STAGES + 2 * E_SLOTS + 2 * MT_SLOTS + 3) * 8 + 8 <= 512, "barrier area");
    static_assert(SMEM_BYTES <= 227 * 1024, "shared memory per CTA");
    static_assert(BKD % 32 == 0 && 2 * BKD == 128, "a metadata block is two stages");
};

template <int FMT, OutT OUT>
__global__ void __launch_bounds__(SP::THREADS, 1)
sp24_gemm_kernel(const __grid_constant__ CUtensorMap tmA,
                 const __grid_constant__ CUtensorMap tmE,
                 const __grid_constant__ CUtensorMap tmB,
                 const __grid_constant__ CUtensorMap tmC,
                 const TcParams p) {
    extern __shared__ uint8_t smem_raw[];
    const uint32_t raw_addr = smem_u32(smem_raw);
    uint8_t* smem = smem_raw + (((raw_addr + 1023u) & ~1023u) - raw_addr);
    uint8_t* smA = smem;                                               // STAGES x 8 KB
    uint8_t* smB = smA + SP::STAGES * SP::A_STAGE;                     // STAGES x 32 KB
    uint8_t* smE = smB + SP::STAGES * SP::B_STAGE;                     // E_SLOTS x 2 KB
    uint8_t* smStg = smE + SP::E_SLOTS * SP::E_BLOCK;                  // epilogue staging
    uint64_t* bars = reinterpret_cast<uint64_t*>(smStg + SP::EPI_WARPS * 2 * SP::STG_BUF);
    uint64_t* full = bars;                                   // [STAGES] Ac + B landed
    uint64_t* empty = full + SP::STAGES;                     // [STAGES] MMAs done with them
    uint64_t* efull = empty + SP::STAGES;                    // [E_SLOTS] code bytes landed
    uint64_t* eempty = efull + SP::E_SLOTS;                  // [E_SLOTS] writers read them
    uint64_t* mfull = eempty + SP::E_SLOTS;                  // [MT_SLOTS] TMEM metadata written
    uint64_t* mempty = mfull + SP::MT_SLOTS;                 // [MT_SLOTS] MMAs done with it
    uint64_t* tfull = mempty + SP::MT_SLOTS;
    uint64_t* tempty = tfull + 1;
    uint64_t* drain = tempty + 1;
    uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(drain + 1);
    volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_slot + 1);

    const int warp = threadIdx.x >> 5;
    const int lane = threadIdx.x & 31;
    const int ntm = (p.M + SP::BM - 1) / SP::BM;
    const int ntn = (p.N + SP::BN - 1) / SP::BN;
    const int num_tiles = ntm * ntn;
    const int num_kb = (p.K + SP::BKD - 1) / SP::BKD;       // stages per tile
    const int num_blk = (num_kb + 1) / 2;                    // metadata blocks per tile
    const uint64_t limit = p.timeout_ns;

    if (threadIdx.x == 0) {
        for (int s = 0; s < SP::STAGES; ++s) { mbar_init(&full[s], 1); mbar_init(&empty[s], 1); }
        for (int e = 0; e < SP::E_SLOTS; ++e) { mbar_init(&efull[e], 1); mbar_init(&eempty[e], SP::META_WARPS); }
        for (int m = 0; m < SP::MT_SLOTS; ++m) { mbar_init(&mfull[m], SP::META_WARPS); mbar_init(&mempty[m], 1); }
        mbar_init(tfull, 1);
        mbar_init(tempty, SP::EPI_WARPS);
        mbar_init(drain, 1);
        *abort_flag = 0;
        fence_mbar_init();
        fence_proxy_async_smem();
    }
    if (warp == 1) {
        tmem_alloc(tmem_slot, SP::TMEM_COLS);
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
            tma_prefetch_desc(&tmE);
            tma_prefetch_desc(&tmB);
            tma_prefetch_desc(&tmC);
            uint32_t armed = 0, armed_par = 0, earmed = 0, earmed_par = 0, it = 0, gb = 0;
            bool ok = true;
            for (int t = blockIdx.x; t < num_tiles && ok; t += gridDim.x) {
                int tm, tn;
                tile_coords(t, ntm, ntn, p.group_m, tm, tn);
                const int m0 = tm * SP::BM, n0 = tn * SP::BN;
                // B boxes that start past column N only feed columns never stored
                const int b_live = min(SP::BN / 64, (p.N - n0 + 63) / 64);
                for (int kb = 0; kb < num_kb; ++kb, ++it) {
                    const uint32_t s = it % SP::STAGES;
                    const uint32_t ph = (it / SP::STAGES) & 1;
                    if (!bounded_wait(&empty[s], ph ^ 1, abort_flag, limit, p.status)) { ok = false; break; }
                    const bool new_blk = (kb & 1) == 0;
                    const uint32_t es = gb % SP::E_SLOTS, eph = (gb / SP::E_SLOTS) & 1;
                    if (new_blk && !bounded_wait(&eempty[es], eph ^ 1, abort_flag, limit, p.status)) {
                        ok = false;
                        break;
                    }
                    if (p.inject == 1 && it == 0 && blockIdx.x == 0) { gb += new_blk; continue; }   // debug
                    if (new_blk) {
                        mbar_arrive_expect_tx(&efull[es], SP::E_BLOCK);
                        earmed |= 1u << es;
                        earmed_par = (earmed_par & ~(1u << es)) | (eph << es);
                        tma_load_2d(smE + es * SP::E_BLOCK, &tmE, &efull[es], kb * (SP::BKD / 8), m0);
                        ++gb;
                    }
                    mbar_arrive_expect_tx(&full[s], SP::A_STAGE + b_live * SP::B_CHUNK);
                    armed |= 1u << s;
                    armed_par = (armed_par & ~(1u << s)) | (ph << s);
                    tma_load_2d(smA + s * SP::A_STAGE, &tmA, &full[s], kb * SP::BKC, m0);
                    for (int j = 0; j < b_live; ++j)
                        tma_load_2d(smB + s * SP::B_STAGE + j * SP::B_CHUNK, &tmB, &full[s],
                                    n0 + 64 * j, kb * SP::BKD);
                }
            }
            if (!ok) {
                // let this CTA's copies in flight land before it exits
                for (int s = 0; s < SP::STAGES; ++s)
                    if (armed & (1u << s)) {
                        volatile int never = 0;
                        bounded_wait(&full[s], (armed_par >> s) & 1, &never, limit, p.status);
                    }
                for (int e = 0; e < SP::E_SLOTS; ++e)
                    if (earmed & (1u << e)) {
                        volatile int never = 0;
                        bounded_wait(&efull[e], (earmed_par >> e) & 1, &never, limit, p.status);
                    }
            }
        }
        __syncwarp();
    } else if (warp == 1) {
        // ------------------------------------------------------- MMA issuer
        if (elect_one()) {
            constexpr uint32_t idesc0 = make_idesc(FMT, SP::BM, SP::BN, 0, 1) | (1u << 2);
            uint32_t it = 0, gb = 0, tl = 0;
            bool ok = true;
            for (int t = blockIdx.x; t < num_tiles && ok; t += gridDim.x, ++tl) {
                if (!bounded_wait(tempty, (tl & 1) ^ 1, abort_flag, limit, p.status)) { ok = false; break; }
                tc_fence_after();
                uint32_t mslot = 0;
                for (int kb = 0; kb < num_kb; ++kb, ++it) {
                    const uint32_t s = it % SP::STAGES;
                    const uint32_t ph = (it / SP::STAGES) & 1;
                    if ((kb & 1) == 0) {
                        mslot = gb % SP::MT_SLOTS;
                        if (!bounded_wait(&mfull[mslot], (gb / SP::MT_SLOTS) & 1, abort_flag, limit, p.status)) {
                            ok = false;
                            break;
                        }
                    }
                    if (!bounded_wait(&full[s], ph, abort_flag, limit, p.status)) { ok = false; break; }
                    tc_fence_after();
                    const uint32_t a_addr = smem_u32(smA + s * SP::A_STAGE);
                    const uint32_t b_addr = smem_u32(smB + s * SP::B_STAGE);
#pragma unroll
                    for (int j = 0; j < SP::BKD / 32; ++j) {
                        // A: K-major, 16 compressed values = 32 bytes inside the
                        // 64-byte swizzled rows; B: N-major, 32 k rows of 128 B
                        const uint64_t ad = sw128_desc(a_addr + j * 32, 16, 512, 4);
                        const uint64_t bd = sw128_desc(b_addr + j * 32 * 128, SP::B_CHUNK, 1024);
                        const uint32_t col = 2 * (kb & 1) + j;           // instruction in the block
                        const uint32_t e_addr = tmem_base + SP::META_COL + 4 * mslot + (col & ~1u);
                        mma_f16_sp(tmem_base, ad, bd, idesc0 | (col & 1u), (kb | j) != 0, e_addr);
                    }
                    mma_commit(&empty[s]);
                    if ((kb & 1) == 1 || kb == num_kb - 1) {
                        mma_commit(&mempty[mslot]);
                        ++gb;
                    }
                }
                if (!ok) break;
                mma_commit(tfull);
            }
            mma_commit(drain);
            volatile int never = 0;
            bounded_wait(drain, 0, &never, limit, p.status);
        }
        __syncwarp();
    } else if (warp < 2 + SP::EPI_WARPS) {
        // --------------------------------------------------------- epilogue
        const int q = warp & 3;
        uint8_t* stg0 = smStg + (warp - 2) * 2 * SP::STG_BUF;
        uint32_t tl = 0, nstore = 0;
        for (int t = blockIdx.x; t < num_tiles; t += gridDim.x, ++tl) {
            int tm, tn;
            tile_coords(t, ntm, ntn, p.group_m, tm, tn);
            if (!bounded_wait(tfull, tl & 1, abort_flag, limit, p.status)) break;
            tc_fence_after();
            epilogue_tile<OUT, SP::BN, false, 2>(&tmC, p, tmem_base, q, lane, tm * SP::BM + q * 32,
                                                 tn * SP::BN, stg0, nstore);
            tc_fence_before();
            __syncwarp();
            if (lane == 0) mbar_arrive(tempty);
        }
        if (lane == 0) bulk_wait<0>();
        __syncwarp();
    } else {
        // ------------------------------------------------- metadata writers
        const int quarter = warp & 3;                          // TMEM lanes this warp may access
        const int L = quarter * 32 + lane;
        const int rA = L & ~8;                                 // rows rA and rA + 8 ...
        const uint32_t sel = (L & 8) ? 0x7632u : 0x5410u;      // ... their k-half (L >> 3) & 1
        uint32_t gb = 0;
        bool ok = true;
        for (int t = blockIdx.x; t < num_tiles && ok; t += gridDim.x) {
            for (int b = 0; b < num_blk; ++b, ++gb) {
                const uint32_t es = gb % SP::E_SLOTS, ms = gb % SP::MT_SLOTS;
                if (!bounded_wait(&efull[es], (gb / SP::E_SLOTS) & 1, abort_flag, limit, p.status) ||
                    !bounded_wait(&mempty[ms], ((gb / SP::MT_SLOTS) & 1) ^ 1, abort_flag, limit, p.status)) {
                    ok = false;
                    break;
                }
                tc_fence_after();
                const uint8_t* eb = smE + es * SP::E_BLOCK;
                const uint4 ra = *reinterpret_cast<const uint4*>(eb + rA * 16);
                const uint4 rb = *reinterpret_cast<const uint4*>(eb + (rA + 8) * 16);
                __syncwarp();
                if (lane == 0) mbar_arrive(&eempty[es]);
                tmem_st_32x32b_x4(tmem_base + (static_cast<uint32_t>(quarter * 32) << 16) + SP::META_COL + 4 * ms,
                                  __byte_perm(ra.x, rb.x, sel), __byte_perm(ra.y, rb.y, sel),
                                  __byte_perm(ra.z, rb.z, sel), __byte_perm(ra.w, rb.w, sel));
                tmem_st_wait();
                tc_fence_before();
                __syncwarp();
                if (lane == 0) mbar_arrive(&mfull[ms]);
            }
        }
    }

    tc_fence_before();
    __syncthreads();
    if (warp == 1) {
        tc_fence_after();
        tmem_dealloc(tmem_base, SP::TMEM_COLS);
    }
}

// ------------------------------------------------------------ CTA pairs
//
// The same GEMM on CTA pairs (cta_group::2), 256 x 256 output tiles: CTA
// rank r of a pair stages the compressed A rows [128 r, 128 r + 128) of the
// tile, their position codes, and its half of the tile's B columns
// ([128 r, 128 r + 128)); its metadata writers fill its own tensor memory.
// The leader issues tcgen05.mma.sp.cta_group::2 with M = 256, N = 256: each
// SM reads 4 KB of compressed A and 4 KB of B per 32 dense k instead of
// 4 KB + 8 KB, and each CTA's TMEM receives its 128 rows x 256 columns.
//   full[s]    leader only: both producers arm it (count 2) with their own
//              byte counts; both CTAs' A and B copies complete on it.
//   empty[s], mempty[m], tfull   in each CTA: the leader's commits arrive on both.
//   efull / eempty   in each CTA (its own code bytes, its own writers).
//   mfull[m]   leader only: the writer warps of both CTAs (count 8), after
//              their tcgen05.st, wait::st and tcgen05 fence, with a plain
//              arrive on the cluster address (as the epilogue warps' arrive
//              on tempty).  An arrive with release at cluster scope made the
//              writers stall on a memory barrier: 969 us against 622 us at
//              8192^3.
//   tempty     leader only: the 8 epilogue warps of the pair.
struct SP2 {
    static constexpr int BM = 128, PM = 256, BN = 256, HN = 128;
    static constexpr int BKD = 64, BKC = 32;
    static constexpr int STAGES = 7;
    static constexpr int A_STAGE = BM * BKC * 2;         // 8 KB
    static constexpr int B_CHUNK = BKD * 128;            // 8 KB: 64 columns x 64 rows
    static constexpr int B_STAGE = (HN / 64) * B_CHUNK;  // 16 KB
    static constexpr int E_BLOCK = BM * 16;
    static constexpr int E_SLOTS = 2;
    static constexpr int MT_SLOTS = 4;
    static constexpr int ACC_COLS = BN;
    static constexpr int META_COL = ACC_COLS;
    static constexpr int TMEM_COLS = 512;
    static constexpr int STG_BUF = 32 * 128;
    static constexpr int EPI_WARPS = 4, META_WARPS = 4;
    static constexpr int THREADS = 32 * (2 + EPI_WARPS + META_WARPS);
    static constexpr int GROUP_M = 8;                    // pair-tile rows per raster band
    static constexpr int SMEM_DATA = STAGES * (A_STAGE + B_STAGE) + E_SLOTS * E_BLOCK +
                                     EPI_WARPS * 2 * STG_BUF;
    static constexpr int SMEM_BYTES = SMEM_DATA + 512 + 1024;
    static_assert(A_STAGE % 1024 == 0 && B_STAGE % 1024 == 0 && B_CHUNK % 1024 == 0, "swizzle");
    static_assert((STAGES * (A_STAGE + B_STAGE) + E_SLOTS * E_BLOCK) % 1024 == 0, "staging");
    static_assert(META_COL + 4 * MT_SLOTS <= TMEM_COLS, "TMEM columns");
    static_assert((2 * STAGES + 2 * E_SLOTS + 2 * MT_SLOTS + 3) * 8 + 8 <= 512, "barrier area");
    static_assert(SMEM_BYTES <= 227 * 1024, "shared memory per CTA");
    static_assert(2 * BKD == 128, "a metadata block is two stages");
};

template <int FMT, OutT OUT>
__global__ void __launch_bounds__(SP2::THREADS, 1)
sp24_pair_kernel(const __grid_constant__ CUtensorMap tmA,
                 const __grid_constant__ CUtensorMap tmE,
                 const __grid_constant__ CUtensorMap tmB,
                 const __grid_constant__ CUtensorMap tmC,
                 const TcParams p) {
    extern __shared__ uint8_t smem_raw[];
    const uint32_t raw_addr = smem_u32(smem_raw);
    uint8_t* smem = smem_raw + (((raw_addr + 1023u) & ~1023u) - raw_addr);
    uint8_t* smA = smem;
    uint8_t* smB = smA + SP2::STAGES * SP2::A_STAGE;
    uint8_t* smE = smB + SP2::STAGES * SP2::B_STAGE;
    uint8_t* smStg = smE + SP2::E_SLOTS * SP2::E_BLOCK;
    uint64_t* bars = reinterpret_cast<uint64_t*>(smStg + SP2::EPI_WARPS * 2 * SP2::STG_BUF);
    uint64_t* full = bars;
    uint64_t* empty = full + SP2::STAGES;
    uint64_t* efull = empty + SP2::STAGES;
    uint64_t* eempty = efull + SP2::E_SLOTS;
    uint64_t* mfull = eempty + SP2::E_SLOTS;
    uint64_t* mempty = mfull + SP2::MT_SLOTS;
    uint64_t* tfull = mempty + SP2::MT_SLOTS;
    uint64_t* tempty = tfull + 1;
    uint64_t* drain = tempty + 1;
    uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(drain + 1);
    volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_slot + 1);

    const int warp = threadIdx.x >> 5;
    const int lane = threadIdx.x & 31;
    const uint32_t rank = cluster_ctarank();
    const int pair = blockIdx.x >> 1;
    const int npairs = gridDim.x >> 1;
    const int ntm = (p.M + SP2::PM - 1) / SP2::PM;
    const int ntn = (p.N + SP2::BN - 1) / SP2::BN;
    const int num_tiles = ntm * ntn;
    const int num_kb = (p.K + SP2::BKD - 1) / SP2::BKD;
    const int num_blk = (num_kb + 1) / 2;
    const uint64_t limit = p.timeout_ns;

    if (threadIdx.x == 0) {
        for (int s = 0; s < SP2::STAGES; ++s) { mbar_init(&full[s], 2); mbar_init(&empty[s], 1); }
        for (int e = 0; e < SP2::E_SLOTS; ++e) { mbar_init(&efull[e], 1); mbar_init(&eempty[e], SP2::META_WARPS); }
        for (int m = 0; m < SP2::MT_SLOTS; ++m) { mbar_init(&mfull[m], 2 * SP2::META_WARPS); mbar_init(&mempty[m], 1); }
        mbar_init(tfull, 1);
        mbar_init(tempty, 2 * SP2::EPI_WARPS);
        mbar_init(drain, 1);
        *abort_flag = 0;
        fence_mbar_init();
        fence_proxy_async_smem();
    }
    if (warp == 0 && lane == 0) {
        tma_prefetch_desc(&tmA);
        tma_prefetch_desc(&tmE);
        tma_prefetch_desc(&tmB);
        tma_prefetch_desc(&tmC);
    }
    if (warp == 1) {
        tmem_alloc_pair(tmem_slot, SP2::TMEM_COLS);
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
            uint32_t armed = 0, armed_par = 0, earmed = 0, earmed_par = 0, it = 0, gb = 0;
            bool ok = true;
            for (int t = pair; t < num_tiles && ok; t += npairs) {
                int tm, tn;
                tile_coords(t, ntm, ntn, p.group_m, tm, tn);
                const int m0 = tm * SP2::PM + rank * SP2::BM;
                const int n0 = tn * SP2::BN + rank * SP2::HN;
                // boxes entirely past the matrix edge only feed outputs never stored
                const bool a_live = m0 < p.M;
                const int b_live = n0 >= p.N ? 0 : (n0 + 64 < p.N ? 2 : 1);
                const uint32_t bytes = (a_live ? SP2::A_STAGE : 0) + b_live * SP2::B_CHUNK;
                for (int kb = 0; kb < num_kb; ++kb, ++it) {
                    const uint32_t s = it % SP2::STAGES;
                    const uint32_t ph = (it / SP2::STAGES) & 1;
                    if (!bounded_wait(&empty[s], ph ^ 1, abort_flag, limit, p.status)) { ok = false; break; }
                    const bool new_blk = (kb & 1) == 0;
                    const uint32_t es = gb % SP2::E_SLOTS, eph = (gb / SP2::E_SLOTS) & 1;
                    if (new_blk && !bounded_wait(&eempty[es], eph ^ 1, abort_flag, limit, p.status)) {
                        ok = false;
                        break;
                    }
                    if (p.inject == 1 && it == 0 && pair == 0 && rank == 0) { gb += new_blk; continue; }   // debug
                    if (new_blk) {
                        mbar_arrive_expect_tx(&efull[es], SP2::E_BLOCK);
                        earmed |= 1u << es;
                        earmed_par = (earmed_par & ~(1u << es)) | (eph << es);
                        tma_load_2d(smE + es * SP2::E_BLOCK, &tmE, &efull[es], kb * (SP2::BKD / 8), m0);
                        ++gb;
                    }
                    const uint32_t fbar = mapa_shared(smem_u32(&full[s]), 0);
                    mbar_arrive_expect_tx_cluster(fbar, bytes);
                    armed |= 1u << s;
                    armed_par = (armed_par & ~(1u << s)) | (ph << s);
                    if (a_live)
                        tma_load_2d_pair(smA + s * SP2::A_STAGE, &tmA, fbar, kb * SP2::BKC, m0);
                    for (int j = 0; j < b_live; ++j)
                        tma_load_2d_pair(smB + s * SP2::B_STAGE + j * SP2::B_CHUNK, &tmB, fbar,
                                         n0 + 64 * j, kb * SP2::BKD);
                }
            }
            if (!ok) {
                for (int e = 0; e < SP2::E_SLOTS; ++e)
                    if (earmed & (1u << e)) {
                        volatile int never = 0;
                        bounded_wait(&efull[e], (earmed_par >> e) & 1, &never, limit, p.status);
                    }
                if (rank == 0) {
                    for (int s = 0; s < SP2::STAGES; ++s)
                        if (armed & (1u << s)) {
                            volatile int never = 0;
                            bounded_wait(&full[s], (armed_par >> s) & 1, &never, limit, p.status);
                        }
                } else {
                    // this CTA's operand copies complete on the leader's barriers,
                    // which it cannot wait on: give copies in flight 1 ms to land
                    const uint64_t t0 = globaltimer_ns();
                    while (globaltimer_ns() - t0 < 1000000ull) __nanosleep(10000);
                }
            }
        }
        __syncwarp();
    } else if (warp == 1) {
        // ------------------------------------------ MMA issuer (leader only)
        if (rank == 0 && elect_one()) {
            constexpr uint32_t idesc0 = make_idesc(FMT, SP2::PM, SP2::BN, 0, 1) | (1u << 2);
            uint32_t it = 0, gb = 0, tl = 0;
            bool ok = true;
            for (int t = pair; t < num_tiles && ok; t += npairs, ++tl) {
                if (!bounded_wait(tempty, (tl & 1) ^ 1, abort_flag, limit, p.status)) { ok = false; break; }
                tc_fence_after();
                uint32_t mslot = 0;
                for (int kb = 0; kb < num_kb; ++kb, ++it) {
                    const uint32_t s = it % SP2::STAGES;
                    const uint32_t ph = (it / SP2::STAGES) & 1;
                    if ((kb & 1) == 0) {
                        mslot = gb % SP2::MT_SLOTS;
                        if (!bounded_wait(&mfull[mslot], (gb / SP2::MT_SLOTS) & 1, abort_flag, limit,
                                          p.status)) {
                            ok = false;
                            break;
                        }
                    }
                    if (!bounded_wait(&full[s], ph, abort_flag, limit, p.status)) { ok = false; break; }
                    tc_fence_after();
                    const uint32_t a_addr = smem_u32(smA + s * SP2::A_STAGE);
                    const uint32_t b_addr = smem_u32(smB + s * SP2::B_STAGE);
#pragma unroll
                    for (int j = 0; j < SP2::BKD / 32; ++j) {
                        const uint64_t ad = sw128_desc(a_addr + j * 32, 16, 512, 4);
                        const uint64_t bd = sw128_desc(b_addr + j * 32 * 128, SP2::B_CHUNK, 1024);
                        const uint32_t col = 2 * (kb & 1) + j;
                        const uint32_t e_addr = tmem_base + SP2::META_COL + 4 * mslot + (col & ~1u);
                        mma_f16_sp_pair(tmem_base, ad, bd, idesc0 | (col & 1u), (kb | j) != 0, e_addr);
                    }
                    const uint32_t e_loc = smem_u32(&empty[s]);
                    mma_commit_pair(mapa_shared(e_loc, 0));
                    mma_commit_pair(mapa_shared(e_loc, 1));
                    if ((kb & 1) == 1 || kb == num_kb - 1) {
                        const uint32_t m_loc = smem_u32(&mempty[mslot]);
                        mma_commit_pair(mapa_shared(m_loc, 0));
                        mma_commit_pair(mapa_shared(m_loc, 1));
                        ++gb;
                    }
                }
                if (!ok) break;
                const uint32_t f_loc = smem_u32(tfull);
                mma_commit_pair(mapa_shared(f_loc, 0));
                mma_commit_pair(mapa_shared(f_loc, 1));
            }
            mma_commit_pair(mapa_shared(smem_u32(drain), 0));
            volatile int never = 0;
            bounded_wait(drain, 0, &never, limit, p.status);
        }
        __syncwarp();
    } else if (warp < 2 + SP2::EPI_WARPS) {
        // --------------------------------------------------- epilogue (both)
        const int q = warp & 3;
        uint8_t* stg0 = smStg + (warp - 2) * 2 * SP2::STG_BUF;
        uint32_t tl = 0, nstore = 0;
        for (int t = pair; t < num_tiles; t += npairs, ++tl) {
            int tm, tn;
            tile_coords(t, ntm, ntn, p.group_m, tm, tn);
            if (!bounded_wait(tfull, tl & 1, abort_flag, limit, p.status)) break;
            tc_fence_after();
            epilogue_tile<OUT, SP2::BN, false, 2>(&tmC, p, tmem_base, q, lane,
                                                  tm * SP2::PM + rank * SP2::BM + q * 32,
                                                  tn * SP2::BN, stg0, nstore);
            tc_fence_before();
            __syncwarp();
            if (lane == 0) mbar_arrive_cluster(mapa_shared(smem_u32(tempty), 0));
        }
        if (lane == 0) bulk_wait<0>();
        __syncwarp();
    } else {
        // ------------------------------------------- metadata writers (both)
        const int quarter = warp & 3;
        const int L = quarter * 32 + lane;
        const int rA = L & ~8;
        const uint32_t sel = (L & 8) ? 0x7632u : 0x5410u;
        uint32_t gb = 0;
        bool ok = true;
        for (int t = pair; t < num_tiles && ok; t += npairs) {
            for (int b = 0; b < num_blk; ++b, ++gb) {
                const uint32_t es = gb % SP2::E_SLOTS, ms = gb % SP2::MT_SLOTS;
                if (!bounded_wait(&efull[es], (gb / SP2::E_SLOTS) & 1, abort_flag, limit, p.status) ||
                    !bounded_wait(&mempty[ms], ((gb / SP2::MT_SLOTS) & 1) ^ 1, abort_flag, limit, p.status)) {
                    ok = false;
                    break;
                }
                tc_fence_after();
                const uint8_t* eb = smE + es * SP2::E_BLOCK;
                const uint4 ra = *reinterpret_cast<const uint4*>(eb + rA * 16);
                const uint4 rb = *reinterpret_cast<const uint4*>(eb + (rA + 8) * 16);
                __syncwarp();
                if (lane == 0) mbar_arrive(&eempty[es]);
                tmem_st_32x32b_x4(tmem_base + (static_cast<uint32_t>(quarter * 32) << 16) + SP2::META_COL + 4 * ms,
                                  __byte_perm(ra.x, rb.x, sel), __byte_perm(ra.y, rb.y, sel),
                                  __byte_perm(ra.z, rb.z, sel), __byte_perm(ra.w, rb.w, sel));
                tmem_st_wait();
                tc_fence_before();
                __syncwarp();
                if (lane == 0) mbar_arrive_cluster(mapa_shared(smem_u32(&mfull[ms]), 0));
            }
        }
    }

    tc_fence_before();
    __syncthreads();
    cluster_sync_all();          // the pair is done with each other's barriers and TMEM
    if (warp == 1) {
        tc_fence_after();
        tmem_dealloc_pair(tmem_base, SP2::TMEM_COLS);
    }
}

template <int FMT, OutT OUT>
int run_sp24_pair(const GemmArgs& a, const void* E, int64_t lde, CUtensorMapDataType dt, int slot) {
    if (pair_kernels_disabled()) return kUnsupported;
    int dev = 0;
    const DeviceInfo* di = current_device(&dev);
    if (!di) return kNoDevice;
    CUtensorMap tA, tE, tB, tC;
    if (!tensor_map_2d(&tA, a.A, dt, 2, a.K / 2, a.M, a.lda * 2, SP2::BKC, SP2::BM, SWZ_64))
        return kCudaError;
    if (!tensor_map_2d(&tE, E, CU_TENSOR_MAP_DATA_TYPE_UINT8, 1, (a.K + 7) / 8, a.M, lde, 16, SP2::BM,
                       SWZ_NONE))
        return kCudaError;
    if (!tensor_map_2d(&tB, a.B, dt, 2, a.N, a.K, a.ldb * 2, 64, SP2::BKD, SWZ_128))
        return kCudaError;
    if (!tensor_map_2d(&tC, a.C, dt, 2, a.N, a.M, a.ldc * 2, 64, 32, SWZ_128))
        return kCudaError;
    auto kern = sp24_pair_kernel<FMT, OUT>;
    if (set_smem_attr(reinterpret_cast<const void*>(kern), SP2::SMEM_BYTES, slot) != cudaSuccess)
        return kCudaError;
    const long long tiles = ((a.M + SP2::PM - 1) / SP2::PM) * ((a.N + SP2::BN - 1) / SP2::BN);
    const int npairs = static_cast<int>(persistent_grid(tiles, di->num_sms / 2, a.ctas));
    TcParams p = {};
    p.M = static_cast<int>(a.M);
    p.N = static_cast<int>(a.N);
    p.K = static_cast<int>(a.K);
    p.relu = a.relu;
    p.group_m = a.group_m > 0 ? a.group_m : SP2::GROUP_M;
    p.inject = inject_mode();
    p.timeout_ns = wait_limit_ns();
    p.status = device_status_ptr();
    p.C = a.C;
    p.ldc = a.ldc;
    if (!p.status) return kCudaError;
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3(2 * npairs, 1, 1);
    cfg.blockDim = dim3(SP2::THREADS, 1, 1);
    cfg.dynamicSmemBytes = SP2::SMEM_BYTES;
    cfg.stream = static_cast<cudaStream_t>(a.stream);
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeClusterDimension;
    attr[0].val.clusterDim.x = 2;
    attr[0].val.clusterDim.y = 1;
    attr[0].val.clusterDim.z = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    if (cudaLaunchKernelEx(&cfg, kern, tA, tE, tB, tC, p) != cudaSuccess) {
        cudaGetLastError();                       // clear; the caller falls back
        return kUnsupported;
    }
    return kOk;
}

template <int FMT, OutT OUT>
int run_sp24(const GemmArgs& a, const void* E, int64_t lde, CUtensorMapDataType dt, int slot) {
    int dev = 0;
    const DeviceInfo* di = current_device(&dev);
    if (!di) return kNoDevice;
    CUtensorMap tA, tE, tB, tC;
    // Ac: K/2 values per row; boxes of 32 values (64 bytes) x 128 rows
    if (!tensor_map_2d(&tA, a.A, dt, 2, a.K / 2, a.M, a.lda * 2, SP::BKC, SP::BM, SWZ_64))
        return kCudaError;
    // E: ceil(K/8) bytes per row; boxes of 16 bytes (128 dense k) x 128 rows
    if (!tensor_map_2d(&tE, E, CU_TENSOR_MAP_DATA_TYPE_UINT8, 1, (a.K + 7) / 8, a.M, lde, 16, SP::BM,
                       SWZ_NONE))
        return kCudaError;
    if (!tensor_map_2d(&tB, a.B, dt, 2, a.N, a.K, a.ldb * 2, 64, SP::BKD, SWZ_128))
        return kCudaError;
    if (!tensor_map_2d(&tC, a.C, dt, 2, a.N, a.M, a.ldc * 2, 64, 32, SWZ_128))
        return kCudaError;
    auto kern = sp24_gemm_kernel<FMT, OUT>;
    if (set_smem_attr(reinterpret_cast<const void*>(kern), SP::SMEM_BYTES, slot) != cudaSuccess)
        return kCudaError;
    const long long tiles = ((a.M + SP::BM - 1) / SP::BM) * ((a.N + SP::BN - 1) / SP::BN);
    const int grid = static_cast<int>(persistent_grid(tiles, di->num_sms, a.ctas));
    TcParams p = {};
    p.M = static_cast<int>(a.M);
    p.N = static_cast<int>(a.N);
    p.K = static_cast<int>(a.K);
    p.relu = a.relu;
    p.group_m = a.group_m > 0 ? a.group_m : SP::GROUP_M;
    p.inject = inject_mode();
    p.timeout_ns = wait_limit_ns();
    p.status = device_status_ptr();
    p.C = a.C;
    p.ldc = a.ldc;
    if (!p.status) return kCudaError;
    kern<<<grid, SP::THREADS, SP::SMEM_BYTES, static_cast<cudaStream_t>(a.stream)>>>(tA, tE, tB, tC, p);
    return cudaGetLastError() == cudaSuccess ? kOk : kCudaError;
}

}  // namespace

// a.A = Ac (values), a.lda = its row pitch (elements); E / lde (bytes).
// CTA pairs unless the tuning table asks for one CTA per tile or the device
// refuses the cluster launch.
int launch_sp24(const GemmArgs& a, const void* E, int64_t lde, int bf16) {
    if (a.path != PATH_ONE_CTA) {
        const int r = bf16 ? run_sp24_pair<1, OutT::BF16>(a, E, lde, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 61)
                           : run_sp24_pair<0, OutT::F16>(a, E, lde, CU_TENSOR_MAP_DATA_TYPE_FLOAT16, 62);
        if (r != kUnsupported) return r;
    }
    return bf16 ? run_sp24<1, OutT::BF16>(a, E, lde, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 56)
                : run_sp24<0, OutT::F16>(a, E, lde, CU_TENSOR_MAP_DATA_TYPE_FLOAT16, 57);
}

}  // namespace tg
