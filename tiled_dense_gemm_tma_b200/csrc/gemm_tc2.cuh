// gemm_tc2.cuh -- the fp16 / bf16 GEMM and the TF32 mode of the fp32 GEMM
// on CTA pairs (tcgen05 cta_group::2).
//
// Same warp roles as gemm_tc.cuh, but two CTAs on neighbouring SMs (a
// cluster of 2) share one 256 x 256 output tile: CTA rank r owns rows
// [128 r, 128 r + 128) of the tile and stages its own A rows and its own half
// of the tile's B columns ([128 r, 128 r + 128)).  The leader (rank 0) issues
// tcgen05.mma.cta_group::2 with M = 256, N = 256: the tensor cores of both
// SMs read A from their own CTA and B from both, and each CTA's TMEM receives
// its 128 rows x 256 columns.  Per MMA each SM reads 4 KB of A and 4 KB of B
// from its shared memory instead of 4 KB + 8 KB in the single-CTA kernel,
// which relieves the shared-memory -> tensor-core path.  TF32 (fp32
// operands, kind::tf32, fp32 output): the same 128-byte rows hold 32 k, B
// arrives in 32-column boxes with the 32-byte-unit swizzle the tensor core
// requires for MN-major 32-bit data, and each MMA covers 8 k.
//
// Synchronisation across the pair:
//   full[s]   leader only; both producers arm it (count 2) with their own byte
//             counts, and both CTAs' TMA loads complete on it (.cta_group::2).
//   empty[s]  in each CTA; the leader's MMA commit arrives on both.
//   tfull[a]  in each CTA; the leader's MMA commit arrives on both.
//   tempty[a] leader only; all 8 epilogue warps of the pair arrive (count 8).
//
// Hybrid schedule (tail_split / tail_item of tile_sched.h): whole tiles fill
// the full waves; if the last wave holds at most half as many tiles as there
// are pairs, each of those tiles is split into two halves of its k-blocks.
// Per CTA (its 128 rows) the two halves meet through the workspace: each
// checks in on a counter; the first writes its fp32 partial and publishes
// it; the second waits for that, adds the partial into its accumulator in
// TMEM and runs the ordinary epilogue (a + b is exact-order free: the two
// possible orders give the same bits).  A half is the last item of its pair,
// so its operand ring is idle by then: the partial goes out and comes in
// through the ring by 128 KB bulk copies.
// Operand-swapped mode (TOUT, 128-column pair tiles) for M <= 128: the
// caller passes B^T as A and A^T as B, so the kernel computes C^T with the
// weight columns as its 256-row side and the M activation rows as its
// 128-column side.  Each CTA then stages 128 weight columns and 64 of the
// activation rows, where the plain form has one CTA of the pair staging all
// M rows of A and its partner none; the epilogue writes the tile transposed.
// Loads are plain tiled TMA copies: each CTA reads only its own tiles into
// its own shared memory.  Every wait is bounded; the CTAs meet on a cluster
// barrier after set-up and before freeing TMEM.
#pragma once
#include "gemm_tc.cuh"

namespace tg {

// A_MN_ = 1: A is stored transposed (K x M row-major), so its tiles arrive
// M-major (64-row boxes along M) and the MMA reads A MN-major.  B_MN_ = 0: B
// is stored transposed (N x K row-major) and is read K-major.  The default
// (0, 1) is the row-major A (M x K) and B (K x N) of the plain GEMM.
// BN_: columns of a pair tile (256, or 128: each CTA stages 64 B columns).
// TOUT_ = 1: the kernel computes the transpose D = C^T of the output (the
// caller swaps the operands) and writes it transposed into C.
template <int FMT_, OutT OUT_, int STAGES_, int A_MN_ = 0, int B_MN_ = 1, int BN_ = 256, int TOUT_ = 0>
struct Tc2Cfg {
    static constexpr int FMT = FMT_;                    // idesc format: 0 f16, 1 bf16, 2 tf32
    static constexpr OutT OUT = OUT_;
    static constexpr int A_MN = A_MN_;
    static constexpr int B_MN = B_MN_;
    static constexpr int IN_BYTES = FMT_ == 2 ? 4 : 2;
    static constexpr int OUT_BYTES = OUT_ == OutT::F32 ? 4 : 2;
    static constexpr int BM = 128;                      // rows per CTA
    static constexpr int PM = 256;                      // rows per pair tile
    static constexpr int TOUT = TOUT_;
    static constexpr int BN = BN_;                      // columns per pair tile
    static constexpr int HN = BN_ / 2;                  // B columns staged per CTA
    static_assert(BN_ == 256 || BN_ == 128, "pair tile width");
    // TF32: the plain layout only (A M x K, B K x N, 256-column tiles), fp32 out
    static_assert(FMT_ != 2 || (A_MN_ == 0 && B_MN_ == 1 && BN_ == 256 && TOUT_ == 0 && OUT_ == OutT::F32),
                  "TF32 pair configuration");
    static constexpr int BK = 128 / IN_BYTES;           // k per 128-byte swizzle row: 64 or 32
    static constexpr int MMA_K = 32 / IN_BYTES;         // k per MMA: 16 or 8
    static constexpr int CHUNK_N = 128 / IN_BYTES;      // B columns per MN-major box row
    static constexpr int STAGES = STAGES_;
    static constexpr int A_STAGE = BM * 128;            // 16 KB
    static constexpr int A_CHUNK = BK * 128;            // 8 KB: 64 rows of A x 64 k (M-major A)
    static constexpr int B_CHUNK = BK * 128;            // CHUNK_N columns x BK rows: 8 KB / 4 KB
    static constexpr int B_STAGE = (HN / CHUNK_N) * B_CHUNK;   // 16 KB (K-major B: HN rows x 128 B)
    // MN-major B: 16-bit data in the 8-row swizzle atom, tf32 in the 4-row one
    static constexpr uint32_t B_LAYOUT = IN_BYTES == 4 ? 1u : 2u;
    static constexpr uint32_t B_SBO = IN_BYTES == 4 ? 512u : 1024u;
    static constexpr int STG_BUF = 32 * 128;
    static_assert(STG_BUF == 64 * 64, "a staging buffer holds 32 x 128 bytes or, transposed, 64 x 64");
    static constexpr int EPI_WARPS = 4;
    static constexpr int TMEM_COLS = 2 * BN;            // 512: double-buffered accumulator
    static constexpr int THREADS = 64 + 32 * EPI_WARPS;
    static constexpr int GROUP_M = 8;                   // pair-tile rows per raster band
    static constexpr int SMEM_DATA = STAGES * (A_STAGE + B_STAGE) + EPI_WARPS * 2 * STG_BUF;
    static constexpr int PART_BYTES = BM * BN * 4;      // one CTA's fp32 partial of a split tile
    static_assert(STAGES * (A_STAGE + B_STAGE) >= PART_BYTES, "the ring holds a partial");
    static constexpr int SMEM_BYTES = SMEM_DATA + 256 + 1024;
};

// Epilogue of an operand-swapped tile: the accumulator holds D = C^T (a
// TMEM lane is a column n of C, a TMEM column a row m of C; p.M and p.N are
// the kernel's dimensions, N and M of C).  For each 64 rows m, lane n stores
// its 64 values down column n of a [64 m][32 n] staging tile, so each row of
// the tile is one contiguous 64-byte run, and one TMA store writes the tile
// into C at (column n0, row m0): the copy engine drops the rows past M and
// the columns past N, the latter in whole 16-byte units, so a column tail
// that is not a whole number of them is written with plain stores instead.
// The staging buffer is the 4 KB of the plain epilogue.
template <OutT OUT, int BN, int NBUF>
__device__ __forceinline__ void epilogue_tile_t(const CUtensorMap* tmC, const TcParams& p,
                                                uint32_t tmem_tile, int q, int lane,
                                                int n0, int m_base, uint8_t* stg0,
                                                uint32_t& nstore) {
    static_assert(OUT != OutT::F32, "16-bit output");
    constexpr int STG_BUF = 64 * 64;
    if (n0 >= p.M) return;                                 // warp-uniform
#pragma unroll 1
    for (int c = 0; c < BN / 64; ++c) {
        const int m0 = m_base + 64 * c;
        if (m0 >= p.N) break;
        const uint32_t taddr = tmem_tile + (static_cast<uint32_t>(q * 32) << 16) + 64 * c;
        uint32_t v[64];
        tmem_ld_32x32b_x32(taddr, *reinterpret_cast<uint32_t(*)[32]>(&v[0]));
        tmem_ld_32x32b_x32(taddr + 32, *reinterpret_cast<uint32_t(*)[32]>(&v[32]));
        tmem_ld_wait();
        auto out16 = [&](int j) -> uint16_t {
            float x = __uint_as_float(v[j]);
            if (p.relu) x = fmaxf(x, 0.f);
            if constexpr (OUT == OutT::BF16) return __bfloat16_as_ushort(__float2bfloat16_rn(x));
            else return __half_as_ushort(__float2half_rn(x));
        };
        const int ncols = p.M - n0;                        // columns of C left from n0
        if (ncols < 32 && (ncols * 2) % 16 != 0) {
            // lane n writes its column; per row the lanes' stores are contiguous
            if (lane < ncols) {
                uint16_t* dst = static_cast<uint16_t*>(p.C) + static_cast<long long>(m0) * p.ldc + n0 + lane;
                const int rows = p.N - m0;
#pragma unroll
                for (int j = 0; j < 64; ++j)
                    if (j < rows) dst[static_cast<long long>(j) * p.ldc] = out16(j);
            }
            continue;
        }
        uint8_t* stg = stg0 + (nstore % NBUF) * STG_BUF;
        if (lane == 0) bulk_wait_read<NBUF - 1>();         // this buffer's last store has read it
        __syncwarp();
        uint16_t* col = reinterpret_cast<uint16_t*>(stg) + lane;
#pragma unroll
        for (int j = 0; j < 64; ++j) col[32 * j] = out16(j);
        fence_proxy_async_smem();
        __syncwarp();
        if (lane == 0) {
            tma_store_2d(tmC, stg, n0, m0);
            bulk_commit();
        }
        ++nstore;
    }
}

template <class Cfg>
__global__ void __launch_bounds__(Cfg::THREADS, 1)
tc2_gemm_kernel(const __grid_constant__ CUtensorMap tmA,
                const __grid_constant__ CUtensorMap tmB,
                const __grid_constant__ CUtensorMap tmC,
                const TcParams p) {
    extern __shared__ uint8_t smem_raw[];
    const uint32_t raw = smem_u32(smem_raw);
    uint8_t* smem = smem_raw + (((raw + 1023u) & ~1023u) - raw);
    uint8_t* smA = smem;
    uint8_t* smB = smA + Cfg::STAGES * Cfg::A_STAGE;
    uint8_t* smStg = smB + Cfg::STAGES * Cfg::B_STAGE;
    uint64_t* bars = reinterpret_cast<uint64_t*>(smStg + Cfg::EPI_WARPS * 2 * Cfg::STG_BUF);
    uint64_t* full = bars;
    uint64_t* empty = full + Cfg::STAGES;
    uint64_t* tfull = empty + Cfg::STAGES;
    uint64_t* tempty = tfull + 2;
    uint64_t* drain = tempty + 2;
    uint64_t* epi_bar = drain + 1;             // this CTA's epilogue warps joined (count 4)
    uint64_t* flag_bar = epi_bar + 1;          // check-in result published (count 1)
    uint64_t* xbar = flag_bar + 1;             // a partner's partial landed in the ring
    uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(xbar + 1);
    volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_slot + 1);
    volatile int* tail_flag = abort_flag + 1;      // [0] check-in result, [1] partner published

    const int warp = threadIdx.x >> 5;
    const int lane = threadIdx.x & 31;
    const uint32_t rank = cluster_ctarank();
    const int pair = blockIdx.x >> 1;
    const int npairs = gridDim.x >> 1;
    const int ntm = (p.M + Cfg::PM - 1) / Cfg::PM;
    const int ntn = (p.N + Cfg::BN - 1) / Cfg::BN;
    const int num_tiles = ntm * ntn;
    const int num_kb = (p.K + Cfg::BK - 1) / Cfg::BK;
    const int S = p.tail_split > 1 ? p.tail_split : 1;
    const int dp = S > 1 ? p.dp_tiles : num_tiles;
    const int num_items = tail_items(num_tiles, dp, S);
    const uint64_t limit = p.timeout_ns;

    if (threadIdx.x == 0) {
        for (int s = 0; s < Cfg::STAGES; ++s) { mbar_init(&full[s], 2); mbar_init(&empty[s], 1); }
        for (int a = 0; a < 2; ++a) { mbar_init(&tfull[a], 1); mbar_init(&tempty[a], 2 * Cfg::EPI_WARPS); }
        mbar_init(drain, 1);
        mbar_init(epi_bar, Cfg::EPI_WARPS);
        mbar_init(flag_bar, 1);
        mbar_init(xbar, 1);
        *abort_flag = 0;
        tail_flag[0] = 0;
        tail_flag[1] = 0;
        fence_mbar_init();
        fence_proxy_async_smem();
    }
    if (warp == 0 && lane == 0) {
        tma_prefetch_desc(&tmA);
        tma_prefetch_desc(&tmB);
        tma_prefetch_desc(&tmC);
    }
    if (warp == 1) {
        tmem_alloc_pair(tmem_slot, Cfg::TMEM_COLS);
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
            uint32_t armed = 0, armed_par = 0, it = 0;
            bool ok = true;
            for (int w = pair; w < num_items && ok; w += npairs) {
                int t, kb0, kb1, z;
                tail_item(w, dp, S, num_kb, t, kb0, kb1, z);
                int tm, tn;
                tile_coords(t, ntm, ntn, p.group_m, tm, tn);
                const int m0 = tm * Cfg::PM + rank * Cfg::BM;
                const int n0 = tn * Cfg::BN + rank * Cfg::HN;
                // boxes entirely past the matrix edge are not loaded: they only
                // feed output rows / columns that are never stored
                // 64-wide chunks of A rows, CHUNK_N-wide chunks of B columns,
                // that start inside the matrix
                const int a_live = m0 >= p.M ? 0 : (m0 + 64 < p.M ? 2 : 1);
                const int b_left = (p.N - n0 + Cfg::CHUNK_N - 1) / Cfg::CHUNK_N;
                const int b_live = n0 >= p.N ? 0 : (b_left < Cfg::HN / Cfg::CHUNK_N ? b_left : Cfg::HN / Cfg::CHUNK_N);
                const uint32_t a_bytes = Cfg::A_MN ? a_live * Cfg::A_CHUNK : (a_live ? Cfg::A_STAGE : 0);
                const uint32_t b_bytes = Cfg::B_MN ? b_live * Cfg::B_CHUNK : (b_live ? Cfg::B_STAGE : 0);
                const uint32_t bytes = a_bytes + b_bytes;
                for (int kb = kb0; kb < kb1; ++kb, ++it) {
                    const uint32_t s = it % Cfg::STAGES;
                    const uint32_t ph = (it / Cfg::STAGES) & 1;
                    if (!bounded_wait(&empty[s], ph ^ 1, abort_flag, limit, p.status)) { ok = false; break; }
                    if (p.inject == 1 && it == 0 && pair == 0 && rank == 0) continue;   // debug: never arm slot 0
                    const uint32_t fbar = mapa_shared(smem_u32(&full[s]), 0);
                    mbar_arrive_expect_tx_cluster(fbar, bytes);
                    armed |= 1u << s;
                    armed_par = (armed_par & ~(1u << s)) | (ph << s);
                    if constexpr (Cfg::A_MN) {
                        for (int j = 0; j < a_live; ++j)      // stored K x M: boxes of 64 rows of A
                            tma_load_2d_pair(smA + s * Cfg::A_STAGE + j * Cfg::A_CHUNK, &tmA, fbar,
                                             m0 + 64 * j, kb * Cfg::BK);
                    } else if (a_live) {
                        tma_load_2d_pair(smA + s * Cfg::A_STAGE, &tmA, fbar, kb * Cfg::BK, m0);
                    }
                    if constexpr (Cfg::B_MN) {
                        for (int j = 0; j < b_live; ++j)
                            tma_load_2d_pair(smB + s * Cfg::B_STAGE + j * Cfg::B_CHUNK, &tmB, fbar,
                                             n0 + Cfg::CHUNK_N * j, kb * Cfg::BK);
                    } else if (b_live) {                      // stored N x K: one box of 128 columns
                        tma_load_2d_pair(smB + s * Cfg::B_STAGE, &tmB, fbar, kb * Cfg::BK, n0);
                    }
                }
            }
            if (!ok) {
                if (rank == 0) {
                    for (int s = 0; s < Cfg::STAGES; ++s)
                        if (armed & (1u << s)) {
                            volatile int never = 0;
                            bounded_wait(&full[s], (armed_par >> s) & 1, &never, limit, p.status);
                        }
                } else {
                    // this CTA's copies complete on the leader's barriers, which it
                    // cannot wait on: give copies in flight a fixed 1 ms to land
                    const uint64_t t0 = globaltimer_ns();
                    while (globaltimer_ns() - t0 < 1000000ull) __nanosleep(10000);
                }
            }
        }
        __syncwarp();
    } else if (warp == 1) {
        // ------------------------------------------ MMA issuer (leader only)
        if (rank == 0 && elect_one()) {
            constexpr uint32_t idesc = make_idesc(Cfg::FMT, Cfg::PM, Cfg::BN, Cfg::A_MN, Cfg::B_MN);
            uint32_t it = 0, tl = 0;
            bool ok = true;
            for (int w = pair; w < num_items && ok; w += npairs, ++tl) {
                int t, kb0, kb1, z;
                tail_item(w, dp, S, num_kb, t, kb0, kb1, z);
                const uint32_t acc = tl & 1;
                const uint32_t aph = (tl >> 1) & 1;
                if (!bounded_wait(&tempty[acc], aph ^ 1, abort_flag, limit, p.status)) { ok = false; break; }
                tc_fence_after();
                const uint32_t d_tmem = tmem_base + acc * Cfg::BN;
                for (int kb = kb0; kb < kb1; ++kb, ++it) {
                    const uint32_t s = it % Cfg::STAGES;
                    const uint32_t ph = (it / Cfg::STAGES) & 1;
                    if (!bounded_wait(&full[s], ph, abort_flag, limit, p.status)) { ok = false; break; }
                    tc_fence_after();
                    const uint32_t a_addr = smem_u32(smA + s * Cfg::A_STAGE);
                    const uint32_t b_addr = smem_u32(smB + s * Cfg::B_STAGE);
#pragma unroll
                    for (int k = 0; k < Cfg::BK / Cfg::MMA_K; ++k) {
                        // K-major: MMA_K k = 32 bytes along a 128-byte row; MN-major:
                        // MMA_K rows of 128 bytes, chunks LBO apart
                        const uint64_t ad = Cfg::A_MN
                            ? sw128_desc(a_addr + k * Cfg::MMA_K * 128, Cfg::A_CHUNK, 1024)
                            : sw128_desc(a_addr + k * 32, 16, 1024);
                        const uint64_t bd = Cfg::B_MN
                            ? sw128_desc(b_addr + k * Cfg::MMA_K * 128, Cfg::B_CHUNK, Cfg::B_SBO, Cfg::B_LAYOUT)
                            : sw128_desc(b_addr + k * 32, 16, 1024);
                        if constexpr (Cfg::FMT == 2)
                            mma_tf32_pair(d_tmem, ad, bd, idesc, (kb != kb0) || k != 0);
                        else
                            mma_f16_pair(d_tmem, ad, bd, idesc, (kb != kb0) || k != 0);
                    }
                    const uint32_t e_loc = smem_u32(&empty[s]);
                    mma_commit_pair(mapa_shared(e_loc, 0));      // both CTAs' slots
                    mma_commit_pair(mapa_shared(e_loc, 1));
                }
                if (!ok) break;
                const uint32_t f_loc = smem_u32(&tfull[acc]);
                mma_commit_pair(mapa_shared(f_loc, 0));          // both CTAs' accumulators
                mma_commit_pair(mapa_shared(f_loc, 1));
            }
            mma_commit_pair(mapa_shared(smem_u32(drain), 0));
            volatile int never = 0;
            bounded_wait(drain, 0, &never, limit, p.status);
        }
        __syncwarp();
    } else {
        // --------------------------------------------------- epilogue (both)
        const int q = warp & 3;
        uint8_t* stg0 = smStg + (warp - 2) * 2 * Cfg::STG_BUF;
        uint32_t tl = 0, nstore = 0, nflag = 0, nepi = 0, nx = 0;
        for (int w = pair; w < num_items; w += npairs, ++tl) {
            int t, kb0, kb1, z;
            tail_item(w, dp, S, num_kb, t, kb0, kb1, z);
            int tm, tn;
            tile_coords(t, ntm, ntn, p.group_m, tm, tn);
            const uint32_t acc = tl & 1;
            const uint32_t aph = (tl >> 1) & 1;
            if (!bounded_wait(&tfull[acc], aph, abort_flag, limit, p.status)) break;
            tc_fence_after();
            const int row0 = tm * Cfg::PM + rank * Cfg::BM + q * 32;
            const uint32_t tmem_acc = tmem_base + acc * Cfg::BN + (static_cast<uint32_t>(q * 32) << 16);
            bool store_tile = true;
            if (z >= 0) {
                // A half of a split tail tile.  One thread checks in and, as
                // the second, waits for the partner's partial; each result
                // reaches the other warps through flag_bar (one arrival per
                // phase).  The first writes its partial, and the four warps
                // meet on epi_bar before it is published.
                int* ck = p.tickets + ((t - dp) * 2 + rank) * 2;     // [checked in, published]
                // the CTA's 128 x 256 partial as [column / 4][row][4], the
                // same in the workspace and in the ring: the 32 rows of a
                // warp (one per lane) make each 16-byte access of the warp
                // one contiguous 512-byte run of the ring
                float* part = p.ws + static_cast<long long>((t - dp) * 2 + rank) * Cfg::BM * Cfg::BN;
                float4* ring4 = reinterpret_cast<float4*>(smA) + q * 32 + lane;
                if (warp == 2 && lane == 0) {
                    *tail_flag = atomicAdd(ck, 1);
                    mbar_arrive(flag_bar);
                }
                if (!bounded_wait(flag_bar, nflag & 1, abort_flag, limit, p.status)) break;
                ++nflag;
                const bool second = *tail_flag != 0;
                if (!second) {
                    fence_proxy_async_smem();          // copy engine and tensor core are done with the ring
                    if (row0 < p.M) {
#pragma unroll 1
                        for (int c = 0; c < Cfg::BN; c += 32) {
                            uint32_t v[32];
                            tmem_ld_32x32b_x32(tmem_acc + c, v);
                            tmem_ld_wait();
#pragma unroll
                            for (int j = 0; j < 8; ++j)
                                ring4[(c / 4 + j) * Cfg::BM] =
                                    make_float4(__uint_as_float(v[4 * j]), __uint_as_float(v[4 * j + 1]),
                                                __uint_as_float(v[4 * j + 2]), __uint_as_float(v[4 * j + 3]));
                        }
                    }
                    fence_proxy_async_smem();          // the ring's new contents, for the bulk store
                    __syncwarp();
                    if (lane == 0) mbar_arrive(epi_bar);
                    if (!bounded_wait(epi_bar, nepi & 1, abort_flag, limit, p.status)) break;
                    ++nepi;
                    if (warp == 2 && lane == 0) {
                        bulk_store_1d(part, smA, Cfg::PART_BYTES);
                        bulk_commit();
                        bulk_wait<0>();                 // written to global memory
                        fence_proxy_async_global();
                        __threadfence();
                        atomicExch(ck + 1, 1);          // published
                    }
                    store_tile = false;
                } else {
                    // the partner checked in first: wait until it has published
                    if (warp == 2 && lane == 0) {
                        const uint64_t t0 = globaltimer_ns();
                        int ok = 1;
                        while (ld_acquire_gpu(ck + 1) == 0) {
                            if (*abort_flag || globaltimer_ns() - t0 > limit) {
                                *abort_flag = 1;
                                atomicExch(p.status, ST_TIMEOUT);
                                ok = 0;
                                break;
                            }
                            __nanosleep(64);
                        }
                        if (ok) {
                            atomicExch(ck, 0);                 // both words clean for the next call
                            atomicExch(ck + 1, 0);
                            fence_proxy_async_global();        // the partial, for the bulk load
                            mbar_arrive_expect_tx(xbar, Cfg::PART_BYTES);
                            bulk_load_1d(smA, part, Cfg::PART_BYTES, xbar);
                        }
                        tail_flag[1] = ok;
                        mbar_arrive(flag_bar);
                    }
                    if (!bounded_wait(flag_bar, nflag & 1, abort_flag, limit, p.status)) break;
                    ++nflag;
                    if (!tail_flag[1]) break;
                    if (!bounded_wait(xbar, nx & 1, abort_flag, limit, p.status)) break;
                    ++nx;
                    if (row0 < p.M) {
                        // TMEM += partial, 32 columns at a time from the ring
#pragma unroll 1
                        for (int h = 0; h < Cfg::BN; h += 128) {
#pragma unroll
                            for (int c = 0; c < 4; ++c) {
                                uint32_t v[32];
                                tmem_ld_32x32b_x32(tmem_acc + h + 32 * c, v);
                                tmem_ld_wait();
#pragma unroll
                                for (int j = 0; j < 8; ++j) {
                                    const float4 a = ring4[(h / 4 + 8 * c + j) * Cfg::BM];
                                    v[4 * j] = __float_as_uint(__uint_as_float(v[4 * j]) + a.x);
                                    v[4 * j + 1] = __float_as_uint(__uint_as_float(v[4 * j + 1]) + a.y);
                                    v[4 * j + 2] = __float_as_uint(__uint_as_float(v[4 * j + 2]) + a.z);
                                    v[4 * j + 3] = __float_as_uint(__uint_as_float(v[4 * j + 3]) + a.w);
                                }
                                tmem_st_32x32b_x32(tmem_acc + h + 32 * c, v);
                            }
                        }
                        tmem_st_wait();
                    }
                }
            }
            if (store_tile) {
                if constexpr (Cfg::TOUT)
                    epilogue_tile_t<Cfg::OUT, Cfg::BN, 2>(&tmC, p, tmem_base + acc * Cfg::BN, q, lane,
                                                          row0, tn * Cfg::BN, stg0, nstore);
                else
                    epilogue_tile<Cfg::OUT, Cfg::BN, false, 2>(&tmC, p, tmem_base + acc * Cfg::BN, q, lane,
                                                               row0, tn * Cfg::BN, stg0, nstore);
            }
            tc_fence_before();
            __syncwarp();
            if (lane == 0) mbar_arrive_cluster(mapa_shared(smem_u32(&tempty[acc]), 0));
        }
        if (lane == 0) bulk_wait<0>();
        __syncwarp();
    }

    tc_fence_before();
    __syncthreads();
    cluster_sync_all();          // the pair is done with each other's barriers and TMEM
    if (warp == 1) {
        tc_fence_after();
        tmem_dealloc_pair(tmem_base, Cfg::TMEM_COLS);
    }
}

}  // namespace tg
