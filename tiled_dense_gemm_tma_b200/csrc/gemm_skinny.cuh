// gemm_skinny.cuh -- weight-streaming GEMM for few activation rows (small M).
//
// When M is small the GEMM is bound by streaming the K x N weight matrix from
// HBM (the skinny shapes and the small-batch dequantize GEMM).  The tile
// scheme of the tensor-core kernel would leave most SMs idle (N/256 tiles)
// and waste the 128-row MMA on padding rows, so this kernel swaps the
// operands and splits the work finely:
//
//   D[n][m] = sum_k W[k][n] * X[m][k]        (C = D^T, X = A)
//
// * The weight tile (128 columns n x BK rows k) is the MMA's 128-row operand,
//   N-major in shared memory (K-major when B is stored transposed, N x K, as
//   in the backward product dA = dC . B^T); the activations (MPAD >= M rows, zero-padded
//   by the copy engine) are the MMA's N operand, K-major.  D lives in TMEM as
//   128 lanes (n) x MPAD columns (m).
// * Stream-K: the (column group, k-unit) units of all T = ceil(N/GN) column
//   groups (GN = 128 columns, 256 for 4-bit weights; a unit is BK = 128
//   rows of 16-bit or 64 rows of 4-bit weights) are cut into G (one per SM)
//   contiguous, equal ranges.  A CTA accumulates each maximal run of its
//   range inside one group (a segment).  A segment that covers a whole group
//   is written to C directly; otherwise its fp32 partial goes to a workspace
//   slot (row-major: row m of GN values) and the CTA that completes the
//   group's last segment (counted with an atomic ticket) sums the partials
//   in segment order -- deterministic -- applies ReLU, rounds and writes C,
//   and resets the ticket for the next call.
// * Split-K inside clusters (where T groups times a split S in {8, 4, 2, 1}
//   fill at least three quarters of the SMs): group t goes to
//   the S CTAs of cluster t, each taking a contiguous part of its k-units.
//   When its accumulator is final a CTA's ring is idle; the ranks exchange
//   "ring free" signals, store their partials of each rank's GN/S columns
//   into that rank's ring through distributed shared memory (st.async: the
//   owner's mbarrier counts the bytes, so no sender waits on a fence), and
//   each rank sums its columns' S partials in rank order (deterministic) and
//   writes C.
//   No global round trips (partials, fences, tickets) sit between the last
//   MMA and the output, which is where stream-K spends its tail.
// * Weights arrive either as fp16/bf16 tiles by TMA, or as packed 4-bit
//   weights + scales that converter warps expand (dequant.cuh): signed
//   integers with fp16 group scales into fp16 tiles, or FP4 (E2M1) codes
//   with E8M0 block scales into bf16 tiles.
#pragma once
#include "ptx.cuh"
#include "dequant.cuh"
#include "tile_sched.h"     // sk_begin / sk_owner / cl_begin / cl_split
#include "host.cuh"         // max_active_clusters
#include <cuda_bf16.h>
#include <cuda_fp16.h>

namespace tg {

// Weight kinds: 16-bit weights, signed 4-bit integers with fp16 group scales
// (fp16 activations and output), FP4 E2M1 codes with E8M0 block scales
// (bf16 activations and output).
enum class WKind { F16 = 0, BF16 = 1, INT4 = 2, FP4 = 3 };

// WK_ = 1: 16-bit weights stored transposed (B is N x K row-major, the
// op(B) = B^T of a transposed-operand call): each weight tile arrives as
// BK/64 boxes of 128 stored rows (the tile's n) x 64 k and the MMA reads it
// K-major.  WK_ = 0: B is K x N row-major, tiles arrive N-major.
template <WKind W_, int MPAD_, int WK_ = 0>
struct SkCfg {
    static constexpr WKind W = W_;
    static constexpr int MPAD = MPAD_;                  // MMA N: 16, 32, 64 or 128
    static constexpr int WK = WK_;
    static constexpr int TN = 128;                      // weight columns per MMA (MMA M)
    static constexpr bool Q4 = W_ == WKind::INT4 || W_ == WKind::FP4;   // packed 4-bit weights
    static constexpr bool FP4 = W_ == WKind::FP4;
    // activation, MMA operand and output type
    static constexpr WKind OUTW = (W_ == WKind::BF16 || W_ == WKind::FP4) ? WKind::BF16 : WKind::F16;
    // k rows per unit: 16-bit weights come in 128-row boxes (taller TMA
    // copies stream faster), 4-bit weights in 64-row slices
    static constexpr int BK = Q4 ? 64 : 128;
    static constexpr int KSL = BK / 64;                 // 64-wide activation k-slices per unit
    // 4-bit units span two 128-column sub-tiles so packed rows arrive as
    // 128-byte runs (narrower rows stream markedly slower from HBM)
    static constexpr int NSUB = Q4 ? 2 : 1;
    static constexpr int GN = NSUB * TN;                // weight columns per unit
    static constexpr int W_CHUNK = BK * 128;            // 64 columns x BK rows, bytes
    static constexpr int W_BYTES = NSUB * 2 * W_CHUNK;  // fp16 weight tile of one unit
    static constexpr int X_SLICE = MPAD * 128;          // MPAD rows x 64 fp16
    static constexpr int X_BYTES = KSL * X_SLICE;
    static constexpr int Q_BYTES = Q4 ? BK * GN / 2 : 0;   // 8 KB packed
    // 512 B of scales per unit: one row of GN fp16 group scales (a 128-row
    // group) or two rows of GN E8M0 bytes (two 32-row blocks)
    static constexpr int S_BYTES = Q4 ? GN * 2 : 0;
    // Ring of TMA-filled slots.  16-bit weights: [W | X], released by the MMA.
    // 4-bit weights: [Q | S], released by the converters as soon as they have
    // expanded it into a second ring of fp16 tiles; the activations then
    // travel in a ring of their own, released by the MMA.
    static constexpr int RAW_SLOT_USED = Q4 ? (Q_BYTES + S_BYTES) : (X_BYTES + W_BYTES);
    static constexpr int RAW_SLOT = (RAW_SLOT_USED + 1023) / 1024 * 1024;   // swizzle alignment
    // the fp16 tiles only bridge converters and MMA (on-chip latency): two
    // suffice, which leaves the shared memory to packed weights in flight
    static constexpr int W_STAGES = Q4 ? 2 : 0;
    static constexpr int X_STAGES = !Q4 ? 0 : (X_BYTES * 8 <= 32 * 1024 ? 8 : (32 * 1024) / X_BYTES);
    static constexpr int BUDGET = 212 * 1024 - W_STAGES * W_BYTES - X_STAGES * X_BYTES;
    static constexpr int RAW_STAGES_FIT = BUDGET / RAW_SLOT;
    static constexpr int RAW_STAGES = RAW_STAGES_FIT > 16 ? 16 : RAW_STAGES_FIT;
    static constexpr int EPI_WARPS = 4;
    static constexpr int CONV_WARPS = Q4 ? 8 : 0;
    // rows per warp the reducer sums per round (registers allow more with the
    // 6-warp 16-bit kernel than beside the 4-bit converters)
    static constexpr int RED_ROWS = Q4 ? 2 : 8;
    static constexpr int THREADS = 32 * (2 + EPI_WARPS + CONV_WARPS);
    // Split-K inside a cluster: a CTA's ring, idle once its accumulator is
    // final, receives the partials of the columns it owns from every rank
    // ([rank][MPAD rows][GN/S columns] fp32, MPAD x GN floats in all).
    static constexpr int RING_BYTES = RAW_STAGES * RAW_SLOT;
    static constexpr bool CL_OK = MPAD * GN * 4 <= RING_BYTES;
    // Independent accumulator sets: k-step kk of a unit accumulates into set
    // kk % R, so consecutive small MMAs do not wait on each other's result;
    // the epilogue adds the R sets in a fixed order.
    static constexpr int R = (2 * NSUB * MPAD * 4 <= 512) ? 4 : (2 * NSUB * MPAD * 2 <= 512) ? 2 : 1;
    static constexpr int ACC_COLS = R * NSUB * MPAD;          // one accumulator buffer
    static constexpr int TMEM_USED = 2 * ACC_COLS;
    static constexpr int TMEM_COLS = TMEM_USED <= 32 ? 32 : TMEM_USED <= 64 ? 64 :
                                     TMEM_USED <= 128 ? 128 : TMEM_USED <= 256 ? 256 : 512;
    static_assert(TMEM_USED <= 512, "TMEM");
    static constexpr int SMEM_BYTES = RAW_STAGES * RAW_SLOT + W_STAGES * W_BYTES +
                                      X_STAGES * X_BYTES + 768 + 1024;
    static_assert(MPAD % 16 == 0 && MPAD <= 128, "MPAD");
    // Layout guards: slots and tiles that hold 128-byte-swizzled boxes start
    // on 1024-byte boundaries; the ring keeps at least 3 slots in flight; one
    // CTA fits the 227 KB limit; a 4-bit packed row of a unit is one 128-byte
    // swizzle span.
    static_assert(RAW_SLOT % 1024 == 0 && W_BYTES % 1024 == 0 && X_SLICE % 1024 == 0 &&
                  W_CHUNK % 1024 == 0, "swizzle alignment");
    static_assert(RAW_STAGES >= 3, "ring");
    static_assert(SMEM_BYTES <= 227 * 1024, "shared memory per CTA");
    static_assert(!Q4 || GN / 2 == 128, "packed row");
    static_assert(!WK || (!Q4 && W_CHUNK == 64 * 2 * BK && TN * 128 == 16384),
                  "K-major weights: 16-bit only; BK/64 boxes of 128 rows x 128 B fill W_BYTES");
};

struct SkParams {
    int M, N, K;
    int relu;
    int T, KB, U;             // column groups (GN wide), k-slices per group, units = T * KB
    int J;                    // workspace slots per tile (max segments of a tile)
    int S;                    // 0: stream-K (ws, tickets); S >= 1: column group blockIdx.x / S
                              // split over the S CTAs of one cluster (1: whole groups)
    int inject;               // debug: 1 = CTA 0's producer skips arming the first slot
    unsigned long long timeout_ns;
    int* status;
    void* C;
    long long ldc;
    float* ws;                // [T][J] slots of MPAD*GN fp32: row-major partials (row m: GN values)
    int* tickets;             // [T], zero between calls
};

template <WKind W>
__device__ __forceinline__ void store_out(void* C, long long ldc, int m, int n, float v) {
    if constexpr (W == WKind::BF16) {
        reinterpret_cast<__nv_bfloat16*>(C)[static_cast<long long>(m) * ldc + n] = __float2bfloat16_rn(v);
    } else {
        reinterpret_cast<__half*>(C)[static_cast<long long>(m) * ldc + n] = __float2half_rn(v);
    }
}

// Four neighbouring outputs C[m][n .. n + 3] (n a multiple of 4): one 8-byte
// store when all four are inside N (row pitches are multiples of 16 bytes).
template <WKind W>
__device__ __forceinline__ void store_out4(void* C, long long ldc, int m, int n, int N, const float (&o)[4]) {
    if (n + 3 < N) {
        uint2 pk;
        if constexpr (W == WKind::BF16) {
            __nv_bfloat162 a = __floats2bfloat162_rn(o[0], o[1]), b = __floats2bfloat162_rn(o[2], o[3]);
            pk.x = *reinterpret_cast<uint32_t*>(&a);
            pk.y = *reinterpret_cast<uint32_t*>(&b);
        } else {
            __half2 a = __floats2half2_rn(o[0], o[1]), b = __floats2half2_rn(o[2], o[3]);
            pk.x = *reinterpret_cast<uint32_t*>(&a);
            pk.y = *reinterpret_cast<uint32_t*>(&b);
        }
        *reinterpret_cast<uint2*>(reinterpret_cast<uint16_t*>(C) + static_cast<long long>(m) * ldc + n) = pk;
    } else {
#pragma unroll
        for (int e = 0; e < 4; ++e)
            if (n + e < N) store_out<W>(C, ldc, m, n + e, o[e]);
    }
}

// tmW: fp16/bf16 weights (N x K view: 64-column boxes of BK rows), or the
//      packed 4-bit weights (64-byte boxes of BK rows) for INT4;
// tmS: scales (INT4 only); tmX: activations, K-major boxes of 64 x MPAD.
template <class Cfg>
__global__ void __launch_bounds__(Cfg::THREADS, 1)
skinny_kernel(const __grid_constant__ CUtensorMap tmW,
              const __grid_constant__ CUtensorMap tmS,
              const __grid_constant__ CUtensorMap tmX,
              const SkParams p) {
    extern __shared__ uint8_t smem_raw[];
    const uint32_t raw_addr = smem_u32(smem_raw);
    uint8_t* smem = smem_raw + (((raw_addr + 1023u) & ~1023u) - raw_addr);
    uint8_t* ring = smem;                                            // RAW_STAGES x RAW_SLOT
    uint8_t* wring = ring + Cfg::RAW_STAGES * Cfg::RAW_SLOT;         // W_STAGES x W_BYTES
    uint8_t* xring = wring + Cfg::W_STAGES * Cfg::W_BYTES;           // X_STAGES x X_BYTES
    uint64_t* bars = reinterpret_cast<uint64_t*>(xring + Cfg::X_STAGES * Cfg::X_BYTES);
    uint64_t* full = bars;                                           // [RAW_STAGES]
    uint64_t* rempty = full + Cfg::RAW_STAGES;                       // [RAW_STAGES]
    uint64_t* wfull = rempty + Cfg::RAW_STAGES;                      // [W_STAGES]
    uint64_t* wempty = wfull + Cfg::W_STAGES;                        // [W_STAGES]
    uint64_t* xfull = wempty + Cfg::W_STAGES;                        // [X_STAGES]
    uint64_t* xempty = xfull + Cfg::X_STAGES;                        // [X_STAGES]
    uint64_t* tfull = xempty + Cfg::X_STAGES;                        // [2]
    uint64_t* tempty = tfull + 2;                                    // [2]
    uint64_t* drain = tempty + 2;
    uint64_t* epi_bar = drain + 1;                                   // epilogue warps joined
    uint64_t* flag_bar = epi_bar + 1;                                // ticket result published
    uint64_t* cl_ready = flag_bar + 1;                               // peers' rings may receive
    uint64_t* cl_full = cl_ready + 1;                                // this CTA's columns arrived
    uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(cl_full + 1);
    volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_slot + 1);
    volatile int* last_flag = abort_flag + 1;

    // slot layout: 16-bit weights [W | X]; 4-bit weights [Q | S] (X in xring)
    auto slot_x = [&](int s) { return ring + s * Cfg::RAW_SLOT + Cfg::W_BYTES; };
    auto slot_w = [&](int s) { return ring + s * Cfg::RAW_SLOT; };
    auto slot_q = [&](int s) { return ring + s * Cfg::RAW_SLOT; };
    auto slot_s = [&](int s) { return ring + s * Cfg::RAW_SLOT + Cfg::Q_BYTES; };

    const int warp = threadIdx.x >> 5;
    const int lane = threadIdx.x & 31;
    const int G = gridDim.x;
    const int c = blockIdx.x;
    const int KB = p.KB;
    int u0, u1, crank = 0;                   // crank: rank in the cluster
    if (p.S) {
        const int tg0 = c / p.S;
        crank = c - tg0 * p.S;
        u0 = tg0 * KB + cl_begin(crank, KB, p.S);
        u1 = tg0 * KB + cl_begin(crank + 1, KB, p.S);
    } else {
        u0 = sk_begin(c, p.U, G);
        u1 = sk_begin(c + 1, p.U, G);
    }
    const uint64_t limit = p.timeout_ns;
    bool cl_waited = false;                  // this thread passed the start-up cluster barrier
    bool cl_done = false;                    // this thread arrived on the closing cluster barrier

    if (threadIdx.x == 0) {
        for (int s = 0; s < Cfg::RAW_STAGES; ++s) {
            mbar_init(&full[s], 1);
            mbar_init(&rempty[s], Cfg::Q4 ? Cfg::CONV_WARPS : 1);
        }
        for (int s = 0; s < Cfg::W_STAGES; ++s) {
            mbar_init(&wfull[s], Cfg::CONV_WARPS);
            mbar_init(&wempty[s], 1);
        }
        for (int s = 0; s < Cfg::X_STAGES; ++s) {
            mbar_init(&xfull[s], 1);
            mbar_init(&xempty[s], 1);
        }
        for (int a = 0; a < 2; ++a) { mbar_init(&tfull[a], 1); mbar_init(&tempty[a], Cfg::EPI_WARPS); }
        mbar_init(drain, 1);
        mbar_init(epi_bar, Cfg::EPI_WARPS);
        mbar_init(flag_bar, 1);
        mbar_init(cl_ready, p.S > 1 ? p.S - 1 : 1);
        mbar_init(cl_full, 1);
        // every rank's partial of this CTA's GN/S columns, rows m < M, fp32
        if (p.S > 1) mbar_arrive_expect_tx(cl_full, static_cast<uint32_t>(p.M) * Cfg::GN * 4);
        *abort_flag = 0;
        *last_flag = 0;
        fence_mbar_init();
        fence_proxy_async_smem();
    }
    if (warp == 1) {
        tmem_alloc(tmem_slot, Cfg::TMEM_COLS);
        tmem_relinquish();
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem_base = *tmem_slot;
    // Peers arrive on this CTA's barriers only after a cluster barrier whose
    // arrive is here (after the barriers are initialised); each thread waits
    // on it before its first remote arrive, or at the end.
    if (p.S > 1) cluster_arrive_release();

    if (warp == 0) {
        // ------------------------------------------------------ TMA producer
        if (elect_one()) {
            tma_prefetch_desc(&tmW);
            tma_prefetch_desc(&tmX);
            if constexpr (Cfg::Q4) tma_prefetch_desc(&tmS);
            uint32_t armed = 0, armed_par = 0, xarmed = 0, xarmed_par = 0;
            bool ok = true;
            int it = 0;
            for (int u = u0; u < u1; ++u, ++it) {
                const int t = u / KB, kb = u - (u / KB) * KB;
                const int s = it % Cfg::RAW_STAGES;
                const uint32_t ph = (it / Cfg::RAW_STAGES) & 1;
                if (!bounded_wait(&rempty[s], ph ^ 1, abort_flag, limit, p.status)) { ok = false; break; }
                if constexpr (Cfg::Q4) {
                    const int xs = it % Cfg::X_STAGES;
                    const uint32_t xph = (it / Cfg::X_STAGES) & 1;
                    if (!bounded_wait(&xempty[xs], xph ^ 1, abort_flag, limit, p.status)) { ok = false; break; }
                    if (p.inject == 1 && it == 0 && c == 0) continue;   // debug: never arm slot 0
                    mbar_arrive_expect_tx(&full[s], Cfg::Q_BYTES + Cfg::S_BYTES);
                    tma_load_2d(slot_q(s), &tmW, &full[s], t * (Cfg::GN / 2), kb * Cfg::BK);
                    tma_load_2d(slot_s(s), &tmS, &full[s], t * Cfg::GN,
                                (kb * Cfg::BK) / (Cfg::FP4 ? 32 : 128));
                    mbar_arrive_expect_tx(&xfull[xs], Cfg::X_BYTES);
                    tma_load_2d(xring + xs * Cfg::X_BYTES, &tmX, &xfull[xs], kb * Cfg::BK, 0);
                    xarmed |= 1u << xs;
                    xarmed_par = (xarmed_par & ~(1u << xs)) | (xph << xs);
                } else if constexpr (Cfg::WK) {
                    if (p.inject == 1 && it == 0 && c == 0) continue;   // debug: never arm slot 0
                    // B stored N x K: BK/64 boxes of the tile's 128 n rows x 64 k
                    // (rows past N read the copy engine's zero fill)
                    mbar_arrive_expect_tx(&full[s], Cfg::X_BYTES + Cfg::W_BYTES);
#pragma unroll
                    for (int ks = 0; ks < Cfg::KSL; ++ks) {
                        tma_load_2d(slot_w(s) + ks * (Cfg::TN * 128), &tmW, &full[s],
                                    kb * Cfg::BK + 64 * ks, t * Cfg::TN);
                        tma_load_2d(slot_x(s) + ks * Cfg::X_SLICE, &tmX, &full[s], kb * Cfg::BK + 64 * ks, 0);
                    }
                } else {
                    if (p.inject == 1 && it == 0 && c == 0) continue;   // debug: never arm slot 0
                    // the second 64-column box is skipped when it starts past N
                    const bool second = t * Cfg::TN + 64 < p.N;
                    mbar_arrive_expect_tx(&full[s], Cfg::X_BYTES + (second ? 2 : 1) * Cfg::W_CHUNK);
                    tma_load_2d(slot_w(s), &tmW, &full[s], t * Cfg::TN, kb * Cfg::BK);
                    if (second)
                        tma_load_2d(slot_w(s) + Cfg::W_CHUNK, &tmW, &full[s], t * Cfg::TN + 64,
                                    kb * Cfg::BK);
#pragma unroll
                    for (int ks = 0; ks < Cfg::KSL; ++ks)
                        tma_load_2d(slot_x(s) + ks * Cfg::X_SLICE, &tmX, &full[s], kb * Cfg::BK + 64 * ks, 0);
                }
                armed |= 1u << s;
                armed_par = (armed_par & ~(1u << s)) | (ph << s);
            }
            if (!ok) {
                for (int s = 0; s < Cfg::RAW_STAGES; ++s)
                    if (armed & (1u << s)) {
                        volatile int never = 0;
                        bounded_wait(&full[s], (armed_par >> s) & 1, &never, limit, p.status);
                    }
                for (int s = 0; s < Cfg::X_STAGES; ++s)
                    if (xarmed & (1u << s)) {
                        volatile int never = 0;
                        bounded_wait(&xfull[s], (xarmed_par >> s) & 1, &never, limit, p.status);
                    }
            }
        }
        __syncwarp();
    } else if (warp == 1) {
        // ------------------------------------------------------- MMA issuer
        if (elect_one()) {
            constexpr uint32_t fmt = Cfg::OUTW == WKind::BF16 ? 1u : 0u;
            constexpr uint32_t idesc = make_idesc(fmt, Cfg::TN, Cfg::MPAD, Cfg::WK ? 0 : 1, 0);
            bool ok = true;
            int it = 0, seg = 0;
            uint32_t d_tmem = tmem_base;
            for (int u = u0; u < u1 && ok; ++u, ++it) {
                const int kb = u - (u / KB) * KB;
                const bool first = (u == u0) || kb == 0;
                const bool last = (u == u1 - 1) || kb == KB - 1;
                if (first) {
                    const uint32_t acc = seg & 1;
                    if (!bounded_wait(&tempty[acc], ((seg >> 1) & 1) ^ 1, abort_flag, limit, p.status)) {
                        ok = false;
                        break;
                    }
                    tc_fence_after();
                    d_tmem = tmem_base + acc * Cfg::ACC_COLS;
                }
                const int s = it % Cfg::RAW_STAGES;
                const uint32_t ph = (it / Cfg::RAW_STAGES) & 1;
                uint32_t w_addr, x_addr;
                int w = 0, xs = 0;
                if constexpr (Cfg::Q4) {
                    w = it % Cfg::W_STAGES;
                    xs = it % Cfg::X_STAGES;
                    if (!bounded_wait(&xfull[xs], (it / Cfg::X_STAGES) & 1, abort_flag, limit, p.status) ||
                        !bounded_wait(&wfull[w], (it / Cfg::W_STAGES) & 1, abort_flag, limit, p.status)) {
                        ok = false;
                        break;
                    }
                    w_addr = smem_u32(wring + w * Cfg::W_BYTES);
                    x_addr = smem_u32(xring + xs * Cfg::X_BYTES);
                } else {
                    if (!bounded_wait(&full[s], ph, abort_flag, limit, p.status)) { ok = false; break; }
                    w_addr = smem_u32(slot_w(s));
                    x_addr = smem_u32(slot_x(s));
                }
                tc_fence_after();
#pragma unroll
                for (int j = 0; j < Cfg::NSUB; ++j) {
#pragma unroll
                    for (int k = 0; k < Cfg::BK / 16; ++k) {
                        // weights: N-major, 16 k rows of 128 B per MMA (or, stored
                        // transposed, K-major: 32 B of k inside the 128-byte rows of
                        // the k/4-th box); activations: K-major
                        const uint64_t ad = Cfg::WK
                            ? sw128_desc(w_addr + (k >> 2) * (Cfg::TN * 128) + (k & 3) * 32, 16, 1024)
                            : sw128_desc(w_addr + j * 2 * Cfg::W_CHUNK + k * 16 * 128, Cfg::W_CHUNK, 1024);
                        const uint64_t bd = sw128_desc(x_addr + (k >> 2) * Cfg::X_SLICE + (k & 3) * 32,
                                                       16, 1024);
                        const int set = k % Cfg::R;
                        mma_f16(d_tmem + (set * Cfg::NSUB + j) * Cfg::MPAD, ad, bd, idesc,
                                (first && k < Cfg::R) ? 0u : 1u);
                    }
                }
                if constexpr (Cfg::Q4) {
                    mma_commit(&xempty[xs]);
                    mma_commit(&wempty[w]);
                } else {
                    mma_commit(&rempty[s]);
                }
                if (last) {
                    mma_commit(&tfull[seg & 1]);
                    ++seg;
                }
            }
            mma_commit(drain);
            volatile int never = 0;
            bounded_wait(drain, 0, &never, limit, p.status);
        }
        __syncwarp();
    } else if (warp < 2 + Cfg::EPI_WARPS) {
        // --------------------------------------------------------- epilogue
        const int q = warp & 3;
        const int etid = threadIdx.x - 64;                   // 0..127
        const int lane_n = q * 32 + lane;                    // TMEM lane = tile-local n slot
        // 4-bit weights are stored 0,2,4,6,1,3,5,7 inside 8-column groups
        const int n_loc = Cfg::Q4 ? ((lane_n & ~7) | ((lane_n & 3) << 1) | ((lane_n >> 2) & 1))
                                  : lane_n;
        int seg = 0;
        uint32_t nsync = 0;
        for (int u = u0; u < u1; ++seg) {
            const int t = u / KB;
            const int seg_end = min(u1, (t + 1) * KB);
            const bool whole = (u == t * KB) && (seg_end == (t + 1) * KB);
            u = seg_end;
            const uint32_t acc = seg & 1;
            if (!bounded_wait(&tfull[acc], (seg >> 1) & 1, abort_flag, limit, p.status)) break;
            tc_fence_after();
            // Split-K in a cluster: the accumulator is final, so every unit
            // has been consumed and this CTA's ring is idle.  Once the peers'
            // barriers exist, tell the peers their partials of this CTA's
            // columns may come, and wait until every peer's ring may take
            // this CTA's partials of its columns.
            const bool cl = p.S > 1 && !whole;
            const int CW = Cfg::GN / (p.S > 1 ? p.S : 1);   // columns a rank owns
            if (cl) {
                cluster_wait_acquire();
                cl_waited = true;
                if (etid == 0) {
                    // the copy engine's and the tensor core's accesses to the
                    // ring are complete; the peers' stores come next
                    fence_proxy_async_smem();
                    for (int pr = 0; pr < p.S; ++pr)
                        if (pr != crank) mbar_arrive_relaxed_cluster(mapa_shared(smem_u32(cl_ready), pr));
                }
                if (!bounded_wait_cluster(cl_ready, 0, abort_flag, limit, p.status)) break;
            }
            const uint32_t taddr = tmem_base + (static_cast<uint32_t>(q * 32) << 16) +
                                   acc * Cfg::ACC_COLS;
            // Partials are stored m-major (row m of GN fp32 per slot): the 32
            // lanes of a warp hold 32 neighbouring columns, so each store and
            // each reducer load covers whole 128-byte lines.
            const long long sstride = static_cast<long long>(Cfg::MPAD) * Cfg::GN;
            float* slot = nullptr;
            if (!whole && !cl) {
                const int jseg = c - sk_owner(t * KB, p.U, G);
                slot = p.ws + (static_cast<long long>(t) * p.J + jseg) * sstride;
            }
#pragma unroll
            for (int j = 0; j < Cfg::NSUB; ++j) {
                const int nj = j * Cfg::TN + n_loc;              // column within the unit
                const int n = t * Cfg::GN + nj;
#pragma unroll 1
                for (int mc = 0; mc < Cfg::MPAD; mc += 16) {
                    if (mc >= p.M) break;
                    uint32_t v[16];
                    tmem_ld_32x32b_x16(taddr + j * Cfg::MPAD + mc, v);
                    uint32_t vr[Cfg::R > 1 ? Cfg::R - 1 : 1][16];
#pragma unroll
                    for (int r = 1; r < Cfg::R; ++r)
                        tmem_ld_32x32b_x16(taddr + (r * Cfg::NSUB + j) * Cfg::MPAD + mc, vr[r - 1]);
                    tmem_ld_wait();
#pragma unroll
                    for (int r = 1; r < Cfg::R; ++r)
#pragma unroll
                        for (int i = 0; i < 16; ++i)
                            v[i] = __float_as_uint(__uint_as_float(v[i]) + __uint_as_float(vr[r - 1][i]));
                    if (whole) {
#pragma unroll
                        for (int i = 0; i < 16; ++i) {
                            const int m = mc + i;
                            if (m >= p.M) break;
                            const float x = __uint_as_float(v[i]);
                            if (n < p.N) store_out<Cfg::OUTW>(p.C, p.ldc, m, n, p.relu ? fmaxf(x, 0.f) : x);
                        }
                    } else if (cl) {
                        // into the owner's ring: [this rank][row m][column - o*CW]
                        const int o = nj / CW;
                        const uint32_t dst = mapa_shared(
                            smem_u32(ring) + static_cast<uint32_t>(((crank * Cfg::MPAD + mc) * CW + nj - o * CW) * 4), o);
                        const uint32_t obar = mapa_shared(smem_u32(cl_full), o);
#pragma unroll
                        for (int i = 0; i < 16; ++i)
                            if (mc + i < p.M) st_async_b32(dst + i * CW * 4, v[i], obar);
                    } else {
                        float* col = slot + nj;
#pragma unroll
                        for (int i = 0; i < 16; ++i)
                            if (mc + i < p.M) col[(mc + i) * Cfg::GN] = __uint_as_float(v[i]);
                    }
                }
            }
            if (cl) {
                // This thread stores into no peer after this: arrive on the
                // closing cluster barrier now (relaxed: it only keeps every
                // CTA alive until all peers issued their stores; the owners
                // read their rings after their barriers counted every byte).
                cluster_arrive_relaxed();
                cl_done = true;
            }
            tc_fence_before();
            __syncwarp();
            if (lane == 0) mbar_arrive(&tempty[acc]);
            if (whole) continue;
            if (cl) {
                // Owner: every (warp, sub-tile) slice of this rank's columns
                // from every rank, summed in rank order (deterministic).
                if (!bounded_wait_cluster(cl_full, 0, abort_flag, limit, p.status)) break;
                // CW is 32, 64 or 128 columns: thread etid takes the 4
                // neighbouring columns 4 * (etid % (CW / 4)) of rows
                // etid / (CW / 4), + 512 / CW, ...
                const float4* buf = reinterpret_cast<const float4*>(ring);
                const int lg = __ffs(CW >> 2) - 1;                 // log2(CW / 4)
                const int c4 = etid & ((CW >> 2) - 1);
                const int n = t * Cfg::GN + crank * CW + 4 * c4;
                for (int m = etid >> lg; m < p.M; m += (32 * Cfg::EPI_WARPS) >> lg) {
                    float4 x = make_float4(0.f, 0.f, 0.f, 0.f);
#pragma unroll
                    for (int r = 0; r < 8; ++r)
                        if (r < p.S) {
                            const float4 v4 = buf[((r * Cfg::MPAD + m) << lg) + c4];
                            x.x += v4.x; x.y += v4.y; x.z += v4.z; x.w += v4.w;
                        }
                    float o[4] = {x.x, x.y, x.z, x.w};
                    if (p.relu)
#pragma unroll
                        for (int e = 0; e < 4; ++e) o[e] = fmaxf(o[e], 0.f);
                    store_out4<Cfg::OUTW>(p.C, p.ldc, m, n, p.N, o);
                }
                continue;
            }
            // Publish the partial, take a ticket; the tile's last contributor
            // reduces.  The epilogue warps meet on mbarriers with bounded waits
            // (never an unbounded bar.sync, which a warp that gave up would hang).
            __threadfence();
            __syncwarp();
            if (lane == 0) mbar_arrive(epi_bar);
            if (!bounded_wait(epi_bar, nsync & 1, abort_flag, limit, p.status)) break;
            if (etid == 0) {
                const int first = sk_owner(t * KB, p.U, G);
                const int nseg = sk_owner(t * KB + KB - 1, p.U, G) - first + 1;
                const int old = atomicAdd(&p.tickets[t], 1);
                const int is_last = old == nseg - 1;
                if (is_last) atomicExch(&p.tickets[t], 0);
                *last_flag = is_last ? nseg : 0;
                mbar_arrive(flag_bar);
            }
            if (!bounded_wait(flag_bar, nsync & 1, abort_flag, limit, p.status)) break;
            const int nseg = *last_flag;
            ++nsync;
            if (nseg) {
                // Sum the tile's partials in segment order (deterministic).
                // Warp q takes rows m = q, q + 4, ...; each lane 4 neighbouring
                // columns per 128-column chunk, so a load is 512 contiguous
                // bytes; RR rows x up to 4 segments are in flight per round.
                __threadfence();
                constexpr int CH = Cfg::GN / 128;             // 128-column chunks
                constexpr int RR = Cfg::RED_ROWS;
                const float* base = p.ws + static_cast<long long>(t) * p.J * sstride;
                for (int m0 = q; m0 < p.M; m0 += 4 * RR) {
                    float4 accv[RR][CH];
#pragma unroll
                    for (int r = 0; r < RR; ++r)
#pragma unroll
                        for (int h = 0; h < CH; ++h) accv[r][h] = make_float4(0.f, 0.f, 0.f, 0.f);
                    for (int jj = 0; jj < nseg; jj += 4) {
                        float4 vv[4][RR][CH];
#pragma unroll
                        for (int g = 0; g < 4; ++g)
#pragma unroll
                            for (int r = 0; r < RR; ++r)
#pragma unroll
                                for (int h = 0; h < CH; ++h) {
                                    const int m = m0 + 4 * r;
                                    vv[g][r][h] = (jj + g < nseg && m < p.M)
                                        ? __ldcg(reinterpret_cast<const float4*>(
                                              base + (jj + g) * sstride + static_cast<long long>(m) * Cfg::GN +
                                              h * 128 + 4 * lane))
                                        : make_float4(0.f, 0.f, 0.f, 0.f);
                                }
#pragma unroll
                        for (int g = 0; g < 4; ++g)
#pragma unroll
                            for (int r = 0; r < RR; ++r)
#pragma unroll
                                for (int h = 0; h < CH; ++h) {
                                    accv[r][h].x += vv[g][r][h].x;
                                    accv[r][h].y += vv[g][r][h].y;
                                    accv[r][h].z += vv[g][r][h].z;
                                    accv[r][h].w += vv[g][r][h].w;
                                }
                    }
#pragma unroll
                    for (int r = 0; r < RR; ++r) {
                        const int m = m0 + 4 * r;
                        if (m >= p.M) break;
#pragma unroll
                        for (int h = 0; h < CH; ++h) {
                            const int n = t * Cfg::GN + h * 128 + 4 * lane;
                            float o[4] = {accv[r][h].x, accv[r][h].y, accv[r][h].z, accv[r][h].w};
                            if (p.relu)
#pragma unroll
                                for (int e = 0; e < 4; ++e) o[e] = fmaxf(o[e], 0.f);
                            store_out4<Cfg::OUTW>(p.C, p.ldc, m, n, p.N, o);
                        }
                    }
                }
            }
        }
    } else {
        // ---------------------------------------------- converters (4-bit only)
        if constexpr (Cfg::Q4) {
            const int ctid = threadIdx.x - 32 * (2 + Cfg::EPI_WARPS);
            int it = 0;
            for (int u = u0; u < u1; ++u, ++it) {
                const int s = it % Cfg::RAW_STAGES;
                const uint32_t ph = (it / Cfg::RAW_STAGES) & 1;
                const int w = it % Cfg::W_STAGES;
                const uint32_t wph = (it / Cfg::W_STAGES) & 1;
                if (!bounded_wait(&full[s], ph, abort_flag, limit, p.status) ||
                    !bounded_wait(&wempty[w], wph ^ 1, abort_flag, limit, p.status))
                    break;
                if constexpr (Cfg::FP4)
                    dequant_slice_fp4<Cfg::BK, Cfg::GN, 32 * Cfg::CONV_WARPS, Cfg::W_CHUNK>(
                        slot_q(s), slot_s(s), wring + w * Cfg::W_BYTES, ctid);
                else
                    dequant_slice<Cfg::BK, Cfg::GN, 32 * Cfg::CONV_WARPS, Cfg::W_CHUNK>(
                        slot_q(s), slot_s(s), wring + w * Cfg::W_BYTES, ctid);
                fence_proxy_async_smem();
                __syncwarp();
                if (lane == 0) {
                    mbar_arrive(&wfull[w]);
                    mbar_arrive(&rempty[s]);
                }
            }
        }
    }

    tc_fence_before();
    __syncthreads();
    if (warp == 1) {
        tc_fence_after();
        tmem_dealloc(tmem_base, Cfg::TMEM_COLS);
    }
    if (p.S > 1) {
        // no CTA leaves before every peer has issued its stores
        if (!cl_waited) cluster_wait_acquire();
        if (!cl_done) cluster_arrive_relaxed();
        cluster_wait_acquire();
    }
}

// Host side, shared by the regular and the static entry points.  The
// cluster split of cl_split for T column groups of KB k-units, lowered until
// the device holds all T clusters of that size at once; 0 selects stream-K.
// 4-bit weights too: their pace is set per SM (expanding the packed
// weights), so the split's T*S CTAs leave SMs idle, but the cluster
// reduction costs less than stream-K's tail through global memory.  `slot`
// is the kernel's attribute slot (set_smem_attr done).
template <class Cfg>
inline int skinny_cluster_split(long long T, long long KB, long long cap, int num_sms, int slot) {
    if constexpr (!Cfg::CL_OK) {
        return 0;
    } else {
        const void* k = reinterpret_cast<const void*>(skinny_kernel<Cfg>);
        int max_s = 8;
        for (;;) {
            const int S = cl_split(T, KB, Cfg::GN, cap, num_sms, max_s);
            if (S <= 1) return S;
            if (max_active_clusters(k, slot, S, Cfg::THREADS, Cfg::SMEM_BYTES) >= T) return S;
            max_s = S / 2;
        }
    }
}

// Launch G CTAs; clusters of S CTAs when S > 1 (p.S == S).
template <class Cfg>
inline cudaError_t skinny_launch(long long G, int S, cudaStream_t stream, const CUtensorMap& tW,
                                 const CUtensorMap& tS, const CUtensorMap& tX, const SkParams& p) {
    if (S > 1) {
        cudaLaunchConfig_t cfg = {};
        cfg.gridDim = dim3(static_cast<unsigned>(G), 1, 1);
        cfg.blockDim = dim3(Cfg::THREADS, 1, 1);
        cfg.dynamicSmemBytes = Cfg::SMEM_BYTES;
        cfg.stream = stream;
        cudaLaunchAttribute attr[1];
        attr[0].id = cudaLaunchAttributeClusterDimension;
        attr[0].val.clusterDim.x = static_cast<unsigned>(S);
        attr[0].val.clusterDim.y = 1;
        attr[0].val.clusterDim.z = 1;
        cfg.attrs = attr;
        cfg.numAttrs = 1;
        return cudaLaunchKernelEx(&cfg, skinny_kernel<Cfg>, tW, tS, tX, p);
    }
    skinny_kernel<Cfg><<<static_cast<unsigned>(G), Cfg::THREADS, Cfg::SMEM_BYTES, stream>>>(tW, tS, tX, p);
    return cudaGetLastError();
}

}  // namespace tg
