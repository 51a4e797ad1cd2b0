// gemv.cu -- GEMM for one to four activation rows on the CUDA cores.
//
// With M <= 4 the product is a few dot products per weight column: the work
// is streaming the K x N weight matrix once from HBM.  A tensor-core MMA
// (at least 16 wide in M) would spend most of its operand traffic on padding
// rows, and the 4-bit weights would have to be written back to shared memory
// as fp16 for it.  Here the weights are multiplied where they land:
//
// * The k-split of the weight-streaming tensor-core kernel.  Where T column
//   groups (GN columns each) times a split S of 2 to 8 fill the GPU, group t
//   goes to the S CTAs of cluster t, each taking a contiguous part of its
//   units (GN columns x BK rows of weights).  Otherwise stream-K: the units
//   of all groups are cut into one contiguous, equal range per SM; a maximal
//   run of a range inside one column group is a segment.
// * Warp 0 streams each unit by TMA into a ring of shared-memory slots: the
//   weight tile (unswizzled 128-byte rows: a warp reads whole rows, which
//   touch every bank once), for 4-bit weights the unit's scale rows (fp16
//   group scales, or E8M0 block exponents for FP4), and the activations
//   (MR rows x BK values).
// * Sixteen CUDA-core warps (eight for four activation rows) read the slot:
//   warp w takes a run of consecutive rows (vector reads fetch their
//   activations), each lane its GN/32 neighbouring columns of a row.
//   16-bit weights widen exactly to fp32 and multiply into fp32
//   accumulators.  Signed 4-bit weights decode exactly, two per logic op,
//   into fp16 pairs (nib_pair); mixed-precision FMAs (fp16 inputs, fp32
//   accumulator) form per warp and lane sum_k q[k][n] a[k] over the warp's
//   rows in fp32, which the group scale s[g][n] multiplies once (the
//   dequantised weight W = q * s of the pages' dequantize GEMM, with the
//   scale factored out of the sum).  FP4 codes become exact fp16 pairs by
//   the hardware conversion, are widened to fp32 and multiplied with paired
//   fp32 FMAs; the block's 2^(E - 127) is applied once per warp and column.
// * At a segment's end the warps' sums are added in warp order through
//   shared memory.  A segment that covers its whole column group writes C.
//   In a cluster, rank o owns GN/S columns of the group: every rank stores
//   its partial of them into rank o's receive buffer (distributed shared
//   memory) and rank o adds the partials in rank order.  Under stream-K the
//   fp32 partial goes to a fixed workspace slot (row-major) and the CTA that
//   takes the group's last ticket adds the slots in segment order.  Both
//   orders are fixed (deterministic); the last adder applies ReLU, rounds
//   and writes C.
// Every wait is bounded (mbarriers, timeout -> device status 5).
#include "gemm_skinny.cuh"   // WKind, SkParams, sk_begin / sk_owner, store_out4
#include "host.cuh"
#include "launch.h"

#include <cuda_bf16.h>
#include <cuda_fp16.h>

namespace tg {

namespace {

template <WKind W_, int MR_>
struct GvCfg {
    static constexpr WKind W = W_;
    static constexpr int MR = MR_;                      // activation rows: 1, 2 or 4
    static constexpr bool I4 = W_ == WKind::INT4;      // signed 4-bit integers, fp16 group scales
    static constexpr bool F4 = W_ == WKind::FP4;       // E2M1 codes, E8M0 block scales
    static constexpr bool Q4 = I4 || F4;               // packed two per byte
    static constexpr WKind ACT = I4 ? WKind::F16 : F4 ? WKind::BF16 : W_;   // activations and C
    static constexpr int GN = Q4 ? 256 : 128;           // columns per unit
    // rows per unit: 4-bit units hold SG scale groups of 128 rows (integer
    // weights) or SB blocks of 32 rows (FP4), so that a warp's run of rows (in
    // one group or block) amortises the per-unit work over more rows
    static constexpr int BK = Q4 ? 256 : 128;
    static constexpr int SG = BK / 128;
    static constexpr int SB = BK / 32;
    static constexpr int S_ROWS = I4 ? SG : SB;        // scale rows of a unit
    static constexpr int CPL = GN / 32;                 // columns per lane
    static constexpr int W_CHUNK = BK * 128;            // one 64-column box (16-bit)
    static constexpr int W_BYTES = Q4 ? BK * GN / 2 : 2 * W_CHUNK;
    static constexpr int S_BYTES = I4 ? SG * GN * 2 : F4 ? SB * GN : 0;
    static constexpr int X_ROW = BK * 2;                // one activation row of the unit
    static constexpr int X_BYTES = MR * X_ROW;          // MR rows x BK values
    static constexpr int SLOT = (W_BYTES + S_BYTES + X_BYTES + 1023) / 1024 * 1024;
    // 16 math warps; 8 with four activation rows (their accumulators need
    // more than the 96 registers a 544-thread CTA leaves per thread)
    static constexpr int FMA_WARPS = MR_ == 4 ? 8 : 16;
    static constexpr int FMA_THREADS = 32 * FMA_WARPS;
    static constexpr int THREADS = 32 + FMA_THREADS;
    static constexpr int RED_BYTES = FMA_WARPS * MR * GN * 4;
    // split-K in a cluster: an owner receives [rank][m][GN/S columns] fp32
    static constexpr int RBUF_BYTES = MR * GN * 4;
    // warps that hold the CTA's summed partial (one float4 per thread)
    static constexpr int SUM_WARPS = MR * GN / 128;
    static constexpr int STAGES_FIT = (200 * 1024 - RED_BYTES - RBUF_BYTES) / SLOT;
    static constexpr int STAGES = STAGES_FIT > 16 ? 16 : STAGES_FIT;
    static constexpr int SMEM_BYTES = STAGES * SLOT + RED_BYTES + RBUF_BYTES + 512 + 1024;
    static_assert(SUM_WARPS >= 1 && SUM_WARPS <= FMA_WARPS && MR * GN % 128 == 0,
                  "one float4 of the summed partial per thread of the first SUM_WARPS warps");
    static_assert(STAGES >= 3, "ring");
    // The producer's transaction count is built from these sizes and the
    // launcher's boxes from GN, BK and MR: each box's bytes must be the
    // count it is charged.  4-bit: one (GN/2 bytes x BK rows) weight box and
    // one (GN x SG) fp16 scale box (FP4: (GN x SB) E8M0 bytes); 16-bit: two
    // (64 x BK) weight boxes; then one (BK x MR) 16-bit activation box (at
    // most 256 values wide).  No box is swizzled; slots start on 1024-byte
    // boundaries.
    static_assert(Q4 ? (W_BYTES == (GN / 2) * BK && GN / 2 == 128)
                     : (W_BYTES == 2 * W_CHUNK && W_CHUNK == 64 * 2 * BK), "weight box bytes");
    static_assert(!Q4 || S_BYTES == GN * S_ROWS * (I4 ? 2 : 1), "scale box bytes");
    // a warp's rows of a unit lie in one scale group (block)
    static_assert(!Q4 || (BK % 128 == 0 && (I4 ? 128 : 32) % (BK / FMA_WARPS) == 0), "rows per warp");
    static_assert(X_ROW == BK * 2 && X_BYTES == MR * X_ROW && BK <= 256 && X_ROW % 16 == 0,
                  "activation box bytes");
    static_assert(SLOT % 1024 == 0 && W_CHUNK % 1024 == 0, "boxes on 1024-byte boundaries");
    static_assert(SMEM_BYTES <= 227 * 1024, "shared memory per CTA");
};


// Exact decode of signed 4-bit weights to fp16 pairs, two weights per
// logic op and without a subtraction per weight.  With b = q + 8 in [0, 15]
// (the nibble with bit 3 flipped) placed at mantissa bit p of an fp16 1.0,
// the half is f = 1 + b / D with D = 2^(10 - p); f has at most 11
// significant bits, so f * a is exact in fp32 for an fp16 activation a, and
//     sum_k q[k] a[k] = D sum_k f[k] a[k] - (D + 8) sum_k a[k].
// One lop3 keeps the nibbles at bits p and p + 16 of x, flips their bit 3
// and sets the exponent of 1.0 in both halves: a bit set in `keep` takes x's
// bit (inverted where `set` has it set), any other bit takes `set`'s.
__device__ __forceinline__ uint32_t nib_pair(uint32_t x, uint32_t keep, uint32_t set) {
    uint32_t r;
    asm("lop3.b32 %0, %1, %2, %3, 0x6A;" : "=r"(r) : "r"(x), "r"(keep), "r"(set));
    return r;
}
constexpr uint32_t kKeepLo = 0x000F000Fu, kSetLo = 0x3C083C08u;   // nibbles at bits 0, 16: D = 1024
constexpr uint32_t kKeepHi = 0x00F000F0u, kSetHi = 0x3C803C80u;   // nibbles at bits 4, 20: D = 64

// The two halves of a packed fp16 pair, and fp32 += fp16 x fp16 (one
// rounding; the product of two fp16 values is exact in fp32).
__device__ __forceinline__ void halves(uint32_t v, unsigned short& lo, unsigned short& hi) {
    asm("mov.b32 {%0, %1}, %2;" : "=h"(lo), "=h"(hi) : "r"(v));
}
__device__ __forceinline__ void fma_f16_f32(float& d, unsigned short x, unsigned short y) {
    asm("fma.rn.f32.f16 %0, %1, %2, %0;" : "+f"(d) : "h"(x), "h"(y));
}
__device__ __forceinline__ void add_f16_f32(float& d, unsigned short x) {
    asm("add.rn.f32.f16 %0, %1, %0;" : "+f"(d) : "h"(x));
}

// Paired fp32 arithmetic (two independent IEEE operations per instruction,
// each rounded as its scalar form).
__device__ __forceinline__ uint64_t pk(float x, float y) {
    uint64_t r;
    asm("mov.b64 %0, {%1, %2};" : "=l"(r) : "f"(x), "f"(y));
    return r;
}
__device__ __forceinline__ float2 upk(uint64_t v) {
    float2 r;
    asm("mov.b64 {%0, %1}, %2;" : "=f"(r.x), "=f"(r.y) : "l"(v));
    return r;
}
__device__ __forceinline__ void fma2(uint64_t& d, uint64_t x, uint64_t y) {
    asm("fma.rn.f32x2 %0, %1, %2, %0;" : "+l"(d) : "l"(x), "l"(y));
}

// The two E2M1 codes of the low byte of x (low nibble first) as an fp32
// pair: the hardware conversion to an fp16 pair is exact (every E2M1 value
// has at most two significant bits), and so is the widening.
__device__ __forceinline__ uint64_t e2m1_pair_f32(uint32_t x) {
    uint64_t r;
    asm("{\n\t.reg .b8 c;\n\t.reg .b32 h;\n\t.reg .f16 lo, hi;\n\t.reg .f32 flo, fhi;\n\t"
        "cvt.u8.u32 c, %1;\n\t"
        "cvt.rn.f16x2.e2m1x2 h, c;\n\t"
        "mov.b32 {lo, hi}, h;\n\t"
        "cvt.f32.f16 flo, lo;\n\t"
        "cvt.f32.f16 fhi, hi;\n\t"
        "mov.b64 %0, {flo, fhi};\n\t}"
        : "=l"(r) : "r"(x));
    return r;
}

// fp32 factors 2^(E - 127) of the four E8M0 bytes of e: the byte shifted
// into the exponent field; E = 0 is the subnormal 2^-127 and E = 255 NaN,
// both formed by the fraction bit 0x00400000.
__device__ __forceinline__ void e8m0_factors(uint32_t e, float* f) {
    const uint32_t special = __vcmpeq4(e, 0u) | __vcmpeq4(e, 0xFFFFFFFFu);
#pragma unroll
    for (int b = 0; b < 4; ++b) {
        const uint32_t eb = (e >> (8 * b)) & 0xFFu;
        f[b] = __uint_as_float((eb << 23) | ((special >> (8 * b)) & 1u ? 0x00400000u : 0u));
    }
}

// Two activations (or 16-bit weights) packed in a word, widened to fp32.
template <WKind T>
__device__ __forceinline__ float2 widen2(uint32_t w) {
    if constexpr (T == WKind::BF16) return make_float2(__uint_as_float(w << 16), __uint_as_float(w & 0xFFFF0000u));
    else return __half22float2(*reinterpret_cast<const __half2*>(&w));
}

template <class Cfg>
__global__ void __launch_bounds__(Cfg::THREADS, 1)
gemv_kernel(const __grid_constant__ CUtensorMap tmW,
            const __grid_constant__ CUtensorMap tmS,
            const __grid_constant__ CUtensorMap tmX,
            const SkParams p) {
    constexpr int MR = Cfg::MR, GN = Cfg::GN, CPL = Cfg::CPL, BK = Cfg::BK;
    constexpr WKind OUT = Cfg::ACT;                          // output / activation type
    constexpr int ELEMS = MR * GN;                           // one segment's sums
    extern __shared__ uint8_t smem_raw[];
    const uint32_t raw_addr = smem_u32(smem_raw);
    uint8_t* smem = smem_raw + (((raw_addr + 1023u) & ~1023u) - raw_addr);
    uint8_t* ring = smem;                                            // STAGES x SLOT
    float* red = reinterpret_cast<float*>(ring + Cfg::STAGES * Cfg::SLOT);  // [warp][m][column]
    float* rbuf = red + Cfg::FMA_WARPS * ELEMS;                      // [rank][m][column - owner * CW]
    uint64_t* full = reinterpret_cast<uint64_t*>(rbuf + ELEMS);
    uint64_t* empty = full + Cfg::STAGES;
    uint64_t* join = empty + Cfg::STAGES;                            // the FMA warps meet
    uint64_t* flag = join + 1;                                       // ticket result published
    uint64_t* cl_full = flag + 1;                                    // every rank's partial arrived
    volatile int* abort_flag = reinterpret_cast<volatile int*>(cl_full + 1);
    volatile int* last_flag = abort_flag + 1;

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
        for (int s = 0; s < Cfg::STAGES; ++s) {
            mbar_init(&full[s], 1);
            mbar_init(&empty[s], Cfg::FMA_WARPS);
        }
        mbar_init(join, Cfg::FMA_WARPS);
        mbar_init(flag, 1);
        mbar_init(cl_full, 1);
        // every rank's partial of this CTA's columns: MR x GN/S fp32 each
        if (p.S > 1) mbar_arrive_expect_tx(cl_full, Cfg::RBUF_BYTES);
        *abort_flag = 0;
        *last_flag = 0;
        fence_mbar_init();
        fence_proxy_async_smem();
    }
    __syncthreads();
    // Peers store into this CTA's receive buffer and arrive on its barrier
    // only after a cluster barrier whose arrival follows the initialisation.
    if (p.S > 1) cluster_arrive_release();

    if (warp == 0) {
        // ------------------------------------------------------ TMA producer
        if (elect_one()) {
            tma_prefetch_desc(&tmW);
            tma_prefetch_desc(&tmX);
            if constexpr (Cfg::Q4) tma_prefetch_desc(&tmS);
            uint32_t armed = 0, armed_par = 0;
            bool ok = true;
            int it = 0, s = 0;                               // slot s of pass ph
            uint32_t ph = 0;
            int t = u0 / KB, kb = u0 - (u0 / KB) * KB;      // unit u = t * KB + kb
            for (int u = u0; u < u1; ++u, ++it, kb = kb + 1 == KB ? 0 : kb + 1, t += kb == 0,
                     s = s + 1 == Cfg::STAGES ? 0 : s + 1, ph ^= s == 0) {
                if (!bounded_wait(&empty[s], ph ^ 1, abort_flag, limit, p.status)) { ok = false; break; }
                if (p.inject == 1 && it == 0 && c == 0) continue;   // debug: never arm slot 0
                uint8_t* slot = ring + s * Cfg::SLOT;
                uint8_t* xs = slot + Cfg::W_BYTES + Cfg::S_BYTES;
                if constexpr (Cfg::Q4) {
                    mbar_arrive_expect_tx(&full[s], Cfg::W_BYTES + Cfg::S_BYTES + Cfg::X_BYTES);
                    tma_load_2d(slot, &tmW, &full[s], t * (GN / 2), kb * BK);
                    tma_load_2d(slot + Cfg::W_BYTES, &tmS, &full[s], t * GN, kb * Cfg::S_ROWS);
                } else {
                    // the second 64-column box is skipped when it starts past N
                    // (its columns are never stored)
                    const bool second = t * GN + 64 < p.N;
                    mbar_arrive_expect_tx(&full[s], (second ? 2 : 1) * Cfg::W_CHUNK + Cfg::X_BYTES);
                    tma_load_2d(slot, &tmW, &full[s], t * GN, kb * BK);
                    if (second) tma_load_2d(slot + Cfg::W_CHUNK, &tmW, &full[s], t * GN + 64, kb * BK);
                }
                // the unit's activations: MR rows of BK values (X_BYTES)
                tma_load_2d(xs, &tmX, &full[s], kb * BK, 0);
                armed |= 1u << s;
                armed_par = (armed_par & ~(1u << s)) | (ph << s);
            }
            if (!ok) {
                // let the copies in flight land before the CTA exits
                for (int s = 0; s < Cfg::STAGES; ++s)
                    if (armed & (1u << s)) {
                        volatile int never = 0;
                        bounded_wait(&full[s], (armed_par >> s) & 1, &never, limit, p.status);
                    }
            }
        }
        __syncwarp();
    } else {
        // -------------------------------------------------- CUDA-core warps
        const int fw = warp - 1;                        // 0 .. FMA_WARPS - 1
        const int ftid = threadIdx.x - 32;
        uint32_t jphase = 0, fphase = 0;
        // all FMA warps meet (bounded; false if the kernel is aborting)
        auto join_all = [&]() -> bool {
            __syncwarp();
            if (lane == 0) mbar_arrive(join);
            const bool ok = bounded_wait(join, jphase & 1, abort_flag, limit, p.status);
            ++jphase;
            return ok;
        };
        constexpr int RPW = BK / Cfg::FMA_WARPS;        // consecutive rows per warp and unit
        const int r0 = fw * RPW;
        float acc[MR][CPL];
#pragma unroll
        for (int m = 0; m < MR; ++m)
#pragma unroll
            for (int q = 0; q < CPL; ++q) acc[m][q] = 0.f;
        int s = 0;                                          // slot s of pass ph
        uint32_t ph = 0;
        int t = u0 / KB, kb = u0 - (u0 / KB) * KB;          // unit u = t * KB + kb
        for (int u = u0; u < u1; ++u, kb = kb + 1 == KB ? 0 : kb + 1, t += kb == 0,
                 s = s + 1 == Cfg::STAGES ? 0 : s + 1, ph ^= s == 0) {
            if (!bounded_wait(&full[s], ph, abort_flag, limit, p.status)) break;
            const uint8_t* slot = ring + s * Cfg::SLOT;
            const uint8_t* xs = slot + Cfg::W_BYTES + Cfg::S_BYTES + r0 * 2;
            // activations of the warp's RPW rows: one vector read per m, kept
            // packed (two values per word) and widened where used
            uint32_t avw[MR][RPW / 2];
#pragma unroll
            for (int m = 0; m < MR; ++m)
#pragma unroll
                for (int h = 0; h < RPW / 8; ++h) {
                    const uint4 v = *reinterpret_cast<const uint4*>(xs + m * Cfg::X_ROW + 16 * h);
                    avw[m][4 * h] = v.x; avw[m][4 * h + 1] = v.y; avw[m][4 * h + 2] = v.z; avw[m][4 * h + 3] = v.w;
                }
            auto act = [&](int m, int i) -> float {
                const float2 f = widen2<OUT>(avw[m][i >> 1]);
                return (i & 1) ? f.y : f.x;
            };
            if constexpr (Cfg::I4) {
                // f sums per column (nibble j of the lane's word is column j)
                float fac[MR][CPL];
                float suma[MR];
#pragma unroll
                for (int m = 0; m < MR; ++m) {
                    suma[m] = 0.f;
#pragma unroll
                    for (int q = 0; q < CPL; ++q) fac[m][q] = 0.f;
                }
#pragma unroll
                for (int i = 0; i < RPW; ++i) {
                    const int r = r0 + i;
                    // 4 bytes = columns 8 lane .. 8 lane + 7 of row r
                    const uint32_t w = *reinterpret_cast<const uint32_t*>(slot + r * 128 + lane * 4);
                    const uint32_t w8 = w >> 8;
                    // pair j holds columns (j, j + 4): D = 1024 for even j, 64 for odd j
                    const uint32_t hp[4] = {nib_pair(w, kKeepLo, kSetLo), nib_pair(w, kKeepHi, kSetHi),
                                            nib_pair(w8, kKeepLo, kSetLo), nib_pair(w8, kKeepHi, kSetHi)};
#pragma unroll
                    for (int m = 0; m < MR; ++m) {
                        unsigned short a_lo, a_hi;
                        halves(avw[m][i >> 1], a_lo, a_hi);
                        const unsigned short am = (i & 1) ? a_hi : a_lo;
                        add_f16_f32(suma[m], am);
#pragma unroll
                        for (int j = 0; j < 4; ++j) {
                            unsigned short lo, hi;
                            halves(hp[j], lo, hi);
                            fma_f16_f32(fac[m][j], lo, am);
                            fma_f16_f32(fac[m][j + 4], hi, am);
                        }
                    }
                }
                // the warp's rows share one scale group: total += s * sum_k q a
                const uint4 sv = *reinterpret_cast<const uint4*>(slot + Cfg::W_BYTES + (r0 / 128) * GN * 2 +
                                                                 lane * 16);
                const uint32_t sw[4] = {sv.x, sv.y, sv.z, sv.w};
                float sc[8];
#pragma unroll
                for (int j = 0; j < 4; ++j) {
                    const float2 f = widen2<WKind::F16>(sw[j]);
                    sc[2 * j] = f.x;
                    sc[2 * j + 1] = f.y;
                }
#pragma unroll
                for (int m = 0; m < MR; ++m) {
#pragma unroll
                    for (int j = 0; j < CPL; ++j) {
                        const float d = (j & 1) ? 64.f : 1024.f;
                        acc[m][j] = fmaf(sc[j], fmaf(d, fac[m][j], -(d + 8.f) * suma[m]), acc[m][j]);
                    }
                }
            } else if constexpr (Cfg::F4) {
                // column pairs (2j, 2j + 1) = byte j of the lane's word
                uint64_t fac[MR][CPL / 2];
#pragma unroll
                for (int m = 0; m < MR; ++m)
#pragma unroll
                    for (int q = 0; q < CPL / 2; ++q) fac[m][q] = 0ull;
#pragma unroll
                for (int i = 0; i < RPW; ++i) {
                    const int r = r0 + i;
                    // 4 bytes = columns 8 lane .. 8 lane + 7 of row r
                    const uint32_t w = *reinterpret_cast<const uint32_t*>(slot + r * 128 + lane * 4);
                    uint64_t f2[4];
#pragma unroll
                    for (int j = 0; j < 4; ++j) f2[j] = e2m1_pair_f32(w >> (8 * j));
#pragma unroll
                    for (int m = 0; m < MR; ++m) {
                        const float am = act(m, i);
                        const uint64_t a2 = pk(am, am);
#pragma unroll
                        for (int j = 0; j < 4; ++j) fma2(fac[m][j], f2[j], a2);
                    }
                }
                // the warp's rows share one 32-row block: total += 2^(E - 127) * sum_k v a
                const uint2 ev = *reinterpret_cast<const uint2*>(slot + Cfg::W_BYTES + (r0 / 32) * GN + lane * 8);
                float sc[8];
                e8m0_factors(ev.x, sc);
                e8m0_factors(ev.y, sc + 4);
#pragma unroll
                for (int m = 0; m < MR; ++m) {
#pragma unroll
                    for (int j = 0; j < CPL / 2; ++j) {
                        const float2 f = upk(fac[m][j]);
                        acc[m][2 * j] = fmaf(sc[2 * j], f.x, acc[m][2 * j]);
                        acc[m][2 * j + 1] = fmaf(sc[2 * j + 1], f.y, acc[m][2 * j + 1]);
                    }
                }
            } else {
#pragma unroll
                for (int i = 0; i < RPW; ++i) {
                    const int r = r0 + i;
                    // 8 bytes = columns 4 lane .. 4 lane + 3: box lane / 16, bytes
                    // 8 (lane % 16) .. of the box row
                    const uint2 v = *reinterpret_cast<const uint2*>(
                        slot + (lane >> 4) * Cfg::W_CHUNK + r * 128 + (lane & 15) * 8);
                    const float2 w0 = widen2<Cfg::W>(v.x), w1 = widen2<Cfg::W>(v.y);
#pragma unroll
                    for (int m = 0; m < MR; ++m) {
                        const float am = act(m, i);
                        acc[m][0] = fmaf(w0.x, am, acc[m][0]);
                        acc[m][1] = fmaf(w0.y, am, acc[m][1]);
                        acc[m][2] = fmaf(w1.x, am, acc[m][2]);
                        acc[m][3] = fmaf(w1.y, am, acc[m][3]);
                    }
                }
            }
            __syncwarp();
            if (lane == 0) mbar_arrive(&empty[s]);

            if (!(u == u1 - 1 || kb == KB - 1)) continue;
            // ------------------------------------------------ segment end
            const int sb = max(u0, t * KB);
            const bool whole = sb == t * KB && u == t * KB + KB - 1;
#pragma unroll
            for (int m = 0; m < MR; ++m)
#pragma unroll
                for (int q = 0; q < CPL; q += 4) {
                    *reinterpret_cast<float4*>(red + (fw * MR + m) * GN + lane * CPL + q) =
                        make_float4(acc[m][q], acc[m][q + 1], acc[m][q + 2], acc[m][q + 3]);
                    acc[m][q] = acc[m][q + 1] = acc[m][q + 2] = acc[m][q + 3] = 0.f;
                }
            if (!join_all()) break;
            if (p.S > 1 && !whole) {
                // Split-K in a cluster: rank o owns the CW columns
                // [o CW, (o + 1) CW) of the group.  Thread ftid sums one
                // float4 of the CTA's partial and stores it asynchronously
                // into its owner's receive buffer; the owner's barrier counts
                // the bytes.  This CTA stores into no peer after that, so it
                // arrives on the closing cluster barrier at once (relaxed: that
                // barrier only keeps every CTA alive until all peers issued
                // their stores; an owner reads its buffer only after its
                // barrier counted every byte).
                const int CW = GN / p.S;
                cluster_wait_acquire();
                cl_waited = true;
                if (fw < Cfg::SUM_WARPS) {
                    const int e = ftid * 4;
                    float4 v = *reinterpret_cast<const float4*>(red + e);
#pragma unroll
                    for (int w = 1; w < Cfg::FMA_WARPS; ++w) {
                        const float4 x = *reinterpret_cast<const float4*>(red + w * ELEMS + e);
                        v.x += x.x; v.y += x.y; v.z += x.z; v.w += x.w;
                    }
                    const int m = e / GN, col = e - (e / GN) * GN;
                    const int o = col / CW;
                    st_async_v4_f32(mapa_shared(smem_u32(rbuf) + static_cast<uint32_t>(
                                                    ((crank * MR + m) * CW + col - o * CW) * 4), o),
                                    v, mapa_shared(smem_u32(cl_full), o));
                }
                cluster_arrive_relaxed();
                cl_done = true;
                // owner: MR rows x CW columns, every rank's partial summed in
                // rank order (deterministic), one float4 per thread
                const int nq = MR * (CW >> 2);
                if (ftid < nq) {
                    if (!bounded_wait_cluster(cl_full, 0, abort_flag, limit, p.status)) break;
                    const int m = ftid / (CW >> 2), c4 = ftid - m * (CW >> 2);
                    if (m < p.M) {
                        float4 x = *reinterpret_cast<const float4*>(rbuf + m * CW + 4 * c4);
                        for (int r = 1; r < p.S; ++r) {
                            const float4 y = *reinterpret_cast<const float4*>(rbuf + (r * MR + m) * CW + 4 * c4);
                            x.x += y.x; x.y += y.y; x.z += y.z; x.w += y.w;
                        }
                        float o4[4] = {x.x, x.y, x.z, x.w};
                        if (p.relu)
#pragma unroll
                            for (int j = 0; j < 4; ++j) o4[j] = fmaxf(o4[j], 0.f);
                        store_out4<OUT>(p.C, p.ldc, m, t * GN + crank * CW + 4 * c4, p.N, o4);
                    }
                }
                continue;
            }
            const int jseg = c - sk_owner(t * KB, p.U, G);
            float* part = p.ws + (static_cast<long long>(t) * p.J + jseg) * ELEMS;
            for (int e = ftid * 4; e < ELEMS; e += Cfg::FMA_THREADS * 4) {
                float4 v = *reinterpret_cast<const float4*>(red + e);
#pragma unroll
                for (int w = 1; w < Cfg::FMA_WARPS; ++w) {
                    const float4 x = *reinterpret_cast<const float4*>(red + w * ELEMS + e);
                    v.x += x.x; v.y += x.y; v.z += x.z; v.w += x.w;
                }
                const int m = e / GN, col = e - (e / GN) * GN;
                if (whole) {
                    if (m < p.M) {
                        float o[4] = {v.x, v.y, v.z, v.w};
                        if (p.relu)
#pragma unroll
                            for (int j = 0; j < 4; ++j) o[j] = fmaxf(o[j], 0.f);
                        store_out4<OUT>(p.C, p.ldc, m, t * GN + col, p.N, o);
                    }
                } else {
                    *reinterpret_cast<float4*>(part + e) = v;
                }
            }
            __threadfence();
            if (!join_all()) break;            // partials published, red free again
            if (whole) continue;
            if (ftid == 0) {
                const int first = sk_owner(t * KB, p.U, G);
                const int nseg = sk_owner(t * KB + KB - 1, p.U, G) - first + 1;
                const int old = atomicAdd(&p.tickets[t], 1);
                const int is_last = old == nseg - 1;
                if (is_last) atomicExch(&p.tickets[t], 0);
                *last_flag = is_last ? nseg : 0;
                mbar_arrive(flag);
            }
            if (!bounded_wait(flag, fphase & 1, abort_flag, limit, p.status)) break;
            ++fphase;
            const int nseg = *last_flag;
            if (!nseg) continue;
            // the group's last contributor: add its partials in segment order
            __threadfence();
            const float* base = p.ws + static_cast<long long>(t) * p.J * ELEMS;
            for (int e = ftid * 4; e < ELEMS; e += Cfg::FMA_THREADS * 4) {
                const int m = e / GN, col = e - (e / GN) * GN;
                if (m >= p.M) continue;
                float4 v = __ldcg(reinterpret_cast<const float4*>(base + e));
                for (int j = 1; j < nseg; ++j) {
                    const float4 x = __ldcg(reinterpret_cast<const float4*>(base + static_cast<long long>(j) * ELEMS + e));
                    v.x += x.x; v.y += x.y; v.z += x.z; v.w += x.w;
                }
                float o[4] = {v.x, v.y, v.z, v.w};
                if (p.relu)
#pragma unroll
                    for (int j = 0; j < 4; ++j) o[j] = fmaxf(o[j], 0.f);
                store_out4<OUT>(p.C, p.ldc, m, t * GN + col, p.N, o);
            }
        }
    }
    __syncthreads();
    // No CTA of a cluster exits before every peer has issued its stores.
    if (p.S > 1) {
        if (!cl_waited) cluster_wait_acquire();
        if (!cl_done) cluster_arrive_relaxed();
        cluster_wait_acquire();
    }
}

// The cluster split of cl_split for T column groups of KB k-units, lowered
// until the device holds all T clusters of that size at once; 0 selects
// stream-K.  `slot` is the kernel's attribute slot (set_smem_attr done).
template <class Cfg>
int gemv_cluster_split(long long T, long long KB, long long cap, int num_sms, int slot) {
    const void* k = reinterpret_cast<const void*>(gemv_kernel<Cfg>);
    int max_s = 8;
    for (;;) {
        const int S = cl_split(T, KB, Cfg::GN, cap, num_sms, max_s);
        if (S <= 1) return S;
        if (max_active_clusters(k, slot, S, Cfg::THREADS, Cfg::SMEM_BYTES) >= T) return S;
        max_s = S / 2;
    }
}

template <WKind W, int MR>
int run_gemv(const GemmArgs& a) {
    using Cfg = GvCfg<W, MR>;
    int dev = 0;
    const DeviceInfo* di = current_device(&dev);
    if (!di) return kNoDevice;
    auto kern = gemv_kernel<Cfg>;
    const int slot = (W == WKind::FP4 ? 58 : 40 + static_cast<int>(W) * 3) + (MR == 1 ? 0 : MR == 2 ? 1 : 2);
    if (set_smem_attr(reinterpret_cast<const void*>(kern), Cfg::SMEM_BYTES, slot) != cudaSuccess)
        return kCudaError;
    const long long cap = persistent_grid(di->num_sms, di->num_sms, a.ctas);
    SkPlan pl;
    if (!sk_plan(a.N, a.K, Cfg::GN, Cfg::BK, static_cast<int>(cap), &pl)) return kUnsupported;
    long long T = pl.T, KB = pl.KB, U = pl.U, G = pl.G, J = pl.J;
    // Split-K inside clusters where T groups times the split fill the GPU
    // (partials meet in distributed shared memory: no workspace); else
    // stream-K over G CTAs with a per-stream workspace.
    const int S = gemv_cluster_split<Cfg>(T, KB, cap, di->num_sms, slot);
    int* tickets = nullptr;
    float* ws = nullptr;
    if (S > 0) {
        G = T * S;
        J = 1;
    } else if (!stream_workspace(dev, a.stream, T, T * J * MR * Cfg::GN * 4, &tickets, &ws)) {
        return kCudaError;
    }

    const CUtensorMapDataType at = Cfg::ACT == WKind::BF16 ? CU_TENSOR_MAP_DATA_TYPE_BFLOAT16
                                                           : CU_TENSOR_MAP_DATA_TYPE_FLOAT16;
    CUtensorMap tW, tS, tX;
    if constexpr (Cfg::Q4) {
        if (!tensor_map_2d(&tW, a.B, CU_TENSOR_MAP_DATA_TYPE_UINT8, 1, (a.N + 1) / 2, a.K, a.ldb,
                           Cfg::GN / 2, Cfg::BK, SWZ_NONE))
            return kCudaError;
        const bool ok = Cfg::I4 ? tensor_map_2d(&tS, a.scales, CU_TENSOR_MAP_DATA_TYPE_FLOAT16, 2, a.N, a.K / 128,
                                                a.lds * 2, Cfg::GN, Cfg::SG, SWZ_NONE)
                                : tensor_map_2d(&tS, a.scales, CU_TENSOR_MAP_DATA_TYPE_UINT8, 1, a.N, (a.K + 31) / 32,
                                                a.lds, Cfg::GN, Cfg::SB, SWZ_NONE);
        if (!ok) return kCudaError;
    } else {
        if (!tensor_map_2d(&tW, a.B, at, 2, a.N, a.K, a.ldb * 2, 64, Cfg::BK, SWZ_NONE)) return kCudaError;
        tS = tW;                                   // unused
    }
    if (!tensor_map_2d(&tX, a.A, at, 2, a.K, a.M, a.lda * 2, Cfg::BK, MR, SWZ_NONE)) return kCudaError;

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
    const cudaStream_t stream = static_cast<cudaStream_t>(a.stream);
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
        return cudaLaunchKernelEx(&cfg, kern, tW, tS, tX, p) == cudaSuccess ? kOk : kCudaError;
    }
    kern<<<static_cast<int>(G), Cfg::THREADS, Cfg::SMEM_BYTES, stream>>>(tW, tS, tX, p);
    return cudaGetLastError() == cudaSuccess ? kOk : kCudaError;
}

template <WKind W>
int dispatch_gemv(const GemmArgs& a) {
    if (a.M <= 1) return run_gemv<W, 1>(a);
    if (a.M <= 2) return run_gemv<W, 2>(a);
    return run_gemv<W, 4>(a);
}

}  // namespace

int launch_gemv_bf16(const GemmArgs& a) { return dispatch_gemv<WKind::BF16>(a); }
int launch_gemv_f16(const GemmArgs& a) { return dispatch_gemv<WKind::F16>(a); }
int launch_gemv_w4a16(const GemmArgs& a) { return dispatch_gemv<WKind::INT4>(a); }
int launch_gemv_wfp4(const GemmArgs& a) { return dispatch_gemv<WKind::FP4>(a); }

}  // namespace tg
