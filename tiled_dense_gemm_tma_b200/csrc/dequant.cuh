// dequant.cuh -- 4-bit weight -> fp16 conversion into a tensor-core operand tile.
//
// Weight format (the library's reading of the dequantize GEMM the pages
// name, "使用 Tilelang DSL 开发 GPU/CPU/加速器高性能内核", blog.hotdry.top):
// signed 4-bit q in [-8, 7], two per byte, column 2j in the low nibble of
// byte j; fp16 scales s per 128 rows of K; W[k][n] = fp16(q[k][n] * s[k/128][n]).
//
// One 32-bit word of packed weights holds 8 consecutive columns c0..c7.
// Flipping bit 3 of every nibble turns q into u = q + 8 in [0, 15]; placing
// u in the low byte of the fp16 pattern 0x6400 gives the value 1024 + u, and
// subtracting 1032 recovers q exactly.  The byte permutes that build those
// fp16 pairs take one source byte per half, so the 8 columns come out as the
// pairs (c0,c2) (c4,c6) (c1,c3) (c5,c7): the tile stores each 8-column group
// in the order 0,2,4,6,1,3,5,7 and the epilogue undoes it (perm8_src).
// Multiplying the exact q by the fp16 scale with one fp16 multiply rounds
// the exact product once, so the result equals fp16(q * s).
#pragma once
#include <cuda_fp16.h>
#include <cstdint>

namespace tg {

__device__ __forceinline__ uint32_t hsub2_u32(uint32_t a, uint32_t b) {
    __half2 r = __hsub2(*reinterpret_cast<__half2*>(&a), *reinterpret_cast<__half2*>(&b));
    return *reinterpret_cast<uint32_t*>(&r);
}

__device__ __forceinline__ uint32_t hmul2_u32(uint32_t a, uint32_t b) {
    __half2 r = __hmul2(*reinterpret_cast<__half2*>(&a), *reinterpret_cast<__half2*>(&b));
    return *reinterpret_cast<uint32_t*>(&r);
}

// 8 packed weights (one word) times their 4 permuted scale pairs -> 4 words
// of fp16 pairs in the order (c0,c2) (c4,c6) (c1,c3) (c5,c7).
__device__ __forceinline__ uint4 dequant8(uint32_t w, const uint32_t (&sp)[4]) {
    const uint32_t lo = (w & 0x0F0F0F0Fu) ^ 0x08080808u;          // u0 u2 u4 u6
    const uint32_t hi = ((w >> 4) & 0x0F0F0F0Fu) ^ 0x08080808u;   // u1 u3 u5 u7
    const uint32_t k64 = 0x64646464u;
    const uint32_t bias = 0x64086408u;                              // (1032, 1032)
    uint4 r;
    r.x = hmul2_u32(hsub2_u32(__byte_perm(lo, k64, 0x4140), bias), sp[0]);
    r.y = hmul2_u32(hsub2_u32(__byte_perm(lo, k64, 0x4342), bias), sp[1]);
    r.z = hmul2_u32(hsub2_u32(__byte_perm(hi, k64, 0x4140), bias), sp[2]);
    r.w = hmul2_u32(hsub2_u32(__byte_perm(hi, k64, 0x4342), bias), sp[3]);
    return r;
}

// Scale pairs matching dequant8's column order, from 8 consecutive fp16
// scales held as 4 words (s0,s1) (s2,s3) (s4,s5) (s6,s7).
__device__ __forceinline__ void scale_pairs(const uint4 s, uint32_t (&sp)[4]) {
    sp[0] = __byte_perm(s.x, s.y, 0x5410);     // (s0, s2)
    sp[1] = __byte_perm(s.z, s.w, 0x5410);     // (s4, s6)
    sp[2] = __byte_perm(s.x, s.y, 0x7632);     // (s1, s3)
    sp[3] = __byte_perm(s.z, s.w, 0x7632);     // (s5, s7)
}

// Convert a BK x BN weight slice.
//   raw:  BK rows of BN/2 packed bytes, row pitch BN/2, stored by the copy
//         engine with its 128-byte (BN = 256) or 64-byte (BN = 128) swizzle:
//         16-byte unit c of row k sits at unit c ^ (k & 7), resp. c ^ ((k >> 1) & 3)
//   srow: BN fp16 scales of the slice's group (shared memory)
//   dst:  BN/64 column blocks, CHUNK_BYTES apart; in each, row k of 64 fp16
//         at k * 128, 16-byte unit u at ((u ^ (k & 7)) * 16) -- the N-major
//         128-byte-swizzled operand layout.
// NT threads share the work; `tid` in [0, NT).  Each group of 8 consecutive
// threads takes 8 consecutive rows of one 32-column segment, so both its
// swizzled reads and its swizzled writes fall in 8 distinct bank groups.
template <int BK, int BN, int NT, int CHUNK_BYTES>
__device__ __forceinline__ void dequant_slice(const uint8_t* raw, const uint8_t* srow,
                                              uint8_t* dst, int tid) {
    constexpr int PITCH = BN / 2;                 // raw bytes per row: 128 or 64
    constexpr int SEGS = BN / 32;                 // 16 raw bytes = 32 columns per segment
    constexpr int ROWS_PER_PASS = NT / SEGS;
    static_assert(BN == 256 || BN == 128, "raw row must be one swizzle span");
    static_assert(NT % (8 * SEGS) == 0 && BK % ROWS_PER_PASS == 0, "bad split");
    const int seg = (tid >> 3) % SEGS;
    const int r0 = (tid & 7) + 8 * (tid / (8 * SEGS));
    uint32_t sp[4][4];
#pragma unroll
    for (int j = 0; j < 4; ++j)
        scale_pairs(*reinterpret_cast<const uint4*>(srow + seg * 64 + j * 16), sp[j]);
    uint8_t* cbase = dst + (seg >> 1) * CHUNK_BYTES;
    const int ubase = (seg & 1) * 4;
#pragma unroll
    for (int i = 0; i < BK / ROWS_PER_PASS; ++i) {
        const int k = r0 + i * ROWS_PER_PASS;
        const int ru = PITCH == 128 ? (seg ^ (k & 7)) : (seg ^ ((k >> 1) & 3));
        const uint4 w = *reinterpret_cast<const uint4*>(raw + k * PITCH + (ru << 4));
        uint8_t* rowp = cbase + k * 128;
        const uint32_t ws[4] = {w.x, w.y, w.z, w.w};
#pragma unroll
        for (int j = 0; j < 4; ++j)
            *reinterpret_cast<uint4*>(rowp + (((ubase + j) ^ (k & 7)) << 4)) = dequant8(ws[j], sp[j]);
    }
}

// ------------------------------------------------------- FP4 (MXFP4) weights
//
// FP4-weight format (the library's reading of the WFP4 GEMM named on
// "TileLang架构深度剖析" (test.krestaai.com.au), 性能表现与基准测试验证: the
// MXFP4 encoding of the OCP Microscaling Formats (MX) specification v1.0):
// each weight is an E2M1 code -- sign bit 3, exponent bits 2-1 (bias 1),
// mantissa bit 0, magnitudes {0, 0.5, 1, 1.5, 2, 3, 4, 6} -- packed two per
// byte like the 4-bit integers (column 2j in the low nibble); 32 consecutive
// k of a column share one E8M0 scale byte E, 2^(E - 127) (E = 255: NaN).
// W[k][n] = e2m1(code) * 2^(E - 127), formed exactly as a bf16 operand.
//
// Decode without a table: with x = code & 7 and s = code >> 3, the bf16 bit
// pattern s << 15 | x << 6 has exponent field x >> 1 and top mantissa bit
// x & 1, which is the E2M1 value times 2^-126 for every code (x = 1, the
// value 0.5, lands on the bf16 subnormal 2^-127).  Two codes sitting in
// bytes 0 and 2 of a word t become such a bf16 pair with one multiply and
// one mask: t * 0x1040 = t << 12 | t << 6 (the four shifted nibbles do not
// overlap), & 0x81C081C0 keeps the two sign bits and the two magnitudes.
// Two exact bf16 multiplies by powers of two then apply 2^126 * 2^(E - 127):
// m1 = 2^(min(E, 128) - 1) and m2 = 2^(max(E, 128) - 128) (NaN for E = 255),
// both normal bf16; m2 is 1 unless E > 128.  Every product is exact for
// E <= 252 (6 * 2^(E - 127) is then below the bf16 maximum); subnormal
// results (small E) are exact too, as E2M1 values carry two significant bits.

__device__ __forceinline__ uint32_t hmul2_bf16_u32(uint32_t a, uint32_t b) {
    uint32_t r;
    asm("mul.rn.bf16x2 %0, %1, %2;" : "=r"(r) : "r"(a), "r"(b));
    return r;
}

// bf16 pair patterns (value * 2^-126) of the codes in bytes 0 and 2 of t.
__device__ __forceinline__ uint32_t e2m1_pair_scaled_down(uint32_t t) {
    return (t * 0x1040u) & 0x81C081C0u;
}

// Multiplier words for 4 columns whose E8M0 bytes are e (one per byte):
// bytes of m1 = min(E, 128) + 126, bytes of m2 = max(E, 128) - 1, or 255
// where E = 255 (exponent fields of the two bf16 factors).
__device__ __forceinline__ void e8m0_factor_bytes(uint32_t e, uint32_t& m1, uint32_t& m2) {
    m1 = __vminu4(e, 0x80808080u) + 0x7E7E7E7Eu;                 // <= 254 per byte: no carries
    m2 = (__vmaxu4(e, 0x80808080u) - 0x01010101u) | __vcmpeq4(e, 0xFFFFFFFFu);
}

// bf16 pair (2^(a - 127), 2^(b - 127)) from exponent bytes a, b in bytes 0
// and 2 of t (other bytes zero): the bytes shifted into the exponent fields.
__device__ __forceinline__ uint32_t bf16_pow2_pair(uint32_t t) { return t << 7; }

// Scale factors of one thread's 8 consecutive columns c0..c7 (E8M0 bytes
// e_lo = c0..c3, e_hi = c4..c7), in the converter's pair order (c0,c2)
// (c4,c6) (c1,c3) (c5,c7): f1[j] (and f2[j]) multiply pair j.  Returns false
// when every f2 would be 1 (no E above 128), so the second multiply is
// skipped; f2 is then left unset.  A NaN scale (E = 255) makes f2 NaN.
__device__ __forceinline__ bool fp4_scale_pairs(uint32_t e_lo, uint32_t e_hi, uint32_t (&f1)[4],
                                                uint32_t (&f2)[4]) {
    // Every E <= 128 (the usual case): m1 = E + 126 byte by byte and m2 = 1,
    // the same factors as the general path below at a fraction of its
    // per-byte min / max / compare work.  A byte is above 128 exactly when
    // its bit 7 is set and some lower bit too.
    const uint32_t above = (((e_lo & 0x7F7F7F7Fu) + 0x7F7F7F7Fu) & e_lo) |
                           (((e_hi & 0x7F7F7F7Fu) + 0x7F7F7F7Fu) & e_hi);
    if ((above & 0x80808080u) == 0) {
        const uint32_t a = e_lo + 0x7E7E7E7Eu, b = e_hi + 0x7E7E7E7Eu;   // <= 254: no carries
        f1[0] = bf16_pow2_pair(__byte_perm(a, 0u, 0x4240));
        f1[1] = bf16_pow2_pair(__byte_perm(b, 0u, 0x4240));
        f1[2] = bf16_pow2_pair(__byte_perm(a, 0u, 0x4341));
        f1[3] = bf16_pow2_pair(__byte_perm(b, 0u, 0x4341));
        return false;
    }
    uint32_t a1, a2, b1, b2;
    e8m0_factor_bytes(e_lo, a1, a2);
    e8m0_factor_bytes(e_hi, b1, b2);
    f1[0] = bf16_pow2_pair(__byte_perm(a1, 0u, 0x4240));     // (c0, c2)
    f1[1] = bf16_pow2_pair(__byte_perm(b1, 0u, 0x4240));     // (c4, c6)
    f1[2] = bf16_pow2_pair(__byte_perm(a1, 0u, 0x4341));     // (c1, c3)
    f1[3] = bf16_pow2_pair(__byte_perm(b1, 0u, 0x4341));     // (c5, c7)
    if ((a2 | b2) == 0x7F7F7F7Fu) return false;              // every m2 byte 127: factor 1
    const uint32_t na = __vcmpeq4(e_lo, 0xFFFFFFFFu), nb = __vcmpeq4(e_hi, 0xFFFFFFFFu);
    const uint32_t sel[4] = {0x4240, 0x4240, 0x4341, 0x4341};
#pragma unroll
    for (int j = 0; j < 4; ++j) {
        const uint32_t m = (j & 1) ? b2 : a2, n = (j & 1) ? nb : na;
        // byte 255 -> 0x7F80 (inf) plus the quiet bit 0x0040: NaN
        f2[j] = bf16_pow2_pair(__byte_perm(m, 0u, sel[j])) |
                ((__byte_perm(n, 0u, sel[j]) >> 1) & 0x00400040u);
    }
    return true;
}

// 8 packed E2M1 codes (one word: columns c0..c7) -> 4 words of bf16 pairs in
// the order (c0,c2) (c4,c6) (c1,c3) (c5,c7), the 4-bit integer converter's
// order, so the same epilogue column permutation applies.
template <bool TWO>
__device__ __forceinline__ uint4 dequant8_fp4(uint32_t w, const uint32_t (&f1)[4],
                                              const uint32_t (&f2)[4]) {
    const uint32_t lo = w & 0x0F0F0F0Fu;                 // c0 c2 c4 c6
    const uint32_t hi = (w >> 4) & 0x0F0F0F0Fu;          // c1 c3 c5 c7
    uint32_t r[4] = {e2m1_pair_scaled_down(__byte_perm(lo, 0u, 0x4140)),
                     e2m1_pair_scaled_down(__byte_perm(lo, 0u, 0x4342)),
                     e2m1_pair_scaled_down(__byte_perm(hi, 0u, 0x4140)),
                     e2m1_pair_scaled_down(__byte_perm(hi, 0u, 0x4342))};
#pragma unroll
    for (int j = 0; j < 4; ++j) {
        r[j] = hmul2_bf16_u32(r[j], f1[j]);
        if (TWO) r[j] = hmul2_bf16_u32(r[j], f2[j]);
    }
    return make_uint4(r[0], r[1], r[2], r[3]);
}

// Convert a BK x BN FP4 weight slice into the bf16 N-major 128-byte-swizzled
// operand layout of dequant_slice (same raw and destination layouts).
//   sraw: BK/32 rows of BN E8M0 scale bytes (row r covers k in [32r, 32r+32))
// Thread t takes 8 consecutive columns (column group t % (BN/8)) of RPT rows
// inside one 8-row group (so inside one 32-row scale block: its scale
// factors are built once per slice).  A warp covers one row (BN = 256) or
// two neighbouring rows (BN = 128, 64-byte packed rows): its packed reads
// are 128 distinct bytes, and each 8 threads write one 128-byte bf16 row of
// a 64-column chunk as 8 distinct 16-byte units.
template <int BK, int BN, int NT, int CHUNK_BYTES>
__device__ __forceinline__ void dequant_slice_fp4(const uint8_t* raw, const uint8_t* sraw,
                                                  uint8_t* dst, int tid) {
    constexpr int PITCH = BN / 2;
    constexpr int CG = BN / 8;                    // column groups of 8
    constexpr int RB = NT / CG;                   // row blocks
    constexpr int RPT = BK / RB;                  // rows per thread
    constexpr int WR = 32 / CG;                   // row blocks per warp: 1 or 2
    static_assert(BN == 256 || BN == 128, "raw row must be one swizzle span");
    static_assert(NT % 32 == 0 && NT % CG == 0 && BK % RB == 0 && WR * RPT == 8, "bad split");
    const int cg = tid % CG;
    const int rb = tid / CG;
    const int r0 = (rb / WR) * 8 + (rb % WR);     // rows r0 + WR * i, i < RPT
    const uint2 ev = *reinterpret_cast<const uint2*>(sraw + (r0 / 32) * BN + cg * 8);
    uint32_t f1[4], f2[4];
    const bool two = fp4_scale_pairs(ev.x, ev.y, f1, f2);
    uint8_t* cbase = dst + (cg >> 3) * CHUNK_BYTES;
    const int u = cg & 7;                         // 16-byte unit of the 64-column chunk
    const int cu = cg >> 2;                       // 16-byte unit of the packed row
    const int cw = (cg & 3) * 4;                  // byte offset inside it
#pragma unroll
    for (int i = 0; i < RPT; ++i) {
        const int k = r0 + WR * i;
        const int ru = PITCH == 128 ? (cu ^ (k & 7)) : (cu ^ ((k >> 1) & 3));
        const uint32_t w = *reinterpret_cast<const uint32_t*>(raw + k * PITCH + (ru << 4) + cw);
        uint4 v = two ? dequant8_fp4<true>(w, f1, f2) : dequant8_fp4<false>(w, f1, f2);
        *reinterpret_cast<uint4*>(cbase + k * 128 + ((u ^ (k & 7)) << 4)) = v;
    }
}

}  // namespace tg
