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

}  // namespace tg
