// tile_sched.h -- work-distribution arithmetic shared by the kernels and their
// launchers: the stream-K split of the weight-streaming kernels, the grouped
// tile raster of the persistent kernels, and the split-K ranges of the fp32
// FFMA kernel.  Plain C++ with no CUDA types, so that the host tests build it
// with g++ and check every partition it produces.
#pragma once

#if defined(__CUDACC__)
#define TG_HD __host__ __device__ __forceinline__
#else
#define TG_HD inline
#endif

namespace tg {

TG_HD int sched_min(int a, int b) {
#if defined(__CUDA_ARCH__)
    return min(a, b);
#else
    return a < b ? a : b;
#endif
}

TG_HD int sched_max(int a, int b) {
#if defined(__CUDA_ARCH__)
    return max(a, b);
#else
    return a > b ? a : b;
#endif
}

// ---------------------------------------------------------------- stream-K
// U work units (column group t owns units [t*KB, t*KB + KB)) are cut into G
// contiguous ranges, CTA c taking [sk_begin(c), sk_begin(c + 1)).  Range
// sizes are floor(U/G) or ceil(U/G); with G <= U none is empty.

TG_HD int sk_begin(int c, int U, int G) {
    return static_cast<int>((static_cast<long long>(c) * U) / G);
}

// CTA whose range holds unit u (0 <= u < U).  When G > U some ranges are
// empty; the owner is the one non-empty range that holds u.  The first guess
// floor(u*G/U) never lies past the owner (its range starts at or before u),
// so the upward step does the work; the downward one only guards the guess.
TG_HD int sk_owner(int u, int U, int G) {
    int c = static_cast<int>((static_cast<long long>(u) * G) / U);
    while (c + 1 < G && sk_begin(c + 1, U, G) <= u) ++c;
    while (c > 0 && sk_begin(c, U, G) > u) --c;
    return c;
}

// Launch plan of a weight-streaming kernel: T column groups of gn columns,
// KB k-units of bk rows each, U = T*KB units over G = min(U, num_sms) CTAs,
// and J = the most ranges (segments) any one column group is cut into, which
// sizes its split-K partial slots.
struct SkPlan {
    long long T, KB, U, G, J;
};

// False when U does not fit the kernels' int unit indices.
inline bool sk_plan(long long N, long long K, int gn, int bk, int num_sms, SkPlan* p) {
    p->T = (N + gn - 1) / gn;
    p->KB = (K + bk - 1) / bk;
    p->U = p->T * p->KB;
    if (p->U > 0x7fffffffll) return false;
    p->G = p->U < num_sms ? p->U : num_sms;
    p->J = 1;
    const int U = static_cast<int>(p->U), G = static_cast<int>(p->G);
    for (long long t = 0; t < p->T; ++t) {
        const long long n = sk_owner(static_cast<int>(t * p->KB + p->KB - 1), U, G) -
                            sk_owner(static_cast<int>(t * p->KB), U, G) + 1;
        if (n > p->J) p->J = n;
    }
    return true;
}

// ------------------------------------------------- split-K inside a cluster
// The alternative to stream-K when T column groups times a small split S
// fill the GPU: group t goes to the S CTAs of cluster t, and rank r of the
// cluster takes the k-units [t*KB + cl_begin(r), t*KB + cl_begin(r + 1)).
// The ranks then sum their partials through distributed shared memory, each
// rank owning gn/S columns of the group.

TG_HD int cl_begin(int r, int KB, int S) {
    return static_cast<int>((static_cast<long long>(r) * KB) / S);
}

// The split S in {8, 4, 2, 1} for T groups of gn columns and KB k-units, or 0
// (use stream-K): the largest S with no empty range (S <= KB), whole 32-column
// warp slices per owner (gn a multiple of 32*S), T*S <= cap CTAs, and T*S at
// least three quarters of num_sms (fewer CTAs would leave HBM bandwidth
// unused).  `max_s` bounds S (a smaller maximum cluster on the device).
inline int cl_split(long long T, long long KB, int gn, long long cap, int num_sms, int max_s) {
    for (int S = 8; S >= 1; S >>= 1) {
        if (S > max_s || S > KB || gn % (32 * S) != 0 || T * S > cap) continue;
        return T * S * 4 >= 3ll * num_sms ? S : 0;
    }
    return 0;
}

// ------------------------------------------- hybrid schedule of the pairs
// The persistent CTA-pair kernel hands out work items round-robin to its
// npairs pairs.  Whole tiles fill the full waves; when the R tiles left for
// the last wave would leave at least half of the pairs idle (2R <= npairs),
// each of them is split into two halves of its k-blocks, so the last wave
// takes about half a tile's time.  tail_dp() is the number of items that
// are whole tiles (all tiles when there is no split).

TG_HD int tail_split(int num_tiles, int npairs, int num_kb) {
    const int R = num_tiles % npairs;
    return (R > 0 && 2 * R <= npairs && num_kb >= 2) ? 2 : 1;
}

TG_HD int tail_dp(int num_tiles, int npairs, int S) {
    return S > 1 ? num_tiles - num_tiles % npairs : num_tiles;
}

TG_HD int tail_items(int num_tiles, int dp, int S) { return dp + (num_tiles - dp) * S; }

// Item w -> tile t, k-blocks [kb0, kb1), and the half z (-1 for a whole tile).
TG_HD void tail_item(int w, int dp, int S, int num_kb, int& t, int& kb0, int& kb1, int& z) {
    if (S <= 1 || w < dp) {
        t = w;
        kb0 = 0;
        kb1 = num_kb;
        z = -1;
        return;
    }
    const int i = (w - dp) / S;
    z = (w - dp) - i * S;
    t = dp + i;
    kb0 = static_cast<int>((static_cast<long long>(z) * num_kb) / S);
    kb1 = static_cast<int>((static_cast<long long>(z + 1) * num_kb) / S);
}

// ------------------------------------------------------------ tile raster
// Linear tile index t of an ntm x ntn tile grid -> (tm, tn).  Tiles are taken
// in bands of group_m tile rows (the last band may be shorter); inside a band
// the index runs down the rows of one tile column, then to the next column,
// so CTAs working at the same time share the band's A rows and a few B
// columns in L2.
TG_HD void tile_coords(int t, int ntm, int ntn, int group_m, int& tm, int& tn) {
    const int per_group = group_m * ntn;
    const int g = t / per_group;
    const int first_m = g * group_m;
    const int gsz = sched_min(ntm - first_m, group_m);
    const int local = t - g * per_group;
    tm = first_m + local % gsz;
    tn = local / gsz;
}

// ------------------------------------------------------- fp32 split-K
// Number of k ranges per output tile: 1 when the tiles already fill the SMs;
// otherwise enough to fill them, with at most 8 ranges and no more ranges than
// kb_all / 8 (so a range averages at least 8 k-slices).
inline int ffma_splits(long long tiles, long long kb_all, int num_sms) {
    long long s = 1;
    if (tiles < num_sms) {
        s = num_sms / tiles;
        if (s > kb_all / 8) s = kb_all / 8;
        if (s > 8) s = 8;
        if (s < 1) s = 1;
    }
    return static_cast<int>(s);
}

// Split-K ranges over kb_all k-slices: range z is [z * kb_per, z * kb_per +
// ffma_range_len(z * kb_per, kb_per, kb_all)), kb_per = ffma_kb_per(kb_all,
// splits) = ceil(kb_all / splits).  Every range is kb_per long except a
// shorter last one, which is never empty for a split count from ffma_splits.
TG_HD int ffma_kb_per(int kb_all, int splits) { return (kb_all + splits - 1) / splits; }

TG_HD int ffma_range_len(int kb0, int kb_per, int kb_all) {
    return sched_max(0, sched_min(kb_all, kb0 + kb_per) - kb0);
}

}  // namespace tg
