// Host checks of the work-distribution arithmetic the kernels share
// (tile_sched.h): stream-K ranges, the weight-streaming launch plan, the
// grouped tile raster and the fp32 split-K ranges.  Each entry point walks a
// whole parameter grid, counts the properties it checked in *checked and
// returns how many of them failed.  Built with g++ by test_sched_host.py.
#include "tile_sched.h"

#include <vector>

using tg::sk_begin;
using tg::sk_owner;

extern "C" {

// Ranges [sk_begin(c), sk_begin(c+1)) of U units over G CTAs: they tile
// [0, U) in order, differ in size by at most one, are non-empty when G <= U,
// and sk_owner(u) names the range that holds u.
long long check_stream_k(int max_u, int max_g, long long* checked) {
    long long bad = 0, n = 0;
    for (int U = 1; U <= max_u; ++U) {
        for (int G = 1; G <= max_g; ++G) {
            const int lo = U / G, hi = (U + G - 1) / G;
            ++n; bad += sk_begin(0, U, G) != 0;
            ++n; bad += sk_begin(G, U, G) != U;
            for (int c = 0; c < G; ++c) {
                const int len = sk_begin(c + 1, U, G) - sk_begin(c, U, G);
                ++n; bad += len < lo || len > hi;
                if (G <= U) { ++n; bad += len == 0; }
            }
            for (int u = 0; u < U; ++u) {
                const int c = sk_owner(u, U, G);
                ++n;
                bad += c < 0 || c >= G || sk_begin(c, U, G) > u || sk_begin(c + 1, U, G) <= u;
            }
        }
    }
    *checked = n;
    return bad;
}

// The same near the int limit, where c * U overflows 32 bits.
long long check_stream_k_large(long long* checked) {
    long long bad = 0, n = 0;
    const int Us[] = {2147483647, 2147483646, 1 << 30, 1000000007};
    const int Gs[] = {1, 2, 147, 148, 296};
    for (int U : Us) {
        for (int G : Gs) {
            long long prev = 0;
            for (int c = 0; c < G; ++c) {
                const long long b = sk_begin(c, U, G), e = sk_begin(c + 1, U, G);
                ++n; bad += b != prev || e <= b;
                ++n; bad += b != static_cast<long long>(c) * U / G;
                ++n; bad += sk_owner(static_cast<int>(b), U, G) != c;
                ++n; bad += sk_owner(static_cast<int>(e - 1), U, G) != c;
                prev = e;
            }
            ++n; bad += prev != U;
        }
    }
    *checked = n;
    return bad;
}

// sk_plan against a brute-force walk: T and KB are ceilings, G = min(U,
// num_sms), and J is the largest number of CTAs whose ranges touch one
// column group's units, counted by walking every CTA's range unit by unit.
long long check_sk_plan(long long* checked) {
    long long bad = 0, n = 0;
    const long long Ns[] = {1, 2, 127, 128, 129, 255, 256, 257, 1000, 4096, 8192, 14336};
    const long long Ks[] = {1, 63, 64, 65, 128, 129, 1000, 4096, 8192};
    const int gns[] = {128, 256};
    const int bks[] = {64, 128};
    const int smss[] = {1, 7, 148};
    for (long long N : Ns) for (long long K : Ks) for (int gn : gns) for (int bk : bks)
    for (int sms : smss) {
        tg::SkPlan p;
        ++n;
        if (!tg::sk_plan(N, K, gn, bk, sms, &p)) { ++bad; continue; }
        const long long T = (N + gn - 1) / gn, KB = (K + bk - 1) / bk, U = T * KB;
        const long long G = U < sms ? U : sms;
        ++n; bad += p.T != T || p.KB != KB || p.U != U || p.G != G;
        std::vector<int> touching(T, 0), last(T, -1);
        for (int c = 0; c < G; ++c) {
            for (int u = sk_begin(c, int(U), int(G)); u < sk_begin(c + 1, int(U), int(G)); ++u) {
                const long long t = u / KB;
                if (last[t] != c) { last[t] = c; ++touching[t]; }
            }
        }
        long long J = 1;
        for (long long t = 0; t < T; ++t) J = touching[t] > J ? touching[t] : J;
        ++n; bad += p.J != J;
    }
    // unit counts past the int range are refused
    tg::SkPlan p;
    ++n; bad += tg::sk_plan(1ll << 40, 1ll << 20, 128, 128, 148, &p);
    *checked = n;
    return bad;
}

// tile_coords maps [0, ntm*ntn) one-to-one onto the tile grid, keeps index t
// in band t / (group_m * ntn), and inside a band steps down a tile column
// before moving to the next column.
long long check_tile_coords(int max_ntm, int max_ntn, long long* checked) {
    long long bad = 0, n = 0;
    const int groups[] = {1, 2, 3, 4, 8, 16};
    for (int ntm = 1; ntm <= max_ntm; ++ntm) for (int ntn = 1; ntn <= max_ntn; ++ntn)
    for (int gm : groups) {
        std::vector<char> seen(static_cast<size_t>(ntm) * ntn, 0);
        int ptm = -1, ptn = -1;
        for (int t = 0; t < ntm * ntn; ++t) {
            int tm, tn;
            tg::tile_coords(t, ntm, ntn, gm, tm, tn);
            ++n;
            if (tm < 0 || tm >= ntm || tn < 0 || tn >= ntn) { ++bad; continue; }
            char& s = seen[static_cast<size_t>(tm) * ntn + tn];
            ++n; bad += s != 0;
            s = 1;
            const int band = t / (gm * ntn);
            ++n; bad += tm / gm != band;
            if (t > 0 && t % (gm * ntn) != 0) {
                const bool down = tn == ptn && tm == ptm + 1;
                const bool next_col = tn == ptn + 1 && tm == band * gm;
                ++n; bad += !(down || next_col);
            }
            ptm = tm; ptn = tn;
        }
    }
    *checked = n;
    return bad;
}

// ffma_splits stays in [1, 8], is 1 when the tiles fill the SMs, never asks
// for more CTAs than SMs or fewer than 8 k-slices per range on average, and
// its ranges tile [0, kb_all) in order with none empty.
long long check_ffma_splits(int max_tiles, int max_kb, int num_sms, long long* checked) {
    long long bad = 0, n = 0;
    for (int tiles = 1; tiles <= max_tiles; ++tiles) for (int kb = 1; kb <= max_kb; ++kb) {
        const int s = tg::ffma_splits(tiles, kb, num_sms);
        ++n; bad += s < 1 || s > 8;
        if (tiles >= num_sms) { ++n; bad += s != 1; }
        if (s > 1) { ++n; bad += static_cast<long long>(s) * tiles > num_sms || s > kb / 8; }
        const int per = tg::ffma_kb_per(kb, s);
        int next = 0;
        for (int z = 0; z < s; ++z) {
            const int b = z * per, len = tg::ffma_range_len(b, per, kb);
            ++n; bad += b != next || len <= 0 || len > per;
            next = b + len;
        }
        ++n; bad += next != kb;
    }
    *checked = n;
    return bad;
}

// cl_split returns the largest admissible split S (none larger qualifies),
// or 0 exactly when no admissible split fills three quarters of the SMs;
// its cluster ranges tile [0, KB) with none empty.
static bool cl_admissible(long long T, long long KB, int gn, long long cap, int max_s, int S) {
    return S <= max_s && S <= KB && gn % (32 * S) == 0 && T * S <= cap;
}

long long check_cl_split(long long* checked) {
    long long bad = 0, n = 0;
    const int gns[] = {128, 256};
    const int smss[] = {1, 7, 132, 148};
    const int max_ss[] = {1, 2, 8};
    for (long long T = 1; T <= 300; ++T) for (long long KB = 1; KB <= 40; ++KB)
    for (int gn : gns) for (int sms : smss) for (int max_s : max_ss) {
        const long long caps[] = {sms, 2ll * sms, 128};
        for (long long cap : caps) {
            const int S = tg::cl_split(T, KB, gn, cap, sms, max_s);
            ++n;
            if (S != 0 && S != 1 && S != 2 && S != 4 && S != 8) { ++bad; continue; }
            int best = 0;
            for (int c = 8; c >= 1; c >>= 1)
                if (cl_admissible(T, KB, gn, cap, max_s, c)) { best = c; break; }
            const bool fills = best && T * best * 4 >= 3ll * sms;
            ++n; bad += S != (fills ? best : 0);
            if (S) {
                int next = 0;
                for (int r = 0; r < S; ++r) {
                    const int b = tg::cl_begin(r, int(KB), S), e = tg::cl_begin(r + 1, int(KB), S);
                    ++n; bad += b != next || e <= b;
                    next = e;
                }
                ++n; bad += next != KB;
            }
        }
    }
    // the shapes the weight-streaming kernels meet most
    ++n; bad += tg::cl_split(32, 128, 256, 148, 148, 8) != 4;     // 4-bit weights, N = 8192
    ++n; bad += tg::cl_split(64, 64, 128, 148, 148, 8) != 2;      // 16-bit weights, N = 8192
    ++n; bad += tg::cl_split(112, 32, 128, 148, 148, 8) != 1;     // 16-bit, N = 14336: whole groups
    ++n; bad += tg::cl_split(256, 64, 128, 148, 148, 8) != 0;     // more groups than SMs
    ++n; bad += tg::cl_split(20, 64, 128, 148, 148, 8) != 0;      // 80 CTAs at most: stream-K
    *checked = n;
    return bad;
}

// The CTA-pair kernel's hybrid schedule: the items cover every (tile,
// k-block) exactly once; items past the whole tiles are the two halves of
// the last R tiles (2R <= npairs, no half empty); handed out round-robin,
// the halves of a tile go to two different pairs, each pair gets at most
// one half and that is its last item.
long long check_tail_schedule(long long* checked) {
    long long bad = 0, n = 0;
    for (int npairs = 1; npairs <= 80; ++npairs)
    for (int tiles = 1; tiles <= 400; tiles += (tiles < 170 ? 1 : 7))
    for (int kb = 1; kb <= 9; kb += 2) {
        const int S = tg::tail_split(tiles, npairs, kb);
        const int dp = tg::tail_dp(tiles, npairs, S);
        const int items = tg::tail_items(tiles, dp, S);
        const int R = tiles % npairs;
        ++n; bad += !(S == 1 || S == 2);
        ++n; bad += S == 2 && !(R > 0 && 2 * R <= npairs && kb >= 2 && dp == tiles - R);
        ++n; bad += S == 1 && (dp != tiles || (R > 0 && 2 * R <= npairs && kb >= 2));
        std::vector<int> cover(static_cast<size_t>(tiles) * kb, 0);
        std::vector<int> last_item(npairs, -1), halves(npairs, 0), first_pair(tiles, -1);
        for (int w = 0; w < items; ++w) {
            int t, kb0, kb1, z;
            tg::tail_item(w, dp, S, kb, t, kb0, kb1, z);
            ++n;
            if (t < 0 || t >= tiles || kb0 < 0 || kb1 > kb || kb0 >= kb1) { ++bad; continue; }
            ++n; bad += (z >= 0) != (t >= dp);
            for (int k = kb0; k < kb1; ++k) ++cover[static_cast<size_t>(t) * kb + k];
            const int pr = w % npairs;
            last_item[pr] = w;
            if (z >= 0) {
                ++halves[pr];
                if (first_pair[t] < 0) first_pair[t] = pr;
                else { ++n; bad += first_pair[t] == pr; }
            }
        }
        for (int c : cover) { ++n; bad += c != 1; }
        for (int pr = 0; pr < npairs; ++pr) {
            ++n; bad += halves[pr] > 1;
            if (halves[pr]) { ++n; bad += last_item[pr] < dp; }
        }
    }
    *checked = n;
    return bad;
}

}  // extern "C"
