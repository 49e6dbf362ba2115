// block_select.cuh -- exact top-k of up to a few thousand order-preserving
// 32-bit score keys by NW warps of one CTA, synchronised on a named barrier
// (other warps of the CTA may have left).
//
// Each thread holds KPT keys in registers; warp w owns the contiguous
// positions [w * 32 * KPT, (w + 1) * 32 * KPT), lane l the positions
// w * 32 * KPT + j * 32 + l.  Positions at or past n hold key 0, the smallest
// key: they lie after every real position, so they never displace one (a
// real key equal to 0 -- a NaN score -- comes first in position order).
//
// Up to 2 * 32 * NW keys, each thread ranks its keys against all of them
// (keys above, plus equal keys at a lower position) and keeps ranks below k.
// Longer lists:
//   1. A histogram of the top 12 bits of the keys (sign, exponent and three
//      mantissa bits of the score; the wide digit spreads typical scores over
//      many bins, so few lanes of a warp add to the same counter) gives the
//      digit of the k-th largest key T and how many keys lie above it.
//      Counters are 16 bits, two to a word (n < 65536).
//   2. When at most 32 * NW keys share T's digit (the usual case: the top-k
//      of a few thousand scores ends in a thin bin), they are gathered and
//      ranked among themselves, which gives T.  Otherwise two more passes of
//      12 and 8 bits, each over the keys that match the digits found so far,
//      give T's remaining bits.
//   3. A compaction in position order takes every key > T and the first
//      (k - #keys > T) keys equal to T, so equal scores go to the lower
//      position, as the selection rule requires; positions come out
//      ascending.  Each warp counts its segment with ballots, one barrier
//      publishes the warps' counts, and each key's output slot is
//      (#keys > T before it) + min(#keys == T before it, k - #keys > T).
#pragma once

#include "common.cuh"

namespace sa {

constexpr int kBsMaxWarps = 16;
constexpr int kBsBins = 4096;   // widest digit: 12 bits

constexpr int kBsCand = 32 * kBsMaxWarps;   // keys of T's digit ranked directly

struct BsSmem {
    uint32_t hist[2][kBsBins / 2];   // 16-bit counters, bin b in half (b & 1) of word b >> 1
    int misc[2][3];                  // per pass: T's digit, keys above that digit, keys of that digit
    int wcnt[kBsMaxWarps][2];        // per warp: scan totals; keys > T, keys == T
    uint32_t cand[kBsCand];          // keys of T's first digit
    int ncand;
    uint32_t T;
    int take;
};

template <int NT>
__device__ __forceinline__ void named_bar_sync(int id) {
    asm volatile("bar.sync %0, %1;" ::"r"(id), "n"(NT) : "memory");
}

// Positions (ascending) of the top-k keys of keys[0..n) into out[0..k):
// every position when n <= k.  n <= NW * 32 * KPT < 65536.  Called by the
// threads 0 .. NW*32-1 of the CTA together; returns the count (uniform).
template <int NW, int KPT>
__device__ int block_topk32(const uint32_t *keys, int n, int k, int *out, BsSmem &bs, int bar_id) {
    static_assert(NW <= kBsMaxWarps && NW * 32 * KPT < 65536, "shape");
    constexpr int NT = NW * 32;
    constexpr int WPT = kBsBins / 2 / NT;      // histogram words per thread in the scan
    static_assert(WPT * NT * 2 == kBsBins, "scan split");
    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    if (k <= 0 || n <= 0) return 0;
    if (n <= k) {
        for (int i = tid; i < n; i += NT) out[i] = i;
        named_bar_sync<NT>(bar_id);
        return n;
    }
    const unsigned below = (1u << lane) - 1u;
    if (n <= 2 * NT) {
        // rank every key: keys above it, plus equal keys at a lower position
        bool sel[2] = {false, false};
#pragma unroll
        for (int h = 0; h < 2; ++h) {
            const int p = h * NT + tid;
            if (h * NT >= n) break;                       // uniform
            if (p < n) {
                const uint32_t x = keys[p];
                int rk = 0;
                for (int i = 0; i < n; ++i) {
                    const uint32_t y = keys[i];
                    rk += (y > x) | ((y == x) & (i < p));
                }
                sel[h] = rk < k;
            }
        }
        const unsigned m0 = __ballot_sync(0xffffffffu, sel[0]), m1 = __ballot_sync(0xffffffffu, sel[1]);
        if (lane == 0) {
            bs.wcnt[warp][0] = __popc(m0);
            bs.wcnt[warp][1] = __popc(m1);
        }
        named_bar_sync<NT>(bar_id);
        int b0 = 0, t0 = 0, b1 = 0;
#pragma unroll
        for (int w = 0; w < NW; ++w) {
            t0 += bs.wcnt[w][0];
            if (w < warp) {
                b0 += bs.wcnt[w][0];
                b1 += bs.wcnt[w][1];
            }
        }
        if (sel[0]) out[b0 + __popc(m0 & below)] = tid;
        if (sel[1]) out[t0 + b1 + __popc(m1 & below)] = NT + tid;
        named_bar_sync<NT>(bar_id);
        return k;
    }
    const int p0 = warp * 32 * KPT + lane;
    uint32_t r[KPT];
    unsigned valid = 0u;
#pragma unroll
    for (int j = 0; j < KPT; ++j) {
        const bool v = p0 + j * 32 < n;
        r[j] = v ? keys[p0 + j * 32] : 0u;
        valid |= (v ? 1u : 0u) << j;
    }
    for (int i = tid; i < kBsBins / 2; i += NT) bs.hist[0][i] = 0u;
    if (tid == 0) bs.ncand = 0;
    named_bar_sync<NT>(bar_id);

    // ---- 1. T's first digit; 2. T from its digit's keys, or two more digits
    uint32_t prefix = 0u, mask = 0u;
    int kr = k;   // rank of T among the keys that match `prefix`
    uint32_t T = 0u;
#pragma unroll 1
    for (int pass = 0; pass < 3; ++pass) {
        const int bits = pass < 2 ? 12 : 8;
        const int shift = pass == 0 ? 20 : (pass == 1 ? 8 : 0);
        const uint32_t dmask = (1u << bits) - 1u;
        const int cur = pass & 1;
#pragma unroll
        for (int j = 0; j < KPT; ++j)
            if (((valid >> j) & 1u) && (r[j] & mask) == prefix) {
                const uint32_t bin = (r[j] >> shift) & dmask;
                atomicAdd(&bs.hist[cur][bin >> 1], 1u << (16 * (bin & 1u)));
            }
        for (int i = tid; i < kBsBins / 2; i += NT) bs.hist[cur ^ 1][i] = 0u;
        named_bar_sync<NT>(bar_id);
        // thread t scans bins kBsBins-1-2*WPT*t down to kBsBins-2*WPT*(t+1)
        int c[2 * WPT], sum = 0;
#pragma unroll
        for (int w = 0; w < WPT; ++w) {
            const uint32_t x = bs.hist[cur][kBsBins / 2 - 1 - WPT * tid - w];
            c[2 * w] = (int)(x >> 16);
            c[2 * w + 1] = (int)(x & 0xffffu);
            sum += c[2 * w] + c[2 * w + 1];
        }
        int incl = sum;
#pragma unroll
        for (int o = 1; o < 32; o <<= 1) {
            const int t = __shfl_up_sync(0xffffffffu, incl, o);
            if (lane >= o) incl += t;
        }
        if (lane == 31) bs.wcnt[warp][0] = incl;
        named_bar_sync<NT>(bar_id);
#pragma unroll
        for (int w = 0; w < NW; ++w)
            if (w < warp) incl += bs.wcnt[w][0];
        const int excl = incl - sum;
        if (excl < kr && incl >= kr) {
            int run = excl, found = 0, above = 0, inbin = 0;
            bool done = false;
#pragma unroll
            for (int e = 0; e < 2 * WPT; ++e) {
                if (!done && run + c[e] >= kr) {
                    found = kBsBins - 1 - 2 * WPT * tid - e;
                    above = run;
                    inbin = c[e];
                    done = true;
                }
                run += c[e];
            }
            bs.misc[cur][0] = found;
            bs.misc[cur][1] = above;
            bs.misc[cur][2] = inbin;
        }
        named_bar_sync<NT>(bar_id);
        prefix |= (uint32_t)bs.misc[cur][0] << shift;
        mask |= dmask << shift;
        kr -= bs.misc[cur][1];
        T = prefix;
        if (pass == 0 && bs.misc[0][2] <= NT) {
            // the keys of T's digit, gathered in any order and ranked among
            // themselves: T is the one with fewer than kr above it and at
            // least kr at or above it (equal keys write the same values)
            const int m = bs.misc[0][2];
#pragma unroll
            for (int j = 0; j < KPT; ++j)
                if (((valid >> j) & 1u) && (r[j] & mask) == prefix) bs.cand[atomicAdd(&bs.ncand, 1)] = r[j];
            named_bar_sync<NT>(bar_id);
            if (tid < m) {
                const uint32_t x = bs.cand[tid];
                int gt = 0, ge = 0;
                for (int i = 0; i < m; ++i) {
                    const uint32_t y = bs.cand[i];
                    gt += y > x;
                    ge += y >= x;
                }
                if (gt < kr && ge >= kr) {
                    bs.T = x;
                    bs.take = kr - gt;
                }
            }
            named_bar_sync<NT>(bar_id);
            T = bs.T;
            kr = bs.take;
            break;
        }
    }

    // ---- 3. compaction in position order -----------------------------------
    unsigned gtm[KPT], eqm[KPT];
    int G = 0, E = 0;
#pragma unroll
    for (int j = 0; j < KPT; ++j) {
        const bool v = (valid >> j) & 1u;
        gtm[j] = __ballot_sync(0xffffffffu, v && r[j] > T);
        eqm[j] = __ballot_sync(0xffffffffu, v && r[j] == T);
        G += __popc(gtm[j]);
        E += __popc(eqm[j]);
    }
    if (lane == 0) {
        bs.wcnt[warp][0] = G;
        bs.wcnt[warp][1] = E;
    }
    named_bar_sync<NT>(bar_id);
    int gb = 0, eb = 0;
#pragma unroll
    for (int w = 0; w < NW; ++w)
        if (w < warp) {
            gb += bs.wcnt[w][0];
            eb += bs.wcnt[w][1];
        }
#pragma unroll
    for (int j = 0; j < KPT; ++j) {
        const int g_here = gb + __popc(gtm[j] & below), e_here = eb + __popc(eqm[j] & below);
        const bool gt = (gtm[j] >> lane) & 1u, eq = (eqm[j] >> lane) & 1u;
        if (gt || (eq && e_here < kr)) out[g_here + min(e_here, kr)] = p0 + j * 32;
        gb += __popc(gtm[j]);
        eb += __popc(eqm[j]);
    }
    named_bar_sync<NT>(bar_id);
    return k;
}

}  // namespace sa
