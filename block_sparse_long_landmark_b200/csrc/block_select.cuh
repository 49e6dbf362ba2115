// block_select.cuh -- exact top-k of up to a few thousand order-preserving
// 32-bit score keys by NW warps of one CTA, synchronised on a named barrier
// (other warps of the CTA may have left).
//
// Each thread holds KPT keys in registers; warp w owns the contiguous
// positions [w * 32 * KPT, (w + 1) * 32 * KPT), lane l the positions
// w * 32 * KPT + j * 32 + l.  The result is the top-k by (key desc, position
// asc), positions ascending.
//
// Up to 2 * 32 * NW keys: each thread ranks its keys against all of them
// (keys above, plus equal keys at a lower position) and keeps ranks below k.
// Longer lists:
//   1. A lower bound L of the k-th largest key: warp w takes the
//      ceil(k / NW)-th largest of its lanes' maxima, L is the least of these.
//      Each warp then holds at least ceil(k / NW) keys >= L (the maxima of
//      those lanes), so at least k keys are >= L and the top-k all are.
//   2. The keys >= L -- typically a few per cent of the list -- are gathered
//      in position order (ballots and one prefix over the warps) and ranked
//      among themselves; ranks below k are the result.
//   3. When more than kBsCand keys pass L (heavy ties, or keys that rise
//      along the list), a radix select instead: a histogram of the top 12
//      bits of the keys gives the digit of the k-th largest key T and how
//      many keys lie above it; the keys of that digit, when few, are ranked
//      among themselves for T, else two more passes of 12 and 8 bits give the
//      rest of T.  A compaction in position order then takes every key > T
//      and the first (k - #keys > T) keys equal to T.  Counters are 16 bits,
//      two to a word (n < 65536).
#pragma once

#include "common.cuh"

namespace sa {

constexpr int kBsMaxWarps = 16;
constexpr int kBsBins = 4096;   // widest digit: 12 bits
constexpr int kBsCand = 512;    // keys gathered and ranked directly

struct BsSmem {
    uint32_t hist[2][kBsBins / 2];    // 16-bit counters, bin b in half (b & 1) of word b >> 1
    alignas(16) uint32_t cand[kBsCand];   // gathered keys (position order)
    int cpos[kBsCand];                // their positions
    int misc[2][3];                   // per pass: T's digit, keys above that digit, keys of that digit
    int wcnt[kBsMaxWarps][2];         // per warp: counts for the prefixes
    int wsel[kBsCand / 32 + kBsMaxWarps];   // per rank round and warp: selected candidates
    uint32_t wlow[kBsMaxWarps];       // per warp: its bound
    int ncand;
    uint32_t T;
    int take;
};

template <int NT>
__device__ __forceinline__ void named_bar_sync(int id) {
    asm volatile("bar.sync %0, %1;" ::"r"(id), "n"(NT) : "memory");
}

// The kw-th largest (1 <= kw <= 32) of the 32 lanes' values, bit by bit
// below the bits all lanes share.
__device__ __forceinline__ uint32_t warp_kth_largest(uint32_t v, int kw) {
    const uint32_t hi = __reduce_max_sync(0xffffffffu, v), lo = __reduce_min_sync(0xffffffffu, v);
    const uint32_t diff = hi ^ lo;
    if (diff == 0u) return hi;
    int b = 31 - __clz(diff);
    uint32_t T = b == 31 ? 0u : (hi & ~((2u << b) - 1u));
    for (; b >= 0; --b) {
        const uint32_t c = T | (1u << b);
        if (__popc(__ballot_sync(0xffffffffu, v >= c)) >= kw) T = c;
    }
    return T;
}

// Rank of key x at index c among list[0..m): keys above it plus equal keys at
// a lower index.  list is 16-byte aligned; four keys per shared load.
__device__ __forceinline__ int rank_in(const uint32_t *list, int m, uint32_t x, int c) {
    const uint4 *l4 = reinterpret_cast<const uint4 *>(list);
    int r0 = 0, r1 = 0;
    const int m4 = (reinterpret_cast<uintptr_t>(list) & 15u) ? 0 : m >> 2;
#pragma unroll 4
    for (int i4 = 0; i4 < m4; ++i4) {
        const uint4 y = l4[i4];
        const int i = i4 << 2;
        r0 += (y.x > x) | ((y.x == x) & (i < c));
        r1 += (y.y > x) | ((y.y == x) & (i + 1 < c));
        r0 += (y.z > x) | ((y.z == x) & (i + 2 < c));
        r1 += (y.w > x) | ((y.w == x) & (i + 3 < c));
    }
    for (int i = m4 << 2; i < m; ++i) r0 += (list[i] > x) | ((list[i] == x) & (i < c));
    return r0 + r1;
}

// Positions (ascending) of the top-k keys of keys[0..n) into out[0..k):
// every position when n <= k.  n <= NW * 32 * KPT < 65536, k <= 32 * NW.
// Called by the threads 0 .. NW*32-1 of the CTA together; returns the count
// (uniform).
template <int NW, int KPT>
__device__ int block_topk32(const uint32_t *keys, int n, int k, int *out, BsSmem &bs, int bar_id) {
    static_assert(NW <= kBsMaxWarps && NW * 32 * KPT < 65536, "shape");
    constexpr int NT = NW * 32;
    constexpr int WPT = kBsBins / 2 / NT;      // histogram words per thread in the scan
    static_assert(WPT * NT * 2 == kBsBins, "scan split");
    constexpr int RR = (kBsCand + NT - 1) / NT;   // rank rounds over the gathered keys
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
            if (p < n) sel[h] = rank_in(keys, n, keys[p], p) < k;
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

    // ---- 1. the lower bound L ------------------------------------------------
    {
        uint32_t tmax = 0u;
#pragma unroll
        for (int j = 0; j < KPT; ++j)
            if ((valid >> j) & 1u) tmax = max(tmax, r[j]);
        const uint32_t lw = warp_kth_largest(tmax, (k + NW - 1) / NW);
        if (lane == 0) bs.wlow[warp] = lw;
    }
    named_bar_sync<NT>(bar_id);
    uint32_t L = 0xffffffffu;
#pragma unroll
    for (int w = 0; w < NW; ++w) L = min(L, bs.wlow[w]);

    // ---- 2. the keys >= L, gathered in position order and ranked ------------
    unsigned bal[KPT];
    {
        int W = 0;
#pragma unroll
        for (int j = 0; j < KPT; ++j) {
            bal[j] = __ballot_sync(0xffffffffu, ((valid >> j) & 1u) && r[j] >= L);
            W += __popc(bal[j]);
        }
        if (lane == 0) bs.wcnt[warp][0] = W;
    }
    named_bar_sync<NT>(bar_id);
    int base = 0, m = 0;
#pragma unroll
    for (int w = 0; w < NW; ++w) {
        const int c = bs.wcnt[w][0];
        if (w < warp) base += c;
        m += c;
    }
    if (m <= kBsCand) {
#pragma unroll
        for (int j = 0; j < KPT; ++j) {
            if ((bal[j] >> lane) & 1u) {
                const int at = base + __popc(bal[j] & below);
                bs.cand[at] = r[j];
                bs.cpos[at] = p0 + j * 32;
            }
            base += __popc(bal[j]);
        }
        named_bar_sync<NT>(bar_id);
        unsigned sb[RR];
#pragma unroll
        for (int rr = 0; rr < RR; ++rr) {
            const int c = rr * NT + tid;
            bool sel = false;
            if (rr * NT < m && c < m) sel = rank_in(bs.cand, m, bs.cand[c], c) < k;
            sb[rr] = __ballot_sync(0xffffffffu, sel);
            if (lane == 0) bs.wsel[rr * NW + warp] = __popc(sb[rr]);
        }
        named_bar_sync<NT>(bar_id);
        int ob = 0;
#pragma unroll
        for (int rr = 0; rr < RR; ++rr) {
            int before = 0, tot = 0;
#pragma unroll
            for (int w = 0; w < NW; ++w) {
                const int c = bs.wsel[rr * NW + w];
                if (w < warp) before += c;
                tot += c;
            }
            if ((sb[rr] >> lane) & 1u) out[ob + before + __popc(sb[rr] & below)] = bs.cpos[rr * NT + tid];
            ob += tot;
        }
        named_bar_sync<NT>(bar_id);
        return ob;
    }

    // ---- 3. radix select ----------------------------------------------------
    for (int i = tid; i < kBsBins / 2; i += NT) bs.hist[0][i] = 0u;
    if (tid == 0) bs.ncand = 0;
    named_bar_sync<NT>(bar_id);

    // T's first digit; then T from the keys of that digit, or two more digits
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

    // compaction in position order: keys > T, then the first keys equal to T
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
