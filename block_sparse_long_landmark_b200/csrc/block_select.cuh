// block_select.cuh -- exact top-k of up to a few thousand order-preserving
// 32-bit score keys by NW warps of one CTA, synchronised on a named barrier
// (other warps of the CTA may have left).
//
// Each thread holds kpt <= KPT keys in registers; warp w owns the contiguous
// positions [w * 32 * kpt, (w + 1) * 32 * kpt), lane l the positions
// w * 32 * kpt + j * 32 + l.  The result is the top-k by (key desc,
// position asc), positions ascending.
//
// Up to 16 * NW keys: each thread ranks its key against all of them (keys
// above, plus equal keys at a lower position) and keeps ranks below k.
// Longer lists (the bound below is tight when every warp holds keys: the
// caller picks kpt so that the list spreads over all of them):
//   1. A lower bound L of the k-th largest key: warp w takes the
//      ceil(k / NW)-th largest of its lanes' maxima (each lane ranks its
//      maximum against the warp's), L is the least of these.
//      Each warp then holds at least ceil(k / NW) keys >= L (the maxima of
//      those lanes), so at least k keys are >= L and the top-k all are.
//   2. The keys >= L -- typically a few per cent of the list -- are gathered
//      in position order (ballots and one prefix over the warps) and ranked
//      among themselves (up to four threads per key, each over a slice);
//      ranks below k are the result.
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

// The kw-th largest (1 <= kw <= 32) of the 32 lanes' values: each lane ranks
// its value against every lane's (32 independent shuffles; equal values in
// lane order), and the lane of rank kw - 1 holds the answer.
__device__ __forceinline__ uint32_t warp_kth_largest(uint32_t v, int kw) {
    const int lane = threadIdx.x & 31;
    int rk = 0;
#pragma unroll
    for (int j = 0; j < 32; ++j) {
        const uint32_t x = __shfl_sync(0xffffffffu, v, j);
        rk += (x > v) | ((x == v) & (j < lane));
    }
    const unsigned at = __ballot_sync(0xffffffffu, rk == kw - 1);
    return __shfl_sync(0xffffffffu, v, __ffs(at) - 1);
}

// Rank of key x at index c counted over list[lo..hi): keys above it plus
// equal keys at a lower index.  lo a multiple of 4; four keys per shared
// load when list is 16-byte aligned.
__device__ __forceinline__ int rank_range(const uint32_t *list, int lo, int hi, uint32_t x, int c) {
    const uint4 *l4 = reinterpret_cast<const uint4 *>(list);
    int r0 = 0, r1 = 0;
    const int e4 = (reinterpret_cast<uintptr_t>(list) & 15u) ? lo >> 2 : hi >> 2;
#pragma unroll 4
    for (int i4 = lo >> 2; i4 < e4; ++i4) {
        const uint4 y = l4[i4];
        const int i = i4 << 2;
        r0 += (y.x > x) | ((y.x == x) & (i < c));
        r1 += (y.y > x) | ((y.y == x) & (i + 1 < c));
        r0 += (y.z > x) | ((y.z == x) & (i + 2 < c));
        r1 += (y.w > x) | ((y.w == x) & (i + 3 < c));
    }
    for (int i = max(lo, e4 << 2); i < hi; ++i) r0 += (list[i] > x) | ((list[i] == x) & (i < c));
    return r0 + r1;
}
__device__ __forceinline__ int rank_in(const uint32_t *list, int m, uint32_t x, int c) {
    return rank_range(list, 0, m, x, c);
}

// Result of block_select_core: either the keys >= a lower bound of the k-th
// largest key, gathered in position order into bs.cand (keys) and bs.cpos
// (positions), or -- when too many pass the bound, or the list is short --
// the exact top-k positions (ascending) in `out`.  Either way at least k keys
// (counting the whole list) are >= bound when the list has k keys (bound 0
// makes no claim), and the keys handed back hold the top-k.
struct BsResult {
    int n;            // keys gathered, or positions in out
    bool gathered;
    uint32_t bound;
};

// Ranks the m gathered keys cand[0..m) (16-byte aligned, in position order)
// by (key desc, index asc) and writes the indices of the top k, ascending,
// to out.  Returns the count (uniform).
template <int NW>
__device__ int block_rank_gathered(const uint32_t *cand, int m, int k, int *out, BsSmem &bs, int bar_id) {
    constexpr int NT = NW * 32;
    constexpr int RR = (kBsCand + NT - 1) / NT;   // rank rounds over the gathered keys
    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    const unsigned below = (1u << lane) - 1u;
    // tpc adjacent threads rank one candidate, each over a slice of the list
    const int tpc = m <= NT / 4 ? 4 : (m <= NT / 2 ? 2 : 1);
    const int per = ((m + tpc - 1) / tpc + 3) & ~3;
    unsigned sb[RR];
#pragma unroll
    for (int rr = 0; rr < RR; ++rr) {
        const int t = rr * NT + tid, c = t / tpc, part = t % tpc;
        int rk = 0;
        if (c < m) {
            const int lo = part * per, hi = min(m, lo + per);
            if (lo < hi) rk = rank_range(cand, lo, hi, cand[c], c);
        }
        for (int o = 1; o < tpc; o <<= 1) rk += __shfl_xor_sync(0xffffffffu, rk, o);
        sb[rr] = __ballot_sync(0xffffffffu, part == 0 && c < m && rk < k);
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
        if ((sb[rr] >> lane) & 1u) out[ob + before + __popc(sb[rr] & below)] = (rr * NT + tid) / tpc;
        ob += tot;
    }
    named_bar_sync<NT>(bar_id);
    return ob;
}

// Steps 1 and 2 (gather only) or the short-list / radix paths; n <= NW * 32 *
// kpt, kpt <= KPT, NW * 32 * KPT < 65536, k <= 32 * NW, keys 16-byte aligned
// for the wide loads of the short-list ranking.
template <int NW, int KPT>
__device__ BsResult block_select_core(const uint32_t *keys, int n, int k, int *out, BsSmem &bs, int bar_id,
                                      int kpt) {
    static_assert(NW <= kBsMaxWarps && NW * 32 * KPT < 65536, "shape");
    constexpr int NT = NW * 32;
    constexpr int WPT = kBsBins / 2 / NT;      // histogram words per thread in the scan
    static_assert(WPT * NT * 2 == kBsBins, "scan split");
    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    if (k <= 0 || n <= 0) return BsResult{0, false, 0u};
    if (n <= k) {
        for (int i = tid; i < n; i += NT) out[i] = i;
        named_bar_sync<NT>(bar_id);
        return BsResult{n, false, 0u};
    }
    const unsigned below = (1u << lane) - 1u;
    if (n <= NT / 2) {
        // rank every key: keys above it, plus equal keys at a lower position
        const bool sel = tid < n && rank_in(keys, n, keys[tid], tid) < k;
        const unsigned m0 = __ballot_sync(0xffffffffu, sel);
        if (lane == 0) bs.wcnt[warp][0] = __popc(m0);
        named_bar_sync<NT>(bar_id);
        int b0 = 0;
#pragma unroll
        for (int w = 0; w < NW; ++w)
            if (w < warp) b0 += bs.wcnt[w][0];
        if (sel) out[b0 + __popc(m0 & below)] = tid;
        named_bar_sync<NT>(bar_id);
        return BsResult{k, false, 0u};
    }
    const int p0 = warp * 32 * kpt + lane;
    uint32_t r[KPT];
    unsigned valid = 0u;
#pragma unroll
    for (int j = 0; j < KPT; ++j) {
        const bool v = j < kpt && p0 + j * 32 < n;
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

    // ---- 2. the keys >= L, gathered in position order -----------------------
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
        return BsResult{m, true, L};
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
    return BsResult{k, false, T};
}

// Positions (ascending) of the top-k keys of keys[0..n) into out[0..k):
// every position when n <= k.  Shapes as block_select_core.  Returns the
// count (uniform).
template <int NW, int KPT>
__device__ int block_topk32(const uint32_t *keys, int n, int k, int *out, BsSmem &bs, int bar_id, int kpt) {
    const BsResult r = block_select_core<NW, KPT>(keys, n, k, out, bs, bar_id, kpt);
    if (!r.gathered) return r.n;
    const int nc = block_rank_gathered<NW>(bs.cand, r.n, k, out, bs, bar_id);
    for (int i = threadIdx.x; i < nc; i += NW * 32) out[i] = bs.cpos[out[i]];
    named_bar_sync<NW * 32>(bar_id);
    return nc;
}

}  // namespace sa
