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
//   1. The k-th largest key T is found a byte at a time, most significant
//      first: a 256-bin histogram of the keys that match the bytes found so
//      far gives the next byte of T and how many keys lie above it.  Two
//      histograms alternate, so a pass needs two barriers.
//   2. A compaction in position order takes every key > T and the first
//      (k - #keys > T) keys equal to T, so equal scores go to the lower
//      position, as the selection rule requires; positions come out
//      ascending.  Each warp counts its segment with ballots, one barrier
//      publishes the warps' counts, and each key's output slot is
//      (#keys > T before it) + min(#keys == T before it, k - #keys > T).
#pragma once

#include "common.cuh"

namespace sa {

constexpr int kBsMaxWarps = 16;

struct BsSmem {
    int hist[2][256];
    int misc[2][2];            // per pass: T's byte, keys above that byte
    int wcnt[kBsMaxWarps][2];  // per warp: keys > T, keys == T
};

template <int NT>
__device__ __forceinline__ void named_bar_sync(int id) {
    asm volatile("bar.sync %0, %1;" ::"r"(id), "n"(NT) : "memory");
}

// Positions (ascending) of the top-k keys of keys[0..n) into out[0..k):
// every position when n <= k.  n <= NW * 32 * KPT.  Called by the threads
// 0 .. NW*32-1 of the CTA together; returns the count (uniform).
template <int NW, int KPT>
__device__ int block_topk32(const uint32_t *keys, int n, int k, int *out, BsSmem &bs, int bar_id) {
    static_assert(NW <= kBsMaxWarps, "warps");
    constexpr int NT = NW * 32;
    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    if (k <= 0 || n <= 0) return 0;
    if (n <= k) {
        for (int i = tid; i < n; i += NT) out[i] = i;
        named_bar_sync<NT>(bar_id);
        return n;
    }
    const int p0 = warp * 32 * KPT + lane;
    uint32_t r[KPT];
#pragma unroll
    for (int j = 0; j < KPT; ++j) r[j] = p0 + j * 32 < n ? keys[p0 + j * 32] : 0u;
    for (int i = tid; i < 256; i += NT) bs.hist[0][i] = 0;
    named_bar_sync<NT>(bar_id);

    // ---- 1. T = the k-th largest key, a byte per pass ----------------------
    uint32_t prefix = 0u, mask = 0u;
    int kr = k;   // rank of T among the keys that match `prefix`
#pragma unroll 1
    for (int pass = 0; pass < 4; ++pass) {
        const int shift = 24 - 8 * pass, cur = pass & 1;
#pragma unroll
        for (int j = 0; j < KPT; ++j)
            if ((r[j] & mask) == prefix) atomicAdd(&bs.hist[cur][(r[j] >> shift) & 255u], 1);
        for (int i = tid; i < 256; i += NT) bs.hist[cur ^ 1][i] = 0;
        named_bar_sync<NT>(bar_id);
        if (warp == 0) {
            // lane l holds bytes 255 - 8 l .. 248 - 8 l (descending)
            int c[8], sum = 0;
#pragma unroll
            for (int j = 0; j < 8; ++j) {
                c[j] = bs.hist[cur][255 - 8 * lane - j];
                sum += c[j];
            }
            int incl = sum;
#pragma unroll
            for (int o = 1; o < 32; o <<= 1) {
                const int t = __shfl_up_sync(0xffffffffu, incl, o);
                if (lane >= o) incl += t;
            }
            const int excl = incl - sum;
            if (excl < kr && incl >= kr) {
                int run = excl, found = 0, above = 0;
                bool done = false;
#pragma unroll
                for (int j = 0; j < 8; ++j) {
                    if (!done && run + c[j] >= kr) {
                        found = 255 - 8 * lane - j;
                        above = run;
                        done = true;
                    }
                    run += c[j];
                }
                bs.misc[cur][0] = found;
                bs.misc[cur][1] = above;
            }
        }
        named_bar_sync<NT>(bar_id);
        prefix |= (uint32_t)bs.misc[cur][0] << shift;
        mask |= 255u << shift;
        kr -= bs.misc[cur][1];
    }
    const uint32_t T = prefix;

    // ---- 2. compaction in position order -----------------------------------
    const unsigned below = (1u << lane) - 1u;
    unsigned gtm[KPT], eqm[KPT];
    int G = 0, E = 0;
#pragma unroll
    for (int j = 0; j < KPT; ++j) {
        const bool valid = p0 + j * 32 < n;
        gtm[j] = __ballot_sync(0xffffffffu, valid && r[j] > T);
        eqm[j] = __ballot_sync(0xffffffffu, valid && r[j] == T);
        G += __popc(gtm[j]);
        E += __popc(eqm[j]);
    }
    if (lane == 0) {
        bs.wcnt[warp][0] = G;
        bs.wcnt[warp][1] = E;
    }
    named_bar_sync<NT>(bar_id);
    int gb = 0, eb = 0;
    for (int w = 0; w < warp; ++w) {
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
