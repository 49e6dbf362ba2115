// warp_select.cuh -- exact top-k of up to a few thousand order-preserving
// score keys by one warp, with no block-wide barrier: a 4-pass MSB radix
// select over a per-warp shared-memory histogram (lanes that share a digit add
// once, via __match_any_sync), then an index-ordered compaction in which keys
// equal to the threshold are taken lowest position first -- so equal scores
// go to the lower block index, as the selection rule requires.
#pragma once

#include "common.cuh"

namespace sa {

// Exact top-k (n > k) of keys[0..n) for one warp; T = threshold key,
// take_eq = how many keys equal to T are taken (lowest positions first).
__device__ __forceinline__ void warp_radix_select(const uint32_t *keys, int n, int k, int *hist, uint32_t &T, int &take_eq) {
    const int lane = threadIdx.x & 31;
    uint32_t prefix = 0, mask = 0;
    int remaining = k;
    for (int shift = 24; shift >= 0; shift -= 8) {
        for (int b = lane; b < 256; b += 32) hist[b] = 0;
        __syncwarp();
        for (int i0 = 0; i0 < n; i0 += 32) {
            const int i = i0 + lane;
            const uint32_t x = i < n ? keys[i] : 0u;
            const bool take = i < n && (x & mask) == prefix;
            const unsigned act = __ballot_sync(0xffffffffu, take);
            if (take) {
                const int digit = (int)((x >> shift) & 255);
                const unsigned same = __match_any_sync(act, digit);
                if (lane == __ffs(same) - 1) atomicAdd(&hist[digit], __popc(same));
            }
        }
        __syncwarp();
        const int hi = 255 - 8 * lane;
        int loc = 0;
#pragma unroll
        for (int q = 0; q < 8; ++q) loc += hist[hi - q];
        int incl = loc;
#pragma unroll
        for (int o = 1; o < 32; o <<= 1) {
            const int t = __shfl_up_sync(0xffffffffu, incl, o);
            if (lane >= o) incl += t;
        }
        const int excl = incl - loc;
        int digit = 0, above = 0;
        if (excl < remaining && remaining <= incl) {
            int cum = excl;
            for (int q = 0; q < 8; ++q) {
                const int c = hist[hi - q];
                if (cum + c >= remaining) {
                    digit = hi - q;
                    above = cum;
                    break;
                }
                cum += c;
            }
        }
        const unsigned who = __ballot_sync(0xffffffffu, excl < remaining && remaining <= incl);
        const int src = __ffs(who) - 1;
        digit = __shfl_sync(0xffffffffu, digit, src);
        above = __shfl_sync(0xffffffffu, above, src);
        remaining -= above;
        prefix |= (uint32_t)digit << shift;
        mask |= 255u << shift;
        __syncwarp();
    }
    T = prefix;
    take_eq = remaining;
}

// Warp exclusive prefix sum.
__device__ __forceinline__ int warp_excl(int v, int &total) {
    const int lane = threadIdx.x & 31;
    int incl = v;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
        const int t = __shfl_up_sync(0xffffffffu, incl, o);
        if (lane >= o) incl += t;
    }
    total = __shfl_sync(0xffffffffu, incl, 31);
    return incl - v;
}

// Positions (ascending) of the top-k keys of keys[0..n) into out[0..):
// every position when n <= k.  Returns how many (warp-uniform).  `hist`
// holds 256 ints of this warp's own.
__device__ __forceinline__ int warp_topk_positions(const uint32_t *keys, int n, int k, int *hist, int *out) {
    const int lane = threadIdx.x & 31;
    if (k <= 0 || n <= 0) return 0;
    if (n <= k) {
        for (int i = lane; i < n; i += 32) out[i] = i;
        __syncwarp();
        return n;
    }
    uint32_t Tk;
    int take_eq;
    warp_radix_select(keys, n, k, hist, Tk, take_eq);
    const int seg = (n + 31) / 32;
    const int i0 = min(n, lane * seg), i1 = min(n, i0 + seg);
    int neq = 0;
    for (int i = i0; i < i1; ++i) neq += keys[i] == Tk;
    int tot;
    const int eq_base = warp_excl(neq, tot);
    int cntsel = 0;
    {
        int e = eq_base;
        for (int i = i0; i < i1; ++i) {
            const uint32_t x = keys[i];
            cntsel += x > Tk || (x == Tk && e < take_eq);
            e += x == Tk;
        }
    }
    int nsel;
    int pos = warp_excl(cntsel, nsel);
    {
        int e = eq_base;
        for (int i = i0; i < i1; ++i) {
            const uint32_t x = keys[i];
            if (x > Tk || (x == Tk && e < take_eq)) out[pos++] = i;
            e += x == Tk;
        }
    }
    __syncwarp();
    return nsel;
}

}  // namespace sa
