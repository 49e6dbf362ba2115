// lsa_dev.cuh -- device helpers shared by the flat (lsa.cu) and the tree
// (lsa_tree.cu) decode through the clustered index: 64-bit top-K, the
// expansion of chosen clusters into key ranges.
#pragma once

#include "common.cuh"
#include "lsa.cuh"

namespace sa {

constexpr int kLsaThreads = 256;

// fp64 -> uint64 key whose unsigned order is the double order (NaN -> 0,
// below every number).
__device__ __forceinline__ uint64_t ord_key64(double x) {
    const uint64_t u = (uint64_t)__double_as_longlong(x);
    if ((u & 0x7fffffffffffffffull) > 0x7ff0000000000000ull) return 0ull;
    return (u & 0x8000000000000000ull) ? ~u : (u | 0x8000000000000000ull);
}

// Positions (ascending) of the top-k of keys[0..n) (shared or global
// memory), equal keys to the lower position, by one warp (every lane calls
// it); every position when n <= k.  The k-th largest key T is found bit by
// bit below the bits the largest and smallest keys share, then an
// index-ordered ballot compaction takes every key > T and the first keys
// equal to T.  Returns the count (warp-uniform).
__device__ inline int warp_topk64(const uint64_t *keys, int n, int k, int *out) {
    const int lane = threadIdx.x & 31;
    if (k <= 0 || n <= 0) return 0;
    if (n <= k) {
        for (int i = lane; i < n; i += 32) out[i] = i;
        __syncwarp();
        return n;
    }
    unsigned long long mx = 0ull, mn = ~0ull;
    for (int i = lane; i < n; i += 32) {
        mx = max(mx, (unsigned long long)keys[i]);
        mn = min(mn, (unsigned long long)keys[i]);
    }
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) {
        mx = max(mx, __shfl_xor_sync(0xffffffffu, mx, o));
        mn = min(mn, __shfl_xor_sync(0xffffffffu, mn, o));
    }
    const unsigned long long diff = mx ^ mn;
    const int top = diff ? 63 - __clzll((long long)diff) : -1;
    const unsigned long long low = top >= 0 ? (~0ull >> (63 - top)) : 0ull;
    unsigned long long T = mx & ~low;
    for (int bit = top; bit >= 0; --bit) {
        const unsigned long long c = T | (1ull << bit);
        int ge = 0;
        for (int i = lane; i < n; i += 32) ge += keys[i] >= c;
        if (__reduce_add_sync(0xffffffffu, ge) >= k) T = c;
    }
    int gt = 0;
    for (int i = lane; i < n; i += 32) gt += keys[i] > T;
    const int take_eq = k - __reduce_add_sync(0xffffffffu, gt);
    const unsigned below = (1u << lane) - 1u;
    int base = 0, eq_before = 0;
    for (int i0 = 0; i0 < n; i0 += 32) {
        const int i = i0 + lane;
        const unsigned long long x = i < n ? keys[i] : 0ull;
        const bool eq = i < n && x == T;
        const unsigned eqm = __ballot_sync(0xffffffffu, eq);
        const bool sel = i < n && (x > T || (eq && eq_before + __popc(eqm & below) < take_eq));
        const unsigned selm = __ballot_sync(0xffffffffu, sel);
        if (sel) out[base + __popc(selm & below)] = i;
        base += __popc(selm);
        eq_before += __popc(eqm);
    }
    __syncwarp();
    return base;
}

// Kept key ranges of one (batch, kv-head) from the chosen clusters (ids
// ascending in chosen[0..ntop)): the first `sink` positions, every item of
// every chosen cluster (pool keys each) minus what the sink or the window
// already hold, and the last `window` positions (up to the query at N - 1).
// Writes the ranges and their exclusive length prefix; all threads call it.
__device__ inline void expand_ranges(const LsaDecArgs &a, int bg, const int *chosen, int ntop, int *red) {
    const LsaShape &s = a.s;
    const int tid = threadIdx.x;
    const int sink_n = min(s.sink, s.N);
    const int win0 = max(sink_n, s.N - s.window);      // window = [win0, N)
    int32_t *rs = a.rs + (size_t)bg * a.pl.rmax, *rl = a.rl + (size_t)bg * a.pl.rmax, *rp = a.rp + (size_t)bg * a.pl.rmax;
    int nr = 0;
    if (sink_n > 0) {
        if (tid == 0) {
            rs[0] = 0;
            rl[0] = sink_n;
        }
        nr = 1;
    }
    const int total_items = ntop * s.seg;
    for (int e0 = 0; e0 < total_items; e0 += kLsaThreads) {
        const int e = e0 + tid;
        int lo = 0, hi = 0;
        bool ok = false;
        if (e < total_items) {
            const int r = e / s.seg, m = e % s.seg;
            const size_t cid = (size_t)bg * s.ctotal + chosen[r];
            const int sz = min(max(a.sizes[cid], 0), s.seg);
            if (m < sz) {
                const int item = a.members[cid * s.seg + m];
                if (item < 0 || (long long)(item + 1) * s.pool > (long long)s.nseg * s.seg * s.pool) {
                    set_status(a.status, kStatusBadIndex);   // not an item this index holds: skipped
                } else {
                    lo = max(item * s.pool, sink_n);
                    hi = min((item + 1) * s.pool, win0);
                    ok = lo < hi;
                }
            }
        }
        int tot;
        const int at = block_scan_incl(ok ? 1 : 0, red, &tot) - (ok ? 1 : 0);
        if (ok) {
            rs[nr + at] = lo;
            rl[nr + at] = hi - lo;
        }
        nr += tot;
    }
    if (win0 < s.N) {
        if (tid == 0) {
            rs[nr] = win0;
            rl[nr] = s.N - win0;
        }
        nr += 1;
    }
    __syncthreads();
    // exclusive prefix of the lengths
    int carry = 0;
    for (int e0 = 0; e0 < nr; e0 += kLsaThreads) {
        const int e = e0 + tid;
        const int len = e < nr ? rl[e] : 0;
        int tot;
        const int incl = block_scan_incl(len, red, &tot);
        if (e < nr) rp[e] = carry + incl - len;
        carry += tot;
    }
    if (tid == 0) {
        a.cnt[2 * (size_t)bg] = nr;
        a.cnt[2 * (size_t)bg + 1] = carry;
        if (a.kept) a.kept[bg] = carry;
    }
}

}  // namespace sa
