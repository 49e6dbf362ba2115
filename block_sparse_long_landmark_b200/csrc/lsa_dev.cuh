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

// Sum of v over the CTA (kLsaThreads threads); `red` holds 8 ints.
__device__ __forceinline__ int block_sum(int v, int *red) {
    v = __reduce_add_sync(0xffffffffu, v);
    __syncthreads();
    if ((threadIdx.x & 31) == 0) red[threadIdx.x >> 5] = v;
    __syncthreads();
    int t = 0;
#pragma unroll
    for (int w = 0; w < kLsaThreads / 32; ++w) t += red[w];
    __syncthreads();                                // red is free again on return
    return t;
}

// Positions (ascending) of the top-k of keys[0..n) in shared memory, equal
// keys to the lower position, written to out[0..); every position when
// n <= k.  Exact: the k-th largest key T is found bit by bit from the top
// (bits shared by the largest and smallest key are taken as they are), then
// a position-ordered compaction takes every key > T and the first keys == T.
// All threads of the CTA call it; returns the count.
__device__ inline int block_topk64(const uint64_t *keys, int n, int k, int *out, int *red, uint64_t *red64) {
    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    if (k <= 0 || n <= 0) return 0;
    if (n <= k) {
        for (int i = tid; i < n; i += kLsaThreads) out[i] = i;
        __syncthreads();
        return n;
    }
    uint64_t mx = 0ull, mn = ~0ull;
    for (int i = tid; i < n; i += kLsaThreads) {
        mx = max(mx, keys[i]);
        mn = min(mn, keys[i]);
    }
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) {
        mx = max(mx, (uint64_t)__shfl_xor_sync(0xffffffffu, (unsigned long long)mx, o));
        mn = min(mn, (uint64_t)__shfl_xor_sync(0xffffffffu, (unsigned long long)mn, o));
    }
    __syncthreads();
    if (lane == 0) {
        red64[warp] = mx;
        red64[8 + warp] = mn;
    }
    __syncthreads();
    mx = 0ull;
    mn = ~0ull;
#pragma unroll
    for (int w = 0; w < kLsaThreads / 32; ++w) {
        mx = max(mx, red64[w]);
        mn = min(mn, red64[8 + w]);
    }
    const uint64_t diff = mx ^ mn;
    const int top = diff ? 63 - __clzll((long long)diff) : -1;
    const uint64_t low = top >= 0 ? (~0ull >> (63 - top)) : 0ull;
    uint64_t T = mx & ~low;                        // every key >= T
    for (int bit = top; bit >= 0; --bit) {
        const uint64_t c = T | (1ull << bit);
        int ge = 0;
        for (int i = tid; i < n; i += kLsaThreads) ge += keys[i] >= c;
        if (block_sum(ge, red) >= k) T = c;
    }
    int gt = 0;
    for (int i = tid; i < n; i += kLsaThreads) gt += keys[i] > T;
    const int take_eq = k - block_sum(gt, red);
    // compaction in position order: thread t owns positions [i0, i1)
    const int seg = (n + kLsaThreads - 1) / kLsaThreads;
    const int i0 = min(n, tid * seg), i1 = min(n, i0 + seg);
    int neq = 0;
    for (int i = i0; i < i1; ++i) neq += keys[i] == T;
    const int eq_base = block_scan_incl(neq, red, nullptr) - neq;
    int nsel = 0;
    {
        int e = eq_base;
        for (int i = i0; i < i1; ++i) {
            const bool take = keys[i] > T || (keys[i] == T && e < take_eq);
            e += keys[i] == T;
            nsel += take;
        }
    }
    int total;
    int pos = block_scan_incl(nsel, red, &total) - nsel;
    {
        int e = eq_base;
        for (int i = i0; i < i1; ++i) {
            const bool take = keys[i] > T || (keys[i] == T && e < take_eq);
            e += keys[i] == T;
            if (take) out[pos++] = i;
        }
    }
    __syncthreads();
    return total;
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
