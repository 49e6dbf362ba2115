// lsa_dev.cuh -- device helpers shared by the flat (lsa.cu) and the tree
// (lsa_tree.cu) decode through the clustered index: 64-bit block top-K, the
// expansion of chosen clusters into the flat list of kept key positions.
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

// Positions (ascending) of the top-k of keys[0..n) in shared memory, equal
// keys to the lower position, by the whole block (every thread calls it);
// every position when n <= k.  The k-th largest key T is found a byte at a
// time, most significant first: a 256-bin histogram of the keys that match
// the bytes found so far gives the byte of T and how many keys lie above it.
// An index-ordered compaction then takes every key > T and the first keys
// equal to T.  `hist` holds 256 + 8 ints, `red` the block scan's 8.
// Returns the count (block-uniform).
__device__ inline int block_topk64(const uint64_t *keys, int n, int k, int *out, int *hist, int *red) {
    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    if (k <= 0 || n <= 0) return 0;
    if (n <= k) {
        for (int i = tid; i < n; i += kLsaThreads) out[i] = i;
        __syncthreads();
        return n;
    }
    if (n <= kLsaThreads) {
        // a key per thread, ranked by the keys above it (equal keys: the lower
        // position first); the k lowest ranks, compacted in position order
        int sel = 0;
        if (tid < n) {
            const unsigned long long x = keys[tid];
            int r = 0;
            for (int j = 0; j < n; ++j) {
                const unsigned long long y = keys[j];
                r += (y > x) || (y == x && j < tid);
            }
            sel = r < k;
        }
        int tot;
        const int at = block_scan_incl(sel, red, &tot) - sel;
        if (sel) out[at] = tid;
        __syncthreads();
        return tot;
    }
    int *misc = hist + 256;
    unsigned long long prefix = 0ull, mask = 0ull;
    int kr = k;                                    // rank of T among the keys matching `prefix`
    for (int shift = 56; shift >= 0; shift -= 8) {
        for (int i = tid; i < 256; i += kLsaThreads) hist[i] = 0;
        __syncthreads();
        for (int i = tid; i < n; i += kLsaThreads) {
            const unsigned long long x = keys[i];
            if ((x & mask) == prefix) atomicAdd(&hist[(x >> shift) & 255], 1);
        }
        __syncthreads();
        if (warp == 0) {
            // lane l holds digits 255 - 8 l .. 248 - 8 l (descending); counts above each
            int c[8], sum = 0;
#pragma unroll
            for (int j = 0; j < 8; ++j) {
                c[j] = hist[255 - 8 * lane - j];
                sum += c[j];
            }
            int incl = sum;
#pragma unroll
            for (int o = 1; o < 32; o <<= 1) {
                const int t = __shfl_up_sync(0xffffffffu, incl, o);
                if (lane >= o) incl += t;
            }
            const int excl = incl - sum;
            int found = -1, above = 0;
            if (excl < kr && incl >= kr) {
                int run = excl;
#pragma unroll
                for (int j = 0; j < 8; ++j) {
                    if (found < 0 && run + c[j] >= kr) {
                        found = 255 - 8 * lane - j;
                        above = run;
                    }
                    run += c[j];
                }
            }
            if (found >= 0) {
                misc[0] = found;
                misc[1] = above;
            }
        }
        __syncthreads();
        prefix |= (unsigned long long)misc[0] << shift;
        mask |= 255ull << shift;
        kr -= misc[1];
        __syncthreads();
    }
    // compaction in index order: keys > T, then the first kr keys equal to T
    const unsigned long long T = prefix;
    int base = 0, eq_before = 0;
    for (int i0 = 0; i0 < n; i0 += kLsaThreads) {
        const int i = i0 + tid;
        const unsigned long long x = i < n ? keys[i] : 0ull;
        const int eq = (i < n && x == T) ? 1 : 0;
        int eq_tot;
        const int eq_ex = block_scan_incl(eq, red, &eq_tot) - eq;
        const int sel = (i < n && (x > T || (eq && eq_before + eq_ex < kr))) ? 1 : 0;
        int sel_tot;
        const int at = block_scan_incl(sel, red, &sel_tot) - sel;
        if (sel) out[base + at] = i;
        base += sel_tot;
        eq_before += eq_tot;
    }
    __syncthreads();
    return base;
}

// Kept key positions of one (batch, kv-head) from the chosen clusters (ids
// ascending in chosen[0..ntop)), written in order to the flat position list:
// the first `sink` positions, every item of every chosen cluster (pool keys
// each) minus what the sink or the window already hold, and the last `window`
// positions (up to the query at N - 1).  `off` holds ntop + 1 ints, `red`
// the block scan's 8; all threads call it.
__device__ inline void expand_positions(const LsaDecArgs &a, int bg, const int *chosen, int ntop, int *off, int *red) {
    const LsaShape &s = a.s;
    const int tid = threadIdx.x;
    const int sink_n = min(s.sink, s.N);
    const int win0 = max(sink_n, s.N - s.window);      // window = [win0, N)
    int32_t *pos = a.pos + (size_t)bg * a.pl.pmax;
    // items of the chosen clusters: exclusive prefix of their sizes
    int items = 0;
    for (int r0 = 0; r0 < ntop; r0 += kLsaThreads) {
        const int r = r0 + tid;
        const int sz = r < ntop ? min(max(a.sizes[(size_t)bg * s.ctotal + chosen[r]], 0), s.seg) : 0;
        int tot;
        const int incl = block_scan_incl(sz, red, &tot);
        if (r < ntop) off[r] = items + incl - sz;
        items += tot;
    }
    if (tid == 0) off[ntop] = items;
    for (int i = tid; i < sink_n && i < a.pl.pmax; i += kLsaThreads) pos[i] = i;
    __syncthreads();
    // every item: its keys outside the sink and the window, after the sink
    int carry = sink_n;
    for (int e0 = 0; e0 < items; e0 += kLsaThreads) {
        const int e = e0 + tid;
        int lo = 0, len = 0;
        if (e < items) {
            int l = 0, h = ntop - 1;                       // the cluster holding item e
            while (l < h) {
                const int mid = (l + h + 1) >> 1;
                if (off[mid] <= e) l = mid; else h = mid - 1;
            }
            const size_t cid = (size_t)bg * s.ctotal + chosen[l];
            const int item = a.members[cid * s.seg + (e - off[l])];
            if (item < 0 || (long long)(item + 1) * s.pool > (long long)s.nseg * s.seg * s.pool) {
                set_status(a.status, kStatusBadIndex);   // not an item this index holds: skipped
            } else {
                lo = max(item * s.pool, sink_n);
                len = max(0, min((item + 1) * s.pool, win0) - lo);
            }
        }
        int tot;
        const int at = carry + block_scan_incl(len, red, &tot) - len;
        for (int k = 0; k < len && at + k < a.pl.pmax; ++k) pos[at + k] = lo + k;
        carry += tot;
    }
    for (int i = tid; i < s.N - win0 && carry + i < a.pl.pmax; i += kLsaThreads) pos[carry + i] = win0 + i;
    if (tid == 0) {
        const int total = min(carry + max(0, s.N - win0), a.pl.pmax);
        a.cnt[2 * (size_t)bg] = total;
        a.cnt[2 * (size_t)bg + 1] = total;
        if (a.kept) a.kept[bg] = total;
    }
}

}  // namespace sa
