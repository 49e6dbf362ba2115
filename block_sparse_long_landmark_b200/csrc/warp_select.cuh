// warp_select.cuh -- exact top-k of up to a few thousand order-preserving
// score keys by one warp, with no block-wide barrier and no shared-memory
// atomics.
//
//   1. The k-th largest key T is found bit by bit, most significant first:
//      T keeps a candidate bit when at least k keys are >= T with that bit
//      set.  Bits above the highest bit in which the warp's largest and
//      smallest keys differ are common to all keys and are taken as they are.
//      Each step is one compare per key and one warp reduction.
//   2. A compaction in position order takes every key > T and the first
//      (k - #keys > T) keys equal to T, so equal scores go to the lower block
//      index, as the selection rule requires; positions come out ascending.
// Lists of up to 32 * REG_SLOTS keys are held in registers (REG_SLOTS per
// lane), longer ones are read from shared memory at every step; REG_SLOTS = 0
// keeps every list in shared memory (for kernels short of registers).
#pragma once

#include "common.cuh"

namespace sa {

// Count of keys >= c over the warp.
template <int SLOTS>
__device__ __forceinline__ int warp_count_ge_reg(const uint32_t (&r)[SLOTS], uint32_t c) {
    int n = 0;
#pragma unroll
    for (int j = 0; j < SLOTS; ++j) n += r[j] >= c;
    return __reduce_add_sync(0xffffffffu, n);
}
__device__ __forceinline__ int warp_count_ge_smem(const uint32_t *keys, int n, uint32_t c) {
    const int lane = threadIdx.x & 31;
    int m = 0;
    for (int i = lane; i < n; i += 32) m += keys[i] >= c;
    return __reduce_add_sync(0xffffffffu, m);
}

// Positions (ascending) of the top-k keys of keys[0..n) into out[0..):
// every position when n <= k.  Returns how many (warp-uniform).
template <int REG_SLOTS = 16>
__device__ __forceinline__ int warp_topk_positions(const uint32_t *keys, int n, int k, int *out) {
    constexpr int kSlots = REG_SLOTS > 0 ? REG_SLOTS : 1;
    const int lane = threadIdx.x & 31;
    if (k <= 0 || n <= 0) return 0;
    if (n <= k) {
        for (int i = lane; i < n; i += 32) out[i] = i;
        __syncwarp();
        return n;
    }
    // ---- 1. threshold T = the k-th largest key ----------------------------
    const bool in_regs = REG_SLOTS > 0 && n <= 32 * REG_SLOTS;
    uint32_t r[kSlots];
    uint32_t kmax = 0u, kmin = 0xffffffffu;
    if (in_regs) {
#pragma unroll
        for (int j = 0; j < kSlots; ++j) {
            const int i = j * 32 + lane;
            r[j] = i < n ? keys[i] : 0u;   // padding 0: below every candidate, never counted
            if (i < n) {
                kmax = max(kmax, r[j]);
                kmin = min(kmin, r[j]);
            }
        }
    } else {
        for (int i = lane; i < n; i += 32) {
            const uint32_t x = keys[i];
            kmax = max(kmax, x);
            kmin = min(kmin, x);
        }
    }
    kmax = __reduce_max_sync(0xffffffffu, kmax);
    kmin = __reduce_min_sync(0xffffffffu, kmin);
    const uint32_t diff = kmax ^ kmin;
    const int top = diff ? 31 - __clz(diff) : -1;           // highest differing bit
    const uint32_t low = top >= 0 ? (0xffffffffu >> (31 - top)) : 0u;
    uint32_t T = kmax & ~low;                                // common prefix: every key is >= T
    for (int b = top; b >= 0; --b) {
        const uint32_t c = T | (1u << b);
        const int ge = in_regs ? warp_count_ge_reg(r, c) : warp_count_ge_smem(keys, n, c);
        if (ge >= k) T = c;
    }
    int gt = 0;
    if (in_regs) {
#pragma unroll
        for (int j = 0; j < kSlots; ++j) gt += r[j] > T;
    } else {
        for (int i = lane; i < n; i += 32) gt += keys[i] > T;
    }
    gt = __reduce_add_sync(0xffffffffu, gt);
    const int take_eq = k - gt;
    // ---- 2. compaction in position order -----------------------------------
    const unsigned below = (1u << lane) - 1u;
    int base = 0, eq_before = 0;
    for (int i0 = 0; i0 < n; i0 += 32) {
        const int i = i0 + lane;
        const uint32_t x = i < n ? keys[i] : 0u;
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

}  // namespace sa
