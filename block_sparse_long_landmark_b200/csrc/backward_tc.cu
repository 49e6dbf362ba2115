// backward_tc.cu -- backward of the gated block-sparse prefill on the tensor
// cores (bf16, d = 128, block 64 or 128, query groups of 128-row tiles).
//
// [SAS] "Как это применить": the selector's score enters the attention as
// the gate log_sigmoid(s_b - s_local) inside the softmax, which is how the
// loss reaches the selector; "Ключевые факты": the top-K choice is hard, so
// the forward's kept lists are reused as they are.  With P = exp(z - LSE),
// D_i = <dO_i, O_i> and dS = P (dO V^T - D):
//
//   dQ = scale dS K,   dK = scale dS^T Q,   dV = P^T dO,
//   dg_c = sum of dS over the unit's rows and the keys of list entry c.
//
// Three kernels, no atomics, every sum in a fixed order:
//   * bwd_rowprep_kernel: D = rowsum(dO * O) and LSE in log2 units, per row;
//   * bwd_dq_kernel (query-outer, persistent, one CTA per SM): per 128-row
//     query tile of a unit and per 128-key tile of its list,
//       S = Q K^T and dP = dO V^T into tensor memory, two element-wise
//       warpgroups (64 keys each) form dS in bf16 over S, and
//       dQ += dS K accumulates in tensor memory;
//     the gate gradient of each list entry is summed per tile and warp and
//     added up in warp order;
//   * bwd_kv_kernel (key-outer, lsa-free, in backward_kv.cu) for dK and dV.
//
// Tensor memory of bwd_dq_kernel (512 columns): S double-buffered [0, 256),
// dP [256, 384), dQ [384, 512).  While the element-wise warps work on tile t,
// the tensor core computes S for tile t + 1; once dS(t) is written it runs
// dP(t + 1) and then dQ += dS(t) K(t).  Every wait is bounded; on expiry the
// CTA records kStatusTimeout, lets its copies land, frees TMEM and exits.
#include <math_constants.h>

#include <cstdlib>
#include <cstring>

#include "backward_tc.cuh"
#include "bounds.cuh"
#include "common.cuh"
#include "tc_ptx.cuh"

namespace sa {
namespace {

using namespace tc;

constexpr float kLog2e = 1.4426950408889634f;

// ---------------------------------------------------------------------------
// Row preparation: D = <dO, O> (fp32) and LSE * log2(e) per query row, in a
// layout padded to whole blocks ([B,Hq,Npad], Npad = nb * block): padded rows
// and empty rows get lse2 = +inf (so P = 0) and D = 0.
// ---------------------------------------------------------------------------
__global__ void __launch_bounds__(256) bwd_rowprep_kernel(Shape s, const __nv_bfloat16 *O,
                                                          const __nv_bfloat16 *dO, const float *lse, float *D,
                                                          float *lse2, long long rows_pad, int Npad) {
    // 16 lanes per 128-element row (16-byte loads), two rows per warp
    const long long r = ((long long)blockIdx.x * blockDim.x + threadIdx.x) >> 4;
    const int cv = threadIdx.x & 15;
    const long long bh = r / Npad;
    const int pos = (int)(r - bh * Npad);
    const bool real = r < rows_pad && pos < s.N;
    const long long src = bh * s.N + pos;
    float acc = 0.f;
    if (real) {
        float a[8], b[8];
        load16(O + src * 128 + cv * 8, a);
        load16(dO + src * 128 + cv * 8, b);
#pragma unroll
        for (int i = 0; i < 8; ++i) acc = fmaf(a[i], b[i], acc);
    }
#pragma unroll
    for (int o = 8; o > 0; o >>= 1) acc += __shfl_xor_sync(0xffffffffu, acc, o);
    if (r < rows_pad && cv == 0) {
        D[r] = acc;
        const float l = real ? lse[src] : -CUDART_INF_F;
        lse2[r] = l == -CUDART_INF_F ? CUDART_INF_F : l * kLog2e;   // an empty row: P = 0
    }
}

// ---------------------------------------------------------------------------
// dQ kernel
// ---------------------------------------------------------------------------
constexpr int kThreadsQ = 384;
constexpr int kRegsLaunchQ = 168, kRegsLowQ = 56, kRegsHighQ = 224;
static_assert(128 * kRegsLowQ + 256 * kRegsHighQ <= kThreadsQ * kRegsLaunchQ, "register split");
constexpr uint32_t kChunk = 128 * 128;            // 128 rows x 64 bf16
constexpr uint32_t kTile = 2 * kChunk;            // 128 rows x 128 bf16
constexpr int kStages = 2;
constexpr uint32_t kQOff = 0;                     // Q tile
constexpr uint32_t kDOOff = kTile;                // dO tile
constexpr uint32_t kKOff = 2 * kTile;             // K ring
constexpr uint32_t kVOff = kKOff + kStages * kTile;
constexpr uint32_t kBarOff = kVOff + kStages * kTile;
constexpr int kMaxListQ = 258;
constexpr uint32_t kListOff = kBarOff + 512;     // [2 slots] blk[kMaxListQ], gate[kMaxListQ]
constexpr uint32_t kListBytes = 8 * kMaxListQ;
constexpr uint32_t kSmemQ = kListOff + 2 * kListBytes + 64 + 1024;
static_assert(kSmemQ <= 227 * 1024, "shared memory");

enum {
    Q_L = 0,                    // [2 slots] list loaded
    Q_LF = 2,                   // [2 slots] list released (8 element-wise warps)
    Q_Q = 4,                    // Q and dO tiles landed
    Q_QFREE = 5,                // every S / dP of the item issued and done: Q, dO reusable
    Q_KF = 6,                   // [2] K tile landed
    Q_VF = Q_KF + kStages,      // [2] V tile landed
    Q_KE = Q_VF + kStages,      // [2] K stage free
    Q_VE = Q_KE + kStages,      // [2] V stage free
    Q_S = Q_VE + kStages,       // [2 buffers] S ready
    Q_DP = Q_S + 2,             // dP ready
    Q_DS = Q_DP + 1,            // dS written and dP read (256 arrivals)
    Q_DQ = Q_DS + 1,            // the item's dQ complete
    Q_DQF = Q_DQ + 1,           // dQ read out (256 arrivals)
    Q_END = Q_DQF + 1,
    NBARQ
};
static_assert(8 * NBARQ + 8 <= 512, "barrier area");

struct DqArgs {
    Shape s;
    const int32_t *idx;
    const float *score;
    const int32_t *count;
    const float *D, *lse2;      // [B,Hq,Npad], padded to whole blocks
    float *dQ;                  // [B,Hq,N,d] fp32, overwritten
    float *dgp;                 // [units][MT][cap][8 warps] gate-gradient partials
    unsigned *status;
    int MT;                     // 128-row tiles per unit: G * block / 128
    int Npad;                   // nb * block
    int items;                  // units * MT
    unsigned long long wait_ns;
};

struct Item {
    int b, g, j, m;
    size_t lu;                  // (b, g, j) list row
    int unit;
};

// Item order: the items of one (batch, kv-head) are contiguous (their K/V stay
// in L2), blocks from the last down (longest lists first), row tiles inner.
__device__ __forceinline__ Item item_at(const DqArgs &a, int it) {
    const Shape &s = a.s;
    Item w;
    const int per_g = s.nb * a.MT;
    const int bg = it / per_g;
    int r = it % per_g;
    w.j = s.nb - 1 - r / a.MT;
    w.m = r % a.MT;
    w.g = bg % s.Hkv;
    w.b = bg / s.Hkv;
    w.lu = ((size_t)w.b * s.Hkv + w.g) * s.nb + w.j;
    w.unit = (int)w.lu;
    return w;
}

__device__ __forceinline__ int key_tiles(const Shape &s, int cnt) { return s.bs == 64 ? (cnt + 1) >> 1 : cnt; }

// query row r (0..127) of row tile m: (head offset in the group, position)
__device__ __forceinline__ void row_of(const Shape &s, int j, int m, int r, int &hh, int &pos) {
    if (s.bs == 64) {
        hh = 2 * m + (r >> 6);
        pos = j * 64 + (r & 63);
    } else {
        hh = m;
        pos = j * 128 + r;
    }
}

__global__ void __launch_bounds__(kThreadsQ, 1)
bwd_dq_kernel(const __grid_constant__ CUtensorMap tmQ, const __grid_constant__ CUtensorMap tmK,
              const __grid_constant__ CUtensorMap tmV, const __grid_constant__ CUtensorMap tmDO, DqArgs a) {
    const Shape &s = a.s;
    extern __shared__ unsigned char smem_raw[];
    unsigned char *smem = reinterpret_cast<unsigned char *>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                                            ~uintptr_t(1023));
    const uint32_t sbase = smem_u32(smem);
    uint64_t *bars = reinterpret_cast<uint64_t *>(smem + kBarOff);
    volatile int *abort_flag = reinterpret_cast<volatile int *>(smem + kBarOff + 8 * NBARQ);
    uint32_t *tmem_slot = reinterpret_cast<uint32_t *>(smem + kBarOff + 8 * NBARQ + 4);
    int *cnt_s = reinterpret_cast<int *>(smem + kListOff + 2 * kListBytes);   // [2 slots]
    auto blk_of = [&](int slot) { return reinterpret_cast<int *>(smem + kListOff + slot * kListBytes); };
    auto gate_of = [&](int slot) {
        return reinterpret_cast<float *>(smem + kListOff + slot * kListBytes + 4 * kMaxListQ);
    };
    auto bar = [&](int i) { return smem_u32(&bars[i]); };
    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;

    if (tid == 0) {
        for (int i = 0; i < NBARQ; ++i)
            mbar_init(bar(i), (i == Q_DS || i == Q_DQF) ? 256 : (i == Q_LF || i == Q_LF + 1) ? 8 : 1);
        *abort_flag = 0;
        asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
    }
    if (warp == 1) {
        asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(smem_u32(tmem_slot)),
                     "n"(512));
        asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;");
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = *tmem_slot;

    if (warp == 0) {
        // ---- lists and TMA loads ------------------------------------------
        asm volatile("setmaxnreg.dec.sync.aligned.u32 %0;" ::"n"(kRegsLowQ));
        bool ok = true;
        int gt = 0, nq = 0, ul = 0;
        int qlast = -1, klast[kStages], vlast[kStages];
        for (int i = 0; i < kStages; ++i) klast[i] = vlast[i] = -1;
        for (int it = blockIdx.x; it < a.items; it += gridDim.x, ++ul) {
            const Item w = item_at(a, it);
            const int slot = ul & 1;
            if (ul >= 2) ok = mbar_wait(bar(Q_LF + slot), ((ul >> 1) - 1) & 1, abort_flag, a.status, a.wait_ns);
            if (!__all_sync(0xffffffffu, ok)) { ok = false; break; }
            const int cnt = max(0, min(a.count[w.lu], s.cap));
            int *blk_s = blk_of(slot);
            float *gate_s = gate_of(slot);
            const int32_t *il = a.idx + w.lu * s.cap;
            const float *sl = a.score + w.lu * s.cap;
            const float s_loc = cnt > 0 ? sl[cnt - 1] : 0.f;
            for (int e = lane; e < cnt; e += 32) {
                const int blk = il[e];
                const bool good = blk >= 0 && blk <= w.j && (e == 0 || il[e - 1] < blk);
                if (!good && w.m == 0) set_status(a.status, kStatusBadIndex);
                blk_s[e] = good ? blk : -1;
                const bool forced = (blk == w.j && (s.flags & SA_LOCAL)) || (blk == 0 && (s.flags & SA_SINK));
                gate_s[e] = ((s.flags & SA_GATE) && !forced) ? log_sigmoid(sl[e] - s_loc) * kLog2e : 0.f;
            }
            if (lane == 0) cnt_s[slot] = cnt;
            __syncwarp();
            if (lane == 0) mbar_arrive(bar(Q_L + slot));
            const int T = key_tiles(s, cnt);
            if (lane == 0 && T > 0) {
                if (nq >= 1) ok = mbar_wait(bar(Q_QFREE), (nq - 1) & 1, abort_flag, a.status, a.wait_ns);
                if (ok) {
                    qlast = nq;
                    mbar_expect_tx(bar(Q_Q), 2 * kTile);
                    for (int e = 0; e < 2; ++e) {
                        int hh, pos;
                        row_of(s, w.j, w.m, 64 * e, hh, pos);
                        const int y = (w.b * s.Hq + w.g * s.G + hh) * s.N + pos;
                        SA_CHECK_START(a.status, hh, s.G);
                        SA_CHECK_SPAN(a.status, pos, 64, s.nb * s.bs);
                        for (int c = 0; c < 2; ++c) {
                            tma_load_2d(sbase + kQOff + c * kChunk + e * 8192, &tmQ, bar(Q_Q), 64 * c, y);
                            tma_load_2d(sbase + kDOOff + c * kChunk + e * 8192, &tmDO, bar(Q_Q), 64 * c, y);
                        }
                    }
                }
                const int kvbase = (w.b * s.Hkv + w.g) * s.N;
                auto rows_of_tile = [&](int t, int &y0, int &y1) {
                    if (s.bs == 64) {
                        y0 = kvbase + max(0, blk_s[2 * t]) * 64;
                        y1 = kvbase + max(0, blk_s[min(2 * t + 1, cnt - 1)]) * 64;
                    } else {
                        y0 = kvbase + max(0, blk_s[t]) * 128;
                        y1 = y0 + 64;
                    }
                };
                if (ok && it + (int)gridDim.x < a.items) {
                    // the next item's Q and dO rows into L2 while this one runs
                    const Item nx = item_at(a, it + gridDim.x);
                    for (int e = 0; e < 2; ++e) {
                        int hh, pos;
                        row_of(s, nx.j, nx.m, 64 * e, hh, pos);
                        const int y = (nx.b * s.Hq + nx.g * s.G + hh) * s.N + pos;
                        for (int c = 0; c < 2; ++c) {
                            tma_prefetch_2d(&tmQ, 64 * c, y);
                            tma_prefetch_2d(&tmDO, 64 * c, y);
                        }
                    }
                }
                for (int t = 0; ok && t < T; ++t) {
                    const int gg = gt + t, st = gg % kStages, use = gg / kStages;
                    int y0, y1;
                    rows_of_tile(t, y0, y1);
                    SA_CHECK_START(a.status, y0 - kvbase, s.N);
                    SA_CHECK_START(a.status, y1 - kvbase, s.bs == 64 ? s.N : s.nb * s.bs);   // a block's second half: padded extent
                    if (t + kStages < T) {
                        // the tile after the ring's depth into L2 ahead of its load
                        int p0, p1;
                        rows_of_tile(t + kStages, p0, p1);
                        for (int c = 0; c < 2; ++c) {
                            tma_prefetch_2d(&tmK, 64 * c, p0);
                            tma_prefetch_2d(&tmK, 64 * c, p1);
                            tma_prefetch_2d(&tmV, 64 * c, p0);
                            tma_prefetch_2d(&tmV, 64 * c, p1);
                        }
                    }
                    if (gg >= kStages &&
                        !(ok = mbar_wait(bar(Q_KE + st), (use - 1) & 1, abort_flag, a.status, a.wait_ns)))
                        break;
                    mbar_expect_tx(bar(Q_KF + st), kTile);
                    for (int c = 0; c < 2; ++c) {
                        const uint32_t d = sbase + kKOff + st * kTile + c * kChunk;
                        tma_load_2d(d, &tmK, bar(Q_KF + st), 64 * c, y0);
                        tma_load_2d(d + 8192, &tmK, bar(Q_KF + st), 64 * c, y1);
                    }
                    klast[st] = gg;
                    if (gg >= kStages &&
                        !(ok = mbar_wait(bar(Q_VE + st), (use - 1) & 1, abort_flag, a.status, a.wait_ns)))
                        break;
                    mbar_expect_tx(bar(Q_VF + st), kTile);
                    for (int c = 0; c < 2; ++c) {
                        const uint32_t d = sbase + kVOff + st * kTile + c * kChunk;
                        tma_load_2d(d, &tmV, bar(Q_VF + st), 64 * c, y0);
                        tma_load_2d(d + 8192, &tmV, bar(Q_VF + st), 64 * c, y1);
                    }
                    vlast[st] = gg;
                }
            }
            ok = __shfl_sync(0xffffffffu, ok, 0);
            if (!ok) break;
            gt += T;
            if (T > 0) ++nq;
        }
        if (lane == 0 && *abort_flag) {
            volatile int never = 0;
            if (qlast >= 0) mbar_wait(bar(Q_Q), qlast & 1, &never, a.status, a.wait_ns);
            for (int st = 0; st < kStages; ++st) {
                if (klast[st] >= 0) mbar_wait(bar(Q_KF + st), (klast[st] / kStages) & 1, &never, a.status, a.wait_ns);
                if (vlast[st] >= 0) mbar_wait(bar(Q_VF + st), (vlast[st] / kStages) & 1, &never, a.status, a.wait_ns);
            }
        }
    } else if (warp == 1) {
        // ---- MMA issuer -----------------------------------------------------
        asm volatile("setmaxnreg.dec.sync.aligned.u32 %0;" ::"n"(kRegsLowQ));
        constexpr uint32_t idk = idesc_bf16(false, 128), idm = idesc_bf16(true, 128);
        // C = A B^T with A, B both K-major 128 x 128 tiles in shared memory
        auto gemm_kk = [&](uint32_t dtm, uint32_t aoff, uint32_t boff) {
            const uint64_t da = desc_k_sw128(sbase + aoff), db = desc_k_sw128(sbase + boff);
#pragma unroll
            for (int k = 0; k < 8; ++k) {
                const uint32_t off = ((k >> 2) * kChunk + (k & 3) * 32) >> 4;
                mma_ss_w(dtm, da + off, db + off, idk, k > 0);
            }
        };
        // dQ += dS K: A = dS in TMEM (bf16 pairs: keys 0-63 in columns [0, 32) of
        // the S buffer, keys 64-127 in [64, 96)), B = the K tile, MN-major
        auto dq_mma = [&](uint32_t sbuf, int st, bool acc) {
            const uint64_t db = desc_mn_sw128(sbase + kKOff + st * kTile, kChunk);
#pragma unroll
            for (int k = 0; k < 8; ++k) {
                const uint32_t acol = sbuf + (k < 4 ? 8 * k : 64 + 8 * (k - 4));
                mma_ts_w(tmem + 384, acol, db + ((k * 2048) >> 4), idm, acc || k > 0);
            }
        };
        auto wait = [&](int i, int parity) {
            return __all_sync(0xffffffffu, mbar_wait(bar(i), parity, abort_flag, a.status, a.wait_ns));
        };
        bool ok = true;
        int gt = 0, nq = 0, ul = 0;
        for (int it = blockIdx.x; ok && it < a.items; it += gridDim.x, ++ul) {
            const int slot = ul & 1;
            if (!(ok = wait(Q_L + slot, (ul >> 1) & 1))) break;
            const int T = key_tiles(s, cnt_s[slot]);
            if (T == 0) continue;
            if (!(ok = wait(Q_Q, nq & 1))) break;
            // S(0), dP(0)
            if (!(ok = wait(Q_KF + gt % kStages, (gt / kStages) & 1))) break;
            tc_fence_after();
            gemm_kk(tmem + (gt & 1) * 128, kQOff, kKOff + (gt % kStages) * kTile);
            mma_commit_w(bar(Q_S + (gt & 1)));
            if (!(ok = wait(Q_VF + gt % kStages, (gt / kStages) & 1))) break;
            tc_fence_after();
            gemm_kk(tmem + 256, kDOOff, kVOff + (gt % kStages) * kTile);
            mma_commit_w(bar(Q_DP));
            mma_commit_w(bar(Q_VE + gt % kStages));
            if (T == 1) mma_commit_w(bar(Q_QFREE));
            for (int t = 0; ok && t < T; ++t) {
                const int gg = gt + t;
                if (t + 1 < T) {
                    // S(t + 1) into the other buffer (its dS(t - 1) was read by an earlier dQ MMA)
                    const int g1 = gg + 1;
                    if (!(ok = wait(Q_KF + g1 % kStages, (g1 / kStages) & 1))) break;
                    tc_fence_after();
                    gemm_kk(tmem + (g1 & 1) * 128, kQOff, kKOff + (g1 % kStages) * kTile);
                    mma_commit_w(bar(Q_S + (g1 & 1)));
                }
                // dS(t) written, dP(t) read
                if (!(ok = wait(Q_DS, gg & 1))) break;
                tc_fence_after();
                if (t + 1 < T) {
                    const int g1 = gg + 1;
                    if (!(ok = wait(Q_VF + g1 % kStages, (g1 / kStages) & 1))) break;
                    tc_fence_after();
                    gemm_kk(tmem + 256, kDOOff, kVOff + (g1 % kStages) * kTile);
                    mma_commit_w(bar(Q_DP));
                    mma_commit_w(bar(Q_VE + g1 % kStages));
                    if (t + 2 == T) mma_commit_w(bar(Q_QFREE));
                }
                if (t == 0 && nq > 0) {
                    // the previous item's dQ must have been read out
                    if (!(ok = wait(Q_DQF, (nq - 1) & 1))) break;
                    tc_fence_after();
                }
                dq_mma(tmem + (gg & 1) * 128, gg % kStages, t > 0);
                mma_commit_w(bar(Q_KE + gg % kStages));
                if (t == T - 1) mma_commit_w(bar(Q_DQ));
            }
            gt += T;
            ++nq;
        }
        mma_commit_w(bar(Q_END));
        volatile int never = 0;
        mbar_wait(bar(Q_END), 0, &never, a.status, a.wait_ns);
    } else if (warp < 4) {
        asm volatile("setmaxnreg.dec.sync.aligned.u32 %0;" ::"n"(kRegsLowQ));
    } else {
        asm volatile("setmaxnreg.inc.sync.aligned.u32 %0;" ::"n"(kRegsHighQ));
        // ---- element-wise warpgroups: wg 0 keys 0-63, wg 1 keys 64-127 -------
        const int wg = (warp - 4) >> 2;
        const int qq = warp & 3;
        const int r = 32 * qq + lane;                   // row of the tile (TMEM lane)
        const uint32_t lane_off = (uint32_t)(32 * qq) << 16;
        const bool causal = s.flags & SA_CAUSAL;
        const float sc2 = s.scale * kLog2e;
        const int ew = warp - 4;                        // 0..7: slot of this warp's gate-gradient partials
        bool ok = true;
        int gt = 0, nq = 0, ul = 0;
        for (int it = blockIdx.x; ok && it < a.items; it += gridDim.x, ++ul) {
            const Item w = item_at(a, it);
            const int slot = ul & 1;
            ok = mbar_wait(bar(Q_L + slot), (ul >> 1) & 1, abort_flag, a.status, a.wait_ns);
            if (!__all_sync(0xffffffffu, ok)) { ok = false; break; }
            const int cnt = cnt_s[slot];
            const int *blk_s = blk_of(slot);
            const float *gate_s = gate_of(slot);
            const int T = key_tiles(s, cnt);
            int hh, qi;
            row_of(s, w.j, w.m, r, hh, qi);
            const int head = w.g * s.G + hh;
            const bool row_ok = qi < s.N;
            const size_t grow = ((size_t)w.b * s.Hq + head) * s.N + (row_ok ? qi : 0);
            const size_t prow = ((size_t)w.b * s.Hq + head) * a.Npad + qi;    // +inf, 0 past the sequence
            const float l2 = a.lse2[prow];
            const float Dr = a.D[prow];
            float *dgp = a.dgp + ((size_t)w.unit * a.MT + w.m) * s.cap * 8;   // [entry][8 warps]
            for (int t = 0; t < T; ++t) {
                const int gg = gt + t;
                ok = mbar_wait(bar(Q_S + (gg & 1)), (gg >> 1) & 1, abort_flag, a.status, a.wait_ns);
                ok = ok && mbar_wait(bar(Q_DP), gg & 1, abort_flag, a.status, a.wait_ns);
                if (!__all_sync(0xffffffffu, ok)) { ok = false; break; }
                tc_fence_after();
                const uint32_t tS = tmem + lane_off + (gg & 1) * 128 + 64 * wg;
                const uint32_t tP = tmem + lane_off + 256 + 64 * wg;
                float x[64], y[64];
                tmem_ld32(tS, x);
                tmem_ld32(tS + 32, x + 32);
                tmem_ld32(tP, y);
                tmem_ld32(tP + 32, y + 32);
                tmem_wait_ld();
                reg_fence<64>(x);
                reg_fence<64>(y);
                // this warpgroup's 64 keys: their block, gate and masks
                int blk, t0, e;
                if (s.bs == 64) {
                    e = 2 * t + wg;
                    blk = e < cnt ? blk_s[e] : -1;
                    t0 = blk * 64;
                } else {
                    e = t;
                    blk = blk_s[t];
                    t0 = blk * 128 + 64 * wg;
                }
                const float gl = (blk >= 0 && e < cnt) ? gate_s[e] : 0.f;
                const float bias = gl - l2;
                // keys t0 + k with k < lim are visible to this row
                int lim = 0;
                if (row_ok && blk >= 0) {
                    lim = min(64, s.N - t0);
                    if (causal && blk == w.j) lim = min(lim, qi - t0 + 1);
                }
                float dsum = 0.f;
                uint32_t pk[32];
#pragma unroll
                for (int k = 0; k < 64; k += 2) {
                    float ds2[2];
#pragma unroll
                    for (int q2 = 0; q2 < 2; ++q2) {
                        const float p = k + q2 < lim ? ex2(fmaf(x[k + q2], sc2, bias)) : 0.f;
                        ds2[q2] = p * (y[k + q2] - Dr);
                        dsum += ds2[q2];
                    }
                    __nv_bfloat162 h2 = __floats2bfloat162_rn(ds2[0], ds2[1]);
                    pk[k >> 1] = *reinterpret_cast<uint32_t *>(&h2);
                }
                tmem_st16(tS, pk);
                tmem_st16(tS + 16, pk + 16);
                tmem_wait_st();
                tc_fence_before();
                mbar_arrive(bar(Q_DS));
                // the entry's gate gradient over this warp's 32 rows, into its own slot
                // (block 64: entry e lives in warpgroup e & 1; block 128: in both)
#pragma unroll
                for (int o = 16; o > 0; o >>= 1) dsum += __shfl_xor_sync(0xffffffffu, dsum, o);
                if (lane == 0 && e < cnt) dgp[(size_t)e * 8 + ew] = dsum;
            }
            if (!ok) break;
            // ---- epilogue: dQ rows ---------------------------------------------
            float o[64];
            if (T > 0) {
                ok = mbar_wait(bar(Q_DQ), nq & 1, abort_flag, a.status, a.wait_ns);
                if (!__all_sync(0xffffffffu, ok)) { ok = false; break; }
                tc_fence_after();
                const uint32_t tQ = tmem + lane_off + 384 + 64 * wg;
                tmem_ld32(tQ, o);
                tmem_ld32(tQ + 32, o + 32);
                tmem_wait_ld();
                reg_fence<64>(o);
                tc_fence_before();
                mbar_arrive(bar(Q_DQF));
            } else {
#pragma unroll
                for (int k = 0; k < 64; ++k) o[k] = 0.f;
            }
            if (row_ok) {
                float *drow = a.dQ + grow * 128 + 64 * wg;
#pragma unroll
                for (int k = 0; k < 64; k += 4)
                    *reinterpret_cast<float4 *>(drow + k) =
                        make_float4(o[k] * s.scale, o[k + 1] * s.scale, o[k + 2] * s.scale, o[k + 3] * s.scale);
            }
            __syncwarp();
            if (lane == 0) mbar_arrive(bar(Q_LF + slot));
            gt += T;
            if (T > 0) ++nq;
        }
    }

    tc_fence_before();
    __syncthreads();
    if (warp == 1) {
        tc_fence_after();
        asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(tmem), "n"(512));
    }
}

// Gate gradients (summed over the unit's row tiles in order) -> score
// gradients: dg sigmoid(-(s - s_loc)) on gated entries, the local entry minus
// their sum, 0 elsewhere.
__global__ void bwd_score_tc_kernel(Shape s, const int32_t *idx, const float *score, const int32_t *count,
                                    const float *dgp, int MT, float *dscore, int units) {
    const int u = blockIdx.x * blockDim.x + threadIdx.x;
    if (u >= units) return;
    const int j = u % s.nb;
    const int cnt = max(0, min(count[u], s.cap));
    const int32_t *il = idx + (size_t)u * s.cap;
    const float *sl = score + (size_t)u * s.cap;
    float *ds = dscore + (size_t)u * s.cap;
    const float s_loc = cnt > 0 ? sl[cnt - 1] : 0.f;
    float sum = 0.f;
    int loc = -1;
    for (int c = 0; c < s.cap; ++c) {
        float v = 0.f;
        if (c < cnt) {
            const int blk = il[c];
            const bool forced = (blk == j && (s.flags & SA_LOCAL)) || (blk == 0 && (s.flags & SA_SINK));
            if (blk == j) loc = c;
            if ((s.flags & SA_GATE) && !forced && blk >= 0 && blk <= j) {
                // row tiles in order, and in each the warps that held the entry in warp order
                float dg = 0.f;
                for (int m = 0; m < MT; ++m) {
                    const float *p = dgp + (((size_t)u * MT + m) * s.cap + c) * 8;
                    if (s.bs == 64) {
                        for (int q = 0; q < 4; ++q) dg += p[4 * (c & 1) + q];
                    } else {
                        for (int q = 0; q < 8; ++q) dg += p[q];
                    }
                }
                const float x = sl[c] - s_loc;
                v = dg / (1.f + expf(x));          // dg * sigmoid(-x)
                sum += v;
            }
        }
        ds[c] = v;
    }
    if (loc >= 0) ds[loc] -= sum;
}

}  // namespace

bool backward_tc_shape_ok(const Shape &s) {
    if (s.dtype != SA_BF16 || s.d != 128) return false;
    if (s.flags & (SA_HIER | SA_SELECT_PER_QHEAD)) return false;
    if (s.bs != 64 && s.bs != 128) return false;
    if ((s.G * s.bs) % 128) return false;
    return s.cap <= kMaxListQ;
}

bool backward_tc_supported(const Shape &s) {
    if (!backward_tc_shape_ok(s)) return false;
    const char *e = getenv("SPARSE_ATTN_BACKWARD_PATH");
    return !(e && strcmp(e, "simt") == 0);
}

size_t backward_tc_workspace(const Shape &s) {
    const size_t rows = (size_t)s.B * s.Hq * s.nb * s.bs;
    const size_t units = (size_t)s.B * s.Hkv * s.nb;
    const int MT = s.G * s.bs / 128;
    auto al = [](size_t x) { return (x + 255) & ~(size_t)255; };
    return al(rows * 4) * 2 + al(units * MT * s.cap * 8 * 4) + backward_kv_workspace(s);
}

cudaError_t launch_backward_tc(const Shape &s, const void *Q, const void *K, const void *V, const void *O,
                               const float *lse, const void *dO, const int32_t *idx, const float *score,
                               const int32_t *count, float *dQ, float *dK, float *dV, float *dscore, void *ws,
                               cudaStream_t st) {
    auto al = [](size_t x) { return (x + 255) & ~(size_t)255; };
    const int Npad = s.nb * s.bs;
    const size_t rows = (size_t)s.B * s.Hq * Npad;
    const size_t units = (size_t)s.B * s.Hkv * s.nb;
    const int MT = s.G * s.bs / 128;
    unsigned char *w = static_cast<unsigned char *>(ws) + ws_layout(s).scratch;
    float *D = reinterpret_cast<float *>(w);
    w += al(rows * 4);
    float *lse2 = reinterpret_cast<float *>(w);
    w += al(rows * 4);
    float *dgp = reinterpret_cast<float *>(w);
    w += al(units * MT * s.cap * 8 * 4);
    unsigned *status = static_cast<unsigned *>(ws);

    bwd_rowprep_kernel<<<(unsigned)((rows * 16 + 255) / 256), 256, 0, st>>>(
        s, (const __nv_bfloat16 *)O, (const __nv_bfloat16 *)dO, lse, D, lse2, (long long)rows, Npad);
    note_launch();
    cudaError_t e = cudaGetLastError();
    if (e != cudaSuccess) return e;

    // dQ and the gate-gradient partials
    cudaFuncAttributes fa;
    if ((e = cudaFuncGetAttributes(&fa, bwd_dq_kernel)) != cudaSuccess) return e;
    if (fa.numRegs != kRegsLaunchQ) return cudaErrorInvalidDeviceFunction;
    CUtensorMap mq, mk, mv, mdo;
    const uint64_t qrows = (uint64_t)s.B * s.Hq * s.N, krows = (uint64_t)s.B * s.Hkv * s.N;
    if (!make_map_d128(&mq, Q, qrows, 64) || !make_map_d128(&mk, K, krows, 64) || !make_map_d128(&mv, V, krows, 64) ||
        !make_map_d128(&mdo, dO, qrows, 64))
        return cudaErrorInvalidValue;
    DqArgs a{};
    a.s = s;
    a.idx = idx;
    a.score = score;
    a.count = count;
    a.D = D;
    a.lse2 = lse2;
    a.dQ = dQ;
    a.dgp = dgp;
    a.status = status;
    a.MT = MT;
    a.Npad = Npad;
    a.items = (int)(units * MT);
    a.wait_ns = kWaitNs;
    const int sms = sm_count();
    if (sms <= 0) return cudaErrorNoDevice;
    if ((e = cudaFuncSetAttribute(bwd_dq_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)kSmemQ)) !=
        cudaSuccess)
        return e;
    bwd_dq_kernel<<<(unsigned)min(a.items, sms), kThreadsQ, kSmemQ, st>>>(mq, mk, mv, mdo, a);
    note_launch();
    if ((e = cudaGetLastError()) != cudaSuccess) return e;

    // dK and dV (key-outer)
    int *rcnt = reinterpret_cast<int *>(static_cast<unsigned char *>(ws) + ws_layout(s).bwd_kv);
    if ((e = launch_backward_kv(s, Q, K, V, dO, D, lse2, idx, score, count, dK, dV, w, rcnt, status, st)) !=
        cudaSuccess)
        return e;

    bwd_score_tc_kernel<<<(unsigned)((units + 127) / 128), 128, 0, st>>>(s, idx, score, count, dgp, MT, dscore,
                                                                        (int)units);
    note_launch();
    return cudaGetLastError();
}

}  // namespace sa
