// backward_kv.cu -- dK and dV of the gated block-sparse prefill on the tensor
// cores, key tile by key tile ([SAS] "Как это применить": the backward of the
// gated softmax attention over the forward's kept lists).
//
// For a tile of 128 keys (two blocks of 64, or one block of 128) the rows that
// attend to it are those of the units whose lists keep one of its blocks: its
// inverse list.  With P = exp(z - LSE) and dS = P (dO V^T - D):
//
//   dV[tile] = sum over kept units u of  P_u^T dO_u
//   dK[tile] = scale * sum over kept units u of  dS_u^T Q_u
//
// accumulated in tensor memory while the tile's K and V stay in shared memory.
// A 128-row tile of a unit (a "pair") is taken in two halves of 64 rows, each
// with its own tensor-memory buffer: the tensor core computes S^T = K Q_h^T
// and dP^T = V dO_h^T for half h, the element-wise warpgroup h turns them into
// P^T and dS^T in bf16 in place, and dV += P_h^T dO_h, dK += dS_h^T Q_h follow;
// while one warpgroup works on its half the tensor core serves the other.
// Tensor memory: half 0 S^T [0, 64) dP^T [64, 128), half 1 [128, 256),
// dV [256, 384), dK [384, 512).
//
// Preparation (no atomics in the sums, fixed order): a warp per key tile walks
// the later blocks' lists (each ascending) and records, in unit order, the
// units that keep the tile with the gates of its blocks in log2 units; a scan
// turns the counts into offsets, and the work items are ordered group by group
// ((batch, kv-head)), largest first within a group.  The CTAs claim items in
// that order from a global counter, so a CTA that finishes early takes more
// and the CTAs work on one or two groups at a time: the Q and dO rows they
// re-read (those of the units that keep each tile) stay in L2.
// A tile kept by more than 64 units is split into work items of 64; each
// split leaves its accumulators in a partial slot, and for each warp's region
// the split that finishes last sums the slots in split order.  The per-row
// LSE and D come from a layout padded to whole blocks, so that each pair's
// rows are contiguous 16-byte-aligned runs fetched by bulk copies.
#include <math_constants.h>

#include "backward_tc.cuh"
#include "bounds.cuh"
#include "common.cuh"
#include "tc_ptx.cuh"

namespace sa {
namespace {

using namespace tc;

constexpr float kLog2e = 1.4426950408889634f;
constexpr int kUMax = 64;          // units per work item

struct KvLayout {
    int KT, bpt, tiles, MT;
    size_t pairs_max, items_max, slots_max;
    size_t off_tcnt, off_toff, off_tsplit, off_tslot, off_ioff, off_tot, off_ent, off_items, off_order, off_part,
        bytes;
};

KvLayout kv_layout(const Shape &s) {
    KvLayout L{};
    L.bpt = 128 / s.bs;
    L.KT = (s.nb + L.bpt - 1) / L.bpt;
    L.tiles = s.B * s.Hkv * L.KT;
    L.MT = s.G * s.bs / 128;
    const size_t units = (size_t)s.B * s.Hkv * s.nb;
    L.pairs_max = units * s.cap;
    L.slots_max = 2 * L.pairs_max / kUMax + 1;
    L.items_max = (size_t)L.tiles + L.pairs_max / kUMax + 1;
    auto al = [](size_t x) { return (x + 255) & ~(size_t)255; };
    size_t o = 0;
    L.off_tcnt = o;   o += al((size_t)L.tiles * 4);
    L.off_toff = o;   o += al((size_t)L.tiles * 4);
    L.off_tsplit = o; o += al((size_t)L.tiles * 4);
    L.off_tslot = o;  o += al((size_t)L.tiles * 4);
    L.off_ioff = o;   o += al((size_t)L.tiles * 4);
    L.off_tot = o;    o += 256;
    L.off_ent = o;    o += al(L.pairs_max * 16);
    L.off_items = o;  o += al(L.items_max * 16);
    L.off_order = o;  o += al(L.items_max * 4);
    L.off_part = o;   o += al(L.slots_max * 2 * 128 * 128 * 4);
    L.bytes = o;
    return L;
}

struct InvArgs {
    Shape s;
    const int32_t *idx, *count;
    const float *score;
    int KT, bpt, tiles;
    int *tcnt, *toff, *tsplit, *tslot, *ioff, *tot, *order;
    int4 *ent, *items;
};

// list entry of block `blk` in an ascending list, or -1
__device__ __forceinline__ int find_entry(const int32_t *il, int cnt, int blk) {
    int lo = 0, hi = cnt;
    while (lo < hi) {
        const int m = (lo + hi) >> 1;
        if (il[m] < blk) lo = m + 1;
        else hi = m;
    }
    return (lo < cnt && il[lo] == blk) ? lo : -1;
}

// Gate of list entry c (block blk) of unit j in log2 units; -inf when the
// unit does not keep the block.  Forced entries (sink, local) carry no gate.
__device__ __forceinline__ float entry_gate2(const Shape &s, const float *sl, int cnt, int c, int blk, int j) {
    if (c < 0) return -CUDART_INF_F;
    const bool forced = (blk == j && (s.flags & SA_LOCAL)) || (blk == 0 && (s.flags & SA_SINK));
    if (!(s.flags & SA_GATE) || forced) return 0.f;
    return log_sigmoid(sl[c] - sl[cnt - 1]) * kLog2e;
}

// A warp per key tile: pass 0 counts the units that keep one of its blocks,
// pass 1 records them (ascending unit) with their gates, and the tile's work
// items.  Entry: (unit j, gate of the tile's first block, of its second, 0),
// gates as float bits.
__global__ void inv_kernel(InvArgs a, int pass) {
    const int t = (int)(((size_t)blockIdx.x * blockDim.x + threadIdx.x) >> 5), lane = threadIdx.x & 31;
    if (t >= a.tiles) return;
    const Shape &s = a.s;
    const int bg = t / a.KT, kt = t % a.KT;
    const int b0 = kt * a.bpt, b1 = min(s.nb, b0 + a.bpt);
    const int base = pass ? a.toff[t] : 0;
    int n = 0;
    for (int j0 = b0; j0 < s.nb; j0 += 32) {          // a unit keeps only blocks up to its own
        const int j = j0 + lane;
        int c0 = -1, c1 = -1, cnt = 0;
        size_t lu = 0;
        if (j < s.nb) {
            lu = (size_t)bg * s.nb + j;
            cnt = max(0, min(a.count[lu], s.cap));
            const int32_t *il = a.idx + lu * s.cap;
            c0 = find_entry(il, cnt, b0);
            if (b0 + 1 < b1) c1 = find_entry(il, cnt, b0 + 1);
        }
        const bool keep = c0 >= 0 || c1 >= 0;
        const unsigned m = __ballot_sync(0xffffffffu, keep);
        if (pass && keep) {
            const float *sl = a.score + lu * s.cap;
            const float g0 = entry_gate2(s, sl, cnt, c0, b0, j);
            const float g1 = a.bpt == 2 ? entry_gate2(s, sl, cnt, c1, b0 + 1, j) : g0;
            a.ent[base + n + __popc(m & ((1u << lane) - 1u))] =
                make_int4(j, __float_as_int(g0), __float_as_int(g1), 0);
        }
        n += __popc(m);
    }
    if (!pass) {
        if (lane == 0) a.tcnt[t] = n;
        return;
    }
    const int ns = a.tsplit[t];                        // an unkept tile still gets one item (zeros)
    for (int sp = lane; sp < ns; sp += 32)
        a.items[a.ioff[t] + sp] = make_int4(t, base + sp * kUMax, base + min(n, (sp + 1) * kUMax), sp);
}

// One CTA: offsets of every tile's units, items and partial slots.
__global__ void __launch_bounds__(1024) inv_scan_kernel(InvArgs a) {
    __shared__ int wsum[32][3];
    __shared__ int carry[3];
    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    if (tid < 3) carry[tid] = 0;
    __syncthreads();
    for (int t0 = 0; t0 < a.tiles; t0 += 1024) {
        const int t = t0 + tid;
        const int n = t < a.tiles ? a.tcnt[t] : 0;
        const int ns = t < a.tiles ? max(1, (n + kUMax - 1) / kUMax) : 0;
        const int sl = ns > 1 ? ns : 0;
        int v[3] = {n, ns, sl}, incl[3];
#pragma unroll
        for (int q = 0; q < 3; ++q) {
            int x = v[q];
#pragma unroll
            for (int o = 1; o < 32; o <<= 1) {
                const int y = __shfl_up_sync(0xffffffffu, x, o);
                if (lane >= o) x += y;
            }
            incl[q] = x;
            if (lane == 31) wsum[warp][q] = x;
        }
        __syncthreads();
        int add[3] = {0, 0, 0}, tot[3] = {0, 0, 0};
        for (int w = 0; w < 32; ++w)
#pragma unroll
            for (int q = 0; q < 3; ++q) {
                if (w < warp) add[q] += wsum[w][q];
                tot[q] += wsum[w][q];
            }
        if (t < a.tiles) {
            a.toff[t] = carry[0] + add[0] + incl[0] - v[0];
            a.tsplit[t] = ns;
            a.ioff[t] = carry[1] + add[1] + incl[1] - v[1];
            a.tslot[t] = carry[2] + add[2] + incl[2] - v[2];
        }
        __syncthreads();
        if (tid < 3) carry[tid] += tot[tid];
        __syncthreads();
    }
    if (tid == 0) {
        a.tot[0] = carry[1];     // work items
        a.tot[1] = carry[0];     // (tile, unit) entries
        a.tot[2] = carry[2];     // partial slots
        a.tot[3] = 0;            // the dK/dV kernel's claim counter
    }
}

// A CTA per (batch, kv-head): the order of that group's items -- largest first
// (items of equal size in any order; the results do not depend on it).
__global__ void __launch_bounds__(1024) inv_order_kernel(InvArgs a) {
    __shared__ int hist[kUMax + 1], cur[kUMax + 1];
    const int tid = threadIdx.x, bg = blockIdx.x;
    const int t0 = bg * a.KT, t1 = t0 + a.KT;
    if (tid <= kUMax) hist[tid] = 0;
    __syncthreads();
    for (int t = t0 + tid; t < t1; t += blockDim.x) {
        const int n = a.tcnt[t], full = n / kUMax, rem = n - full * kUMax;
        if (full) atomicAdd(&hist[kUMax], full);
        if (rem || n == 0) atomicAdd(&hist[rem], 1);
    }
    __syncthreads();
    if (tid == 0) {
        int pos = a.ioff[t0];           // the group's items start here
        for (int sz = kUMax; sz >= 0; --sz) {
            cur[sz] = pos;
            pos += hist[sz];
        }
    }
    __syncthreads();
    for (int t = t0 + tid; t < t1; t += blockDim.x) {
        const int n = a.tcnt[t], io = a.ioff[t];
        const int ns = max(1, (n + kUMax - 1) / kUMax);
        for (int sp = 0; sp < ns; ++sp) {
            const int sz = min(kUMax, n - sp * kUMax);
            a.order[atomicAdd(&cur[sz], 1)] = io + sp;
        }
    }
}

// ---------------------------------------------------------------------------
// dK / dV kernel
// ---------------------------------------------------------------------------
constexpr int kThreadsKV = 384;
constexpr int kRegsLaunchKV = 168, kRegsLowKV = 56, kRegsHighKV = 224;
static_assert(128 * kRegsLowKV + 256 * kRegsHighKV <= kThreadsKV * kRegsLaunchKV, "register split");
constexpr uint32_t kChunk = 128 * 128;
constexpr uint32_t kTile = 2 * kChunk;
constexpr uint32_t kKOff = 0, kVOff = kTile;
constexpr uint32_t kRingOff = 2 * kTile;           // [2 stages] Q tile, dO tile
constexpr uint32_t kStageBytes = 2 * kTile;
constexpr uint32_t kRowOff = kRingOff + 2 * kStageBytes;    // [2 stages] lse2[128], D[128]
constexpr uint32_t kRowBytes = 2 * 128 * 4;
constexpr uint32_t kInfoOff = kRowOff + 2 * kRowBytes;      // [2 stages] the pair's entry (int4)
constexpr uint32_t kInfoBytes = 16;
constexpr uint32_t kItemOff = kInfoOff + 2 * kInfoBytes;    // [4] claimed item ids (-1: no more)
constexpr uint32_t kBarOffKV = kItemOff + 16 + 32;
constexpr uint32_t kSmemKV = kBarOffKV + 512 + 1024;
static_assert(kSmemKV <= 227 * 1024, "shared memory");
static_assert(kRowOff % 16 == 0 && kRowBytes % 16 == 0, "bulk copy alignment");

enum {
    B_KVF = 0,          // K, V tiles landed
    B_KVE = 1,          // K, V tiles free
    B_PF = 2,           // [2] pair stage full
    B_PE = 4,           // [2] pair stage free
    B_ST = 6,           // [2 halves] S^T, dP^T of the half ready
    B_EW = 8,           // [2 halves] P^T, dS^T of the half written (128 arrivals)
    B_ACC = 10,         // the item's dV, dK complete
    B_ACCF = 11,        // dV, dK read out (256 arrivals)
    B_END = 12,
    B_IF = 13,          // [4] item slot published
    B_IE = 17,          // [4] item slot read (the MMA warp and the 8 element-wise warps)
    NBARKV = 21
};
static_assert(8 * NBARKV + 8 <= 512, "barrier area");

struct KvArgs {
    Shape s;
    const float *D, *lse2;      // [B,Hq,Npad] (Npad = nb * block; rows past N: D 0, lse2 +inf)
    float *dK, *dV;
    const int *tsplit, *tslot, *order;
    int *tot;                   // [0] items; [3] the claim counter (zero at launch)
    int *rcnt;                  // [tiles][8 regions] splits finished
    const int4 *ent, *items;
    float *part;                // [slots][2][128][128]
    unsigned *status;
    int KT, MT, Npad;
    unsigned long long wait_ns;
};

// The CTA's k-th work item, published by warp 0 in item slot k % 4: warps
// 1 and 4..11 wait for it, and one lane of each tells the slot is read.
__device__ __forceinline__ int item_read(const KvArgs &a, const volatile int *itq, uint32_t bar_if, uint32_t bar_ie,
                                         int k, volatile int *abort_flag, bool &ok) {
    ok = tc::mbar_wait(bar_if, (k >> 2) & 1, abort_flag, a.status, a.wait_ns);
    ok = __all_sync(0xffffffffu, ok);
    const int it = ok ? itq[k & 3] : -1;
    __syncwarp();
    if ((threadIdx.x & 31) == 0) tc::mbar_arrive(bar_ie);
    return it;
}

__global__ void __launch_bounds__(kThreadsKV, 1)
bwd_kv_kernel(const __grid_constant__ CUtensorMap tmQ, const __grid_constant__ CUtensorMap tmK,
              const __grid_constant__ CUtensorMap tmV, const __grid_constant__ CUtensorMap tmDO, KvArgs a) {
    const Shape &s = a.s;
    extern __shared__ unsigned char smem_raw[];
    unsigned char *smem = reinterpret_cast<unsigned char *>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                                            ~uintptr_t(1023));
    const uint32_t sbase = smem_u32(smem);
    uint64_t *bars = reinterpret_cast<uint64_t *>(smem + kBarOffKV);
    volatile int *abort_flag = reinterpret_cast<volatile int *>(smem + kBarOffKV + 8 * NBARKV);
    uint32_t *tmem_slot = reinterpret_cast<uint32_t *>(smem + kBarOffKV + 8 * NBARKV + 4);
    auto bar = [&](int i) { return smem_u32(&bars[i]); };
    auto rows_of = [&](int st) { return reinterpret_cast<float *>(smem + kRowOff + st * kRowBytes); };
    auto info_of = [&](int st) { return reinterpret_cast<int4 *>(smem + kInfoOff + st * kInfoBytes); };
    volatile int *itq = reinterpret_cast<volatile int *>(smem + kItemOff);
    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const int nitems = a.tot[0];

    if (tid == 0) {
        for (int i = 0; i < NBARKV; ++i)
            mbar_init(bar(i), (i == B_EW || i == B_EW + 1) ? 128 : i == B_ACCF ? 256 : (i >= B_IE) ? 9 : 1);
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
        // ---- K/V of the tile, then per pair: entry, rows, Q and dO ----------
        asm volatile("setmaxnreg.dec.sync.aligned.u32 %0;" ::"n"(kRegsLowKV));
        bool ok = true;
        int gp = 0, ni = 0;
        int kvlast = -1;                 // phase of the last K/V load issued
        int plast[2] = {-1, -1};         // last pair issued on each ring stage
        // claims run one item ahead of the item being loaded
        int nxt = 0;
        if (lane == 0) nxt = atomicAdd(a.tot + 3, 1);
        for (int k = 0;; ++k) {
            int it = -1;
            if (lane == 0) {
                if (ok && nxt < nitems) {
                    it = a.order[nxt];
                    nxt = atomicAdd(a.tot + 3, 1);
                }
                // publish it in slot k % 4 once the slot's previous item has been read
                if (k >= 4 && !mbar_wait(bar(B_IE + (k & 3)), ((k >> 2) - 1) & 1, abort_flag, a.status, a.wait_ns))
                    ok = false;
                itq[k & 3] = ok ? it : -1;
                mbar_arrive(bar(B_IF + (k & 3)));
            }
            ok = __shfl_sync(0xffffffffu, ok, 0);
            it = __shfl_sync(0xffffffffu, it, 0);
            if (!ok || it < 0) break;
            const int4 item = a.items[it];
            const int np = (item.z - item.y) * a.MT;
            if (np == 0) continue;
            const int bg = item.x / a.KT, kt = item.x % a.KT;
            const int b = bg / s.Hkv, g = bg % s.Hkv;
            if (lane == 0) {
                if (ni >= 1) ok = mbar_wait(bar(B_KVE), (ni - 1) & 1, abort_flag, a.status, a.wait_ns);
                if (ok) {
                    mbar_expect_tx(bar(B_KVF), 2 * kTile);
                    const int y = bg * s.N + kt * 128;
                    SA_CHECK_START(a.status, kt * 128, s.N);
                    for (int c = 0; c < 2; ++c)
                        for (int e = 0; e < 2; ++e) {
                            tma_load_2d(sbase + kKOff + c * kChunk + e * 8192, &tmK, bar(B_KVF), 64 * c, y + 64 * e);
                            tma_load_2d(sbase + kVOff + c * kChunk + e * 8192, &tmV, bar(B_KVF), 64 * c, y + 64 * e);
                        }
                    kvlast = ni;
                }
            }
            ok = __shfl_sync(0xffffffffu, ok, 0);
            if (!ok) break;
            int4 mine = make_int4(0, 0, 0, 0);
            for (int p = 0; p < np; ++p, ++gp) {
                const int st = gp & 1, ui = p / a.MT, m = p % a.MT;
                if (m == 0 && (ui & 31) == 0) {
                    const int e = item.y + ui + lane;
                    mine = e < item.z ? a.ent[e] : make_int4(0, 0, 0, 0);
                }
                int4 en;
                en.x = __shfl_sync(0xffffffffu, mine.x, ui & 31);
                en.y = __shfl_sync(0xffffffffu, mine.y, ui & 31);
                en.z = __shfl_sync(0xffffffffu, mine.z, ui & 31);
                en.w = 0;
                // the Q and dO rows of the pair two ahead into L2 (its unit's entry is
                // in this batch of 32 unless it starts the next one)
                const int pa = p + 2, ua = pa / a.MT;
                const int ja = __shfl_sync(0xffffffffu, mine.x, ua & 31);
                if (lane < 2 && pa < np && (ua >> 5) == (ui >> 5)) {
                    const int ma = pa % a.MT, e = lane;
                    const int hh = s.bs == 64 ? 2 * ma + e : ma;
                    const int pos = s.bs == 64 ? ja * 64 : ja * 128 + 64 * e;
                    const int y = (b * s.Hq + g * s.G + hh) * s.N + pos;
                    for (int c = 0; c < 2; ++c) {
                        tma_prefetch_2d(&tmQ, 64 * c, y);
                        tma_prefetch_2d(&tmDO, 64 * c, y);
                    }
                }
                if (lane == 0) {
                    if (gp >= 2) ok = mbar_wait(bar(B_PE + st), ((gp >> 1) - 1) & 1, abort_flag, a.status, a.wait_ns);
                    if (ok) {
                        const int j = en.x;
                        *info_of(st) = en;
                        mbar_expect_tx(bar(B_PF + st), 2 * kTile + kRowBytes);
                        const uint32_t qd = sbase + kRingOff + st * kStageBytes, dd = qd + kTile;
                        const uint32_t rw = sbase + kRowOff + st * kRowBytes;
                        for (int e = 0; e < 2; ++e) {
                            // rows 64 e .. 64 e + 63: (head, first position)
                            const int hh = s.bs == 64 ? 2 * m + e : m;
                            const int pos = s.bs == 64 ? j * 64 : j * 128 + 64 * e;
                            const int y = (b * s.Hq + g * s.G + hh) * s.N + pos;
                            SA_CHECK_START(a.status, hh, s.G);
                            SA_CHECK_SPAN(a.status, pos, 64, a.Npad);
                            for (int c = 0; c < 2; ++c) {
                                tma_load_2d(qd + c * kChunk + e * 8192, &tmQ, bar(B_PF + st), 64 * c, y);
                                tma_load_2d(dd + c * kChunk + e * 8192, &tmDO, bar(B_PF + st), 64 * c, y);
                            }
                            const size_t rp = (size_t)(b * s.Hq + g * s.G + hh) * a.Npad + pos;
                            bulk_load(rw + 256 * e, a.lse2 + rp, 256, bar(B_PF + st));
                            bulk_load(rw + 512 + 256 * e, a.D + rp, 256, bar(B_PF + st));
                        }
                        plast[st] = gp;
                    }
                }
                ok = __shfl_sync(0xffffffffu, ok, 0);
                if (!ok) break;
            }
            if (!ok) break;
            ++ni;
        }
        if (lane == 0 && *abort_flag) {
            volatile int never = 0;
            if (kvlast >= 0) mbar_wait(bar(B_KVF), kvlast & 1, &never, a.status, a.wait_ns);
            for (int st = 0; st < 2; ++st)
                if (plast[st] >= 0) mbar_wait(bar(B_PF + st), (plast[st] >> 1) & 1, &never, a.status, a.wait_ns);
        }
    } else if (warp == 1) {
        // ---- MMA issuer -----------------------------------------------------
        asm volatile("setmaxnreg.dec.sync.aligned.u32 %0;" ::"n"(kRegsLowKV));
        constexpr uint32_t idh = idesc_bf16(false, 64), idm = idesc_bf16(true, 128);
        // half h of a pair into buffer h: S^T = K Q_h^T (N = 64 rows), dP^T = V dO_h^T
        auto sdp = [&](int st, int h) {
            const uint32_t qo = kRingOff + st * kStageBytes + h * 8192, doo = qo + kTile;
            const uint64_t dk = desc_k_sw128(sbase + kKOff), dv = desc_k_sw128(sbase + kVOff);
            const uint64_t dq = desc_k_sw128(sbase + qo), dd = desc_k_sw128(sbase + doo);
#pragma unroll
            for (int k = 0; k < 8; ++k) {
                const uint32_t off = ((k >> 2) * kChunk + (k & 3) * 32) >> 4;
                mma_ss_w(tmem + 128 * h, dk + off, dq + off, idh, k > 0);
            }
#pragma unroll
            for (int k = 0; k < 8; ++k) {
                const uint32_t off = ((k >> 2) * kChunk + (k & 3) * 32) >> 4;
                mma_ss_w(tmem + 128 * h + 64, dv + off, dd + off, idh, k > 0);
            }
        };
        // dV += P_h^T dO_h, dK += dS_h^T Q_h: A in tensor memory (bf16 pairs of
        // the half's 64 rows in columns [0, 32) of S^T / dP^T), B = the half's
        // rows of the stage's tiles, MN-major
        auto acc_half = [&](int st, int h, bool acc) {
            const uint32_t qo = kRingOff + st * kStageBytes, doo = qo + kTile;
            const uint64_t dd = desc_mn_sw128(sbase + doo, kChunk), dq = desc_mn_sw128(sbase + qo, kChunk);
#pragma unroll
            for (int k = 0; k < 4; ++k)
                mma_ts_w(tmem + 256, tmem + 128 * h + 8 * k, dd + (((4 * h + k) * 2048) >> 4), idm, acc || k > 0);
#pragma unroll
            for (int k = 0; k < 4; ++k)
                mma_ts_w(tmem + 384, tmem + 128 * h + 64 + 8 * k, dq + (((4 * h + k) * 2048) >> 4), idm,
                         acc || k > 0);
        };
        auto wait = [&](int i, int parity) {
            return __all_sync(0xffffffffu, mbar_wait(bar(i), parity, abort_flag, a.status, a.wait_ns));
        };
        bool ok = true;
        int gp = 0, ni = 0;
        for (int k = 0; ok; ++k) {
            const int it = item_read(a, itq, bar(B_IF + (k & 3)), bar(B_IE + (k & 3)), k, abort_flag, ok);
            if (!ok || it < 0) break;
            const int4 item = a.items[it];
            const int np = (item.z - item.y) * a.MT;
            if (np == 0) continue;
            if (!(ok = wait(B_KVF, ni & 1))) break;
            if (!(ok = wait(B_PF + (gp & 1), (gp >> 1) & 1))) break;
            tc_fence_after();
            sdp(gp & 1, 0);
            mma_commit_w(bar(B_ST));
            sdp(gp & 1, 1);
            mma_commit_w(bar(B_ST + 1));
            for (int p = 0; ok && p < np; ++p, ++gp) {
                const int st = gp & 1;
                const bool more = p + 1 < np;
                for (int h = 0; h < 2; ++h) {
                    if (!(ok = wait(B_EW + h, gp & 1))) break;
                    tc_fence_after();
                    if (p == 0 && h == 0 && ni > 0) {
                        // the previous item's accumulators must have been read out
                        if (!(ok = wait(B_ACCF, (ni - 1) & 1))) break;
                        tc_fence_after();
                    }
                    acc_half(st, h, p > 0 || h > 0);
                    if (h == 1) mma_commit_w(bar(B_PE + st));
                    if (more) {
                        // the next pair's half h into the buffer just read (the MMAs run in order)
                        if (h == 0 && !(ok = wait(B_PF + (st ^ 1), ((gp + 1) >> 1) & 1))) break;
                        tc_fence_after();
                        sdp(st ^ 1, h);
                        mma_commit_w(bar(B_ST + h));
                    }
                }
            }
            if (!ok) break;
            mma_commit_w(bar(B_ACC));
            mma_commit_w(bar(B_KVE));
            ++ni;
        }
        mma_commit_w(bar(B_END));
        volatile int never = 0;
        mbar_wait(bar(B_END), 0, &never, a.status, a.wait_ns);
    } else if (warp < 4) {
        asm volatile("setmaxnreg.dec.sync.aligned.u32 %0;" ::"n"(kRegsLowKV));
    } else {
        asm volatile("setmaxnreg.inc.sync.aligned.u32 %0;" ::"n"(kRegsHighKV));
        // ---- element-wise warpgroups: wg h takes half h (rows 64 h .. 64 h + 63)
        // of every pair; for the accumulators, columns 64 wg .. 64 wg + 63 ----
        const int wg = (warp - 4) >> 2, qq = warp & 3, ew = warp - 4;
        const int kl = 32 * qq + lane;                   // key lane of the tile
        const uint32_t lane_off = (uint32_t)(32 * qq) << 16;
        const uint32_t tb = tmem + lane_off + 128 * wg;  // this half's buffer
        const bool causal = s.flags & SA_CAUSAL;
        const float sc2 = s.scale * kLog2e;
        bool ok = true;
        int gp = 0, ni = 0;
        for (int k = 0; ok; ++k) {
            const int it = item_read(a, itq, bar(B_IF + (k & 3)), bar(B_IE + (k & 3)), k, abort_flag, ok);
            if (!ok || it < 0) break;
            const int4 item = a.items[it];
            const int np = (item.z - item.y) * a.MT;
            const int bg = item.x / a.KT, kt = item.x % a.KT;
            const int key = kt * 128 + kl;
            const bool key_ok = key < s.N;
            const int hk = s.bs == 64 ? (kl >> 6) : 0;             // the key's block within the tile
            const int blk = s.bs == 64 ? kt * 2 + hk : kt;
            float *dkrow = a.dK + ((size_t)bg * s.N + (key_ok ? key : 0)) * 128 + 64 * wg;
            float *dvrow = a.dV + ((size_t)bg * s.N + (key_ok ? key : 0)) * 128 + 64 * wg;
            if (np == 0) {
                // a tile no row keeps: its gradients are zero
                if (key_ok)
                    for (int c = 0; c < 64; c += 4) {
                        *reinterpret_cast<float4 *>(dkrow + c) = make_float4(0.f, 0.f, 0.f, 0.f);
                        *reinterpret_cast<float4 *>(dvrow + c) = make_float4(0.f, 0.f, 0.f, 0.f);
                    }
                continue;
            }
            for (int p = 0; p < np; ++p, ++gp) {
                const int st = gp & 1;
                ok = mbar_wait(bar(B_ST + wg), gp & 1, abort_flag, a.status, a.wait_ns) &&
                     mbar_wait(bar(B_PF + st), (gp >> 1) & 1, abort_flag, a.status, a.wait_ns);
                if (!__all_sync(0xffffffffu, ok)) { ok = false; break; }
                tc_fence_after();
                const float *rw = rows_of(st) + 64 * wg;
                const int4 en = *info_of(st);
                const int j = en.x;
                const float gl = __int_as_float(hk ? en.z : en.y);
                const bool kvis = key_ok && gl != -CUDART_INF_F;
                // first position of this half's rows; in the unit's own block, row r
                // (position pos0 + r) sees the key only when r >= key - pos0
                const int pos0 = s.bs == 64 ? j * 64 : j * 128 + 64 * wg;
                const int lim = (causal && blk == j) ? key - pos0 : -1;
                float x[32], y[32];
                uint32_t pp[16], pd[16];
#pragma unroll
                for (int hf = 0; hf < 2; ++hf) {
                    tmem_ld32(tb + 32 * hf, x);
                    tmem_ld32(tb + 64 + 32 * hf, y);
                    tmem_wait_ld();
                    reg_fence<32>(x);
                    reg_fence<32>(y);
#pragma unroll
                    for (int k4 = 0; k4 < 32; k4 += 4) {
                        const float4 l4 = *reinterpret_cast<const float4 *>(rw + 32 * hf + k4);
                        const float4 d4 = *reinterpret_cast<const float4 *>(rw + 128 + 32 * hf + k4);
                        const float lv[4] = {l4.x, l4.y, l4.z, l4.w}, dvv[4] = {d4.x, d4.y, d4.z, d4.w};
                        float pv[4], dv[4];
#pragma unroll
                        for (int q = 0; q < 4; ++q) {
                            const int r = 32 * hf + k4 + q;
                            const bool vis = kvis && r >= lim;
                            const float p = vis ? ex2(fmaf(x[k4 + q], sc2, gl - lv[q])) : 0.f;
                            pv[q] = p;
                            dv[q] = p * (y[k4 + q] - dvv[q]);
                        }
#pragma unroll
                        for (int q = 0; q < 4; q += 2) {
                            __nv_bfloat162 h1 = __floats2bfloat162_rn(pv[q], pv[q + 1]);
                            __nv_bfloat162 h2 = __floats2bfloat162_rn(dv[q], dv[q + 1]);
                            pp[(k4 + q) >> 1] = *reinterpret_cast<uint32_t *>(&h1);
                            pd[(k4 + q) >> 1] = *reinterpret_cast<uint32_t *>(&h2);
                        }
                    }
                    // rows 32 hf .. 32 hf + 31 -> 16 bf16-pair columns at 16 hf: below
                    // column 32 hf, the first one the second half reads
                    tmem_st16(tb + 16 * hf, pp);
                    tmem_st16(tb + 64 + 16 * hf, pd);
                }
                tmem_wait_st();
                tc_fence_before();
                mbar_arrive(bar(B_EW + wg));
            }
            if (!ok) break;
            // ---- the item's accumulators: this warp's 32 keys x 64 columns ----
            ok = mbar_wait(bar(B_ACC), ni & 1, abort_flag, a.status, a.wait_ns);
            if (!__all_sync(0xffffffffu, ok)) { ok = false; break; }
            tc_fence_after();
            float dv[64], dk[64];
            tmem_ld32(tmem + lane_off + 256 + 64 * wg, dv);
            tmem_ld32(tmem + lane_off + 256 + 64 * wg + 32, dv + 32);
            tmem_ld32(tmem + lane_off + 384 + 64 * wg, dk);
            tmem_ld32(tmem + lane_off + 384 + 64 * wg + 32, dk + 32);
            tmem_wait_ld();
            reg_fence<64>(dv);
            reg_fence<64>(dk);
            tc_fence_before();
            mbar_arrive(bar(B_ACCF));
            ++ni;
            const int ns = a.tsplit[item.x];
            if (ns == 1) {
                if (key_ok)
                    for (int c = 0; c < 64; c += 4) {
                        *reinterpret_cast<float4 *>(dkrow + c) =
                            make_float4(dk[c] * s.scale, dk[c + 1] * s.scale, dk[c + 2] * s.scale, dk[c + 3] * s.scale);
                        *reinterpret_cast<float4 *>(dvrow + c) = make_float4(dv[c], dv[c + 1], dv[c + 2], dv[c + 3]);
                    }
                continue;
            }
            // a split tile: this split's slot, then the region's last split sums the slots in order
            float *slot = a.part + (size_t)(a.tslot[item.x] + item.w) * 2 * 128 * 128;
            float *pk = slot + (size_t)kl * 128 + 64 * wg, *pv = slot + 128 * 128 + (size_t)kl * 128 + 64 * wg;
            for (int c = 0; c < 64; c += 4) {
                *reinterpret_cast<float4 *>(pk + c) = make_float4(dk[c], dk[c + 1], dk[c + 2], dk[c + 3]);
                *reinterpret_cast<float4 *>(pv + c) = make_float4(dv[c], dv[c + 1], dv[c + 2], dv[c + 3]);
            }
            __threadfence();
            __syncwarp();
            int last = 0;
            if (lane == 0) last = atomicAdd(a.rcnt + (size_t)item.x * 8 + ew, 1) == ns - 1;
            last = __shfl_sync(0xffffffffu, last, 0);
            if (!last) continue;
            __threadfence();
            const float *s0 = a.part + (size_t)a.tslot[item.x] * 2 * 128 * 128;
            for (int c = 0; c < 64; c += 4) {
                float4 k4 = make_float4(0.f, 0.f, 0.f, 0.f), v4 = k4;
                for (int sp = 0; sp < ns; ++sp) {
                    const float *q = s0 + (size_t)sp * 2 * 128 * 128 + (size_t)kl * 128 + 64 * wg + c;
                    const float4 a4 = __ldcg(reinterpret_cast<const float4 *>(q));
                    const float4 b4 = __ldcg(reinterpret_cast<const float4 *>(q + 128 * 128));
                    k4.x += a4.x; k4.y += a4.y; k4.z += a4.z; k4.w += a4.w;
                    v4.x += b4.x; v4.y += b4.y; v4.z += b4.z; v4.w += b4.w;
                }
                if (key_ok) {
                    *reinterpret_cast<float4 *>(dkrow + c) =
                        make_float4(k4.x * s.scale, k4.y * s.scale, k4.z * s.scale, k4.w * s.scale);
                    *reinterpret_cast<float4 *>(dvrow + c) = v4;
                }
            }
            if (lane == 0) a.rcnt[(size_t)item.x * 8 + ew] = 0;
        }
    }

    tc_fence_before();
    __syncthreads();
    if (warp == 1) {
        tc_fence_after();
        asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(tmem), "n"(512));
    }
}

}  // namespace

size_t backward_kv_workspace(const Shape &s) { return kv_layout(s).bytes; }

cudaError_t launch_backward_kv(const Shape &s, const void *Q, const void *K, const void *V, const void *dO,
                               const float *D, const float *lse2, const int32_t *idx, const float *score,
                               const int32_t *count, float *dK, float *dV, void *work, int *rcnt,
                               unsigned *status, cudaStream_t st) {
    const KvLayout L = kv_layout(s);
    unsigned char *w = static_cast<unsigned char *>(work);
    InvArgs ia{};
    ia.s = s;
    ia.idx = idx;
    ia.count = count;
    ia.score = score;
    ia.KT = L.KT;
    ia.bpt = L.bpt;
    ia.tiles = L.tiles;
    ia.tcnt = reinterpret_cast<int *>(w + L.off_tcnt);
    ia.toff = reinterpret_cast<int *>(w + L.off_toff);
    ia.tsplit = reinterpret_cast<int *>(w + L.off_tsplit);
    ia.tslot = reinterpret_cast<int *>(w + L.off_tslot);
    ia.ioff = reinterpret_cast<int *>(w + L.off_ioff);
    ia.tot = reinterpret_cast<int *>(w + L.off_tot);
    ia.order = reinterpret_cast<int *>(w + L.off_order);
    ia.ent = reinterpret_cast<int4 *>(w + L.off_ent);
    ia.items = reinterpret_cast<int4 *>(w + L.off_items);
    const unsigned wgrid = (unsigned)(((size_t)L.tiles * 32 + 255) / 256);
    inv_kernel<<<wgrid, 256, 0, st>>>(ia, 0);
    note_launch();
    inv_scan_kernel<<<1, 1024, 0, st>>>(ia);
    note_launch();
    inv_kernel<<<wgrid, 256, 0, st>>>(ia, 1);
    note_launch();
    inv_order_kernel<<<(unsigned)(s.B * s.Hkv), 1024, 0, st>>>(ia);
    note_launch();
    cudaError_t e = cudaGetLastError();
    if (e != cudaSuccess) return e;

    cudaFuncAttributes fa;
    if ((e = cudaFuncGetAttributes(&fa, bwd_kv_kernel)) != cudaSuccess) return e;
    if (fa.numRegs != kRegsLaunchKV) return cudaErrorInvalidDeviceFunction;
    CUtensorMap mq, mk, mv, mdo;
    const uint64_t qrows = (uint64_t)s.B * s.Hq * s.N, krows = (uint64_t)s.B * s.Hkv * s.N;
    if (!make_map_d128(&mq, Q, qrows, 64) || !make_map_d128(&mk, K, krows, 64) || !make_map_d128(&mv, V, krows, 64) ||
        !make_map_d128(&mdo, dO, qrows, 64))
        return cudaErrorInvalidValue;
    if ((reinterpret_cast<uintptr_t>(D) | reinterpret_cast<uintptr_t>(lse2)) & 15) return cudaErrorInvalidValue;
    KvArgs a{};
    a.s = s;
    a.D = D;
    a.lse2 = lse2;
    a.dK = dK;
    a.dV = dV;
    a.tsplit = ia.tsplit;
    a.tslot = ia.tslot;
    a.tot = ia.tot;
    a.order = ia.order;
    a.rcnt = rcnt;
    a.ent = ia.ent;
    a.items = ia.items;
    a.part = reinterpret_cast<float *>(w + L.off_part);
    a.status = status;
    a.KT = L.KT;
    a.MT = L.MT;
    a.Npad = s.nb * s.bs;
    a.wait_ns = kWaitNs;
    const int sms = sm_count();
    if (sms <= 0) return cudaErrorNoDevice;
    if ((e = cudaFuncSetAttribute(bwd_kv_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)kSmemKV)) !=
        cudaSuccess)
        return e;
    bwd_kv_kernel<<<(unsigned)sms, kThreadsKV, kSmemKV, st>>>(mq, mk, mv, mdo, a);
    note_launch();
    return cudaGetLastError();
}

}  // namespace sa
