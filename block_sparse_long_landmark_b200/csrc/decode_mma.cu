// decode_mma.cu -- block-sparse decode for bf16, d = 128, block 64: a TMA
// ring of kept K/V blocks feeding warp-level tensor-core tiles.
//
// [HiLS] "Ключевые факты": sparse access to a KV cache kept whole (so do the
// Latent Sparse Attention post's last section and [SAS]'s selected blocks);
// gated mode adds [SAS]'s log-sigmoid gate inside the softmax; hierarchical
// mode ([HiLS] opening section) gives every kept block its own softmax and
// weights the block outputs by softmax_b(s_b).
//
// The step is HBM-bound: every kept block is 16 KB of K and 16 KB of V read
// once.  The work is cut into items (unit, split): up to `bps` consecutive
// entries of one (batch, kv-head) list.  The kernel is persistent: each CTA
// takes items blockIdx.x, blockIdx.x + grid, ... and its warp 0 streams all
// their kept blocks, item after item, with cp.async.bulk.tensor (128-byte
// swizzle) through one shared-memory ring, so the ring stays full across item
// boundaries.  Each stage carries a small record (block, gate, item, first /
// last block of the consumer warp in the item).  Consumer warp w takes the
// CTA's stream positions w, w + kNW, ... and computes, with mma.sync
// m16n8k16 bf16 tiles,
//   S[16 x 64] = q[16 x 128] K_b^T     (rows = the group's query heads, padded)
//   O[16 x 128] += P[16 x 64] V_b      (P straight from S's registers)
// keeping an online softmax; at its last block of an item it leaves (max,
// sum, acc) per head in the item's partial record, and the producer marks
// the records of warps that got no block of an item empty.  Every record
// written is counted towards its unit (after a fence), so the merge launch
// that follows, started early, combines each unit's kNW x splits records as
// soon as the count is complete, while other units still stream.  The launch
// may start early too (programmatic dependent launch) and waits for the
// lists on the device: for the whole selection launch, or, in a decode step,
// for each item's own unit (the selection publishes each list with the
// step's epoch), so items of early units stream while later ones are chosen.
#include <cuda.h>
#include <cudaTypedefs.h>
#include <math_constants.h>

#include <cstdlib>
#include <cstring>
#include <mutex>

#include "bounds.cuh"
#include "common.cuh"

namespace sa {
namespace {

constexpr int kNW = 2;                          // consumer warps
constexpr int kThreadsD = 32 * (kNW + 1);
constexpr int kNST = 2;                         // ring stages
// Stream position gi goes to stage gi % kNST and to consumer warp gi % kNW.
// With kNST a multiple of kNW every stage has a single consumer warp, which
// waits on its phases strictly in order; a shared stage would let one warp
// wait on a parity two phases ahead of the barrier and pass before its data
// landed.
static_assert(kNST % kNW == 0, "each ring stage must belong to one consumer warp");
constexpr uint32_t kHalf = 64 * 128;            // one 64-row x 64-col bf16 box (8 KB)
constexpr uint32_t kBlockBytes = 2 * kHalf;     // 64 x 128 bf16 (16 KB)
constexpr uint32_t kStageBytes = 2 * kBlockBytes;  // K + V
constexpr uint32_t kBarOffD = kNST * kStageBytes;
constexpr uint32_t kMetaOffD = kBarOffD + 64;   // [kNST] int4 stage records
constexpr uint32_t kSmemD = kMetaOffD + 16 * kNST + 1024;
constexpr int kMaxBps = 64;
constexpr int kRec = 130;                       // floats per head in a partial record: max, sum, acc[128]
constexpr unsigned long long kWaitNsD = 2000000000ull;
enum { F_FIRST = 1, F_LAST = 2, F_END = 4 };

struct DmArgs {
    Shape s;
    const __nv_bfloat16 *q;
    const int32_t *idx;
    const float *score;
    const int32_t *count;
    unsigned *status;
    float *part;                // [units][S][kNW][heads_per][kRec]
    unsigned *ucnt;             // [units] records written (the merge launch waits on it, then clears it)
    const unsigned *ready;      // [units] epoch of the unit's latest list, or null (wait for the whole launch)
    unsigned epoch;
    int S, bps, items;
};

__device__ __forceinline__ uint32_t su32(const void *p) { return static_cast<uint32_t>(__cvta_generic_to_shared(p)); }
__device__ __forceinline__ bool try_wait(uint32_t bar, uint32_t parity) {
    uint32_t ok;
    asm volatile(
        "{\n\t.reg .pred p;\n\tmbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2;\n\tselp.u32 %0, 1, 0, p;\n\t}"
        : "=r"(ok) : "r"(bar), "r"(parity) : "memory");
    return ok != 0;
}
__device__ __forceinline__ unsigned long long now_ns() {
    unsigned long long t;
    asm volatile("mov.u64 %0, %%globaltimer;" : "=l"(t));
    return t;
}
__device__ __forceinline__ bool wait_bar(uint32_t bar, uint32_t parity, volatile int *abort_flag, unsigned *status) {
    if (try_wait(bar, parity)) return true;
    const unsigned long long t0 = now_ns();
    for (uint32_t it = 0;; ++it) {
        if (try_wait(bar, parity)) return true;
        if ((it & 63) == 63) {
            if (*abort_flag) return false;
            if (now_ns() - t0 > kWaitNsD) {
                *abort_flag = 1;
                set_status(status, kStatusTimeout);
                return false;
            }
        }
    }
}
__device__ __forceinline__ void ldsm_x4(uint32_t addr, uint32_t &r0, uint32_t &r1, uint32_t &r2, uint32_t &r3) {
    asm volatile("ldmatrix.sync.aligned.m8n8.x4.shared.b16 {%0,%1,%2,%3}, [%4];"
                 : "=r"(r0), "=r"(r1), "=r"(r2), "=r"(r3) : "r"(addr));
}
__device__ __forceinline__ void ldsm_x4_t(uint32_t addr, uint32_t &r0, uint32_t &r1, uint32_t &r2, uint32_t &r3) {
    asm volatile("ldmatrix.sync.aligned.m8n8.x4.trans.shared.b16 {%0,%1,%2,%3}, [%4];"
                 : "=r"(r0), "=r"(r1), "=r"(r2), "=r"(r3) : "r"(addr));
}
__device__ __forceinline__ void mma16816(float *c, uint32_t a0, uint32_t a1, uint32_t a2, uint32_t a3, uint32_t b0,
                                         uint32_t b1) {
    asm volatile(
        "mma.sync.aligned.m16n8k16.row.col.f32.bf16.bf16.f32 {%0,%1,%2,%3}, {%4,%5,%6,%7}, {%8,%9}, "
        "{%0,%1,%2,%3};"
        : "+f"(c[0]), "+f"(c[1]), "+f"(c[2]), "+f"(c[3])
        : "r"(a0), "r"(a1), "r"(a2), "r"(a3), "r"(b0), "r"(b1));
}
__device__ __forceinline__ float ex2f(float x) {
    float y;
    asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
    return y;
}
__device__ __forceinline__ uint32_t pack_bf16(float lo, float hi) {
    __nv_bfloat162 h = __floats2bfloat162_rn(lo, hi);
    return *reinterpret_cast<uint32_t *>(&h);
}
// byte offset of (row, 16-byte unit u) in a 64-row box with 128-byte swizzle
__device__ __forceinline__ uint32_t swz(int row, int u) { return row * 128 + ((u ^ (row & 7)) << 4); }

__device__ __forceinline__ void pdl_wait() { asm volatile("griddepcontrol.wait;" ::: "memory"); }
__device__ __forceinline__ void pdl_launch() { asm volatile("griddepcontrol.launch_dependents;" ::: "memory"); }

// Counts n records of unit u as written (the warp's own writes fenced first).
__device__ __forceinline__ void count_records(const DmArgs &a, int u, int n) {
    __threadfence();
    __syncwarp();
    if ((threadIdx.x & 31) == 0) atomicAdd(a.ucnt + u, (unsigned)n);
    __syncwarp();
}

__global__ void __launch_bounds__(kThreadsD, 3)
decode_mma_kernel(const __grid_constant__ CUtensorMap tmK, const __grid_constant__ CUtensorMap tmV, DmArgs a) {
    constexpr float kLog2e = 1.4426950408889634f;
    const Shape &s = a.s;
    extern __shared__ unsigned char dsm_raw[];
    unsigned char *sm = reinterpret_cast<unsigned char *>((reinterpret_cast<uintptr_t>(dsm_raw) + 1023) &
                                                          ~uintptr_t(1023));
    const uint32_t sb = su32(sm);
    uint64_t *bars = reinterpret_cast<uint64_t *>(sm + kBarOffD);      // full[kNST], empty[kNST]
    volatile int *abort_flag = reinterpret_cast<volatile int *>(sm + kBarOffD + 8 * 2 * kNST);
    int4 *meta = reinterpret_cast<int4 *>(sm + kMetaOffD);
    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const bool hier = s.flags & SA_HIER;
    const bool perq = s.flags & SA_SELECT_PER_QHEAD;
    const int HP = s.heads_per;

    if (tid == 0) {
        for (int i = 0; i < kNST; ++i) {
            asm volatile("mbarrier.init.shared::cta.b64 [%0], 1;" ::"r"(su32(&bars[i])));
            asm volatile("mbarrier.init.shared::cta.b64 [%0], 1;" ::"r"(su32(&bars[kNST + i])));
        }
        *abort_flag = 0;
        asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
    }
    __syncthreads();
    pdl_launch();
    if (!a.ready) pdl_wait();   // the lists come from the launch before this one

    if (warp == 0) {
        // ---- producer: every item's kept blocks, in order ------------------
        int gi = 0, issued = 0;
        bool ok = true;
        // the next item's count and list entries are loaded one item ahead
        // (entries c0 + lane + 32 r of the list row, read whatever the count;
        // the row has cap entries, so every read stays inside it)
        int p_cnt = 0, p_il[2] = {-1, -1}, p_ilm[2] = {-1, -1};
        float p_sl[2] = {0.f, 0.f};
        auto preload = [&](int item) {
            if (item >= a.items) return;
            const int u = item / a.S, c0 = (item % a.S) * a.bps;
            if (a.ready) {
                // this unit's list of this step: bounded wait on its epoch
                int gave_up = 0;
                if (lane == 0) {
                    const unsigned long long t0 = now_ns();
                    unsigned v;
                    for (;;) {
                        asm volatile("ld.acquire.gpu.global.u32 %0, [%1];" : "=r"(v) : "l"(a.ready + u) : "memory");
                        if (v == a.epoch) break;
                        if (*abort_flag || now_ns() - t0 > kWaitNsD) {
                            if (!*abort_flag) set_status(a.status, kStatusTimeout);
                            *abort_flag = 1;
                            gave_up = 1;
                            break;
                        }
                        __nanosleep(128);
                    }
                }
                if (__shfl_sync(0xffffffffu, gave_up, 0)) {
                    p_cnt = 0;
                    return;
                }
                // every lane reads the list below: each takes the acquire itself
                unsigned v;
                asm volatile("ld.acquire.gpu.global.u32 %0, [%1];" : "=r"(v) : "l"(a.ready + u) : "memory");
                (void)v;
            }
            p_cnt = a.count[u];
#pragma unroll
            for (int r = 0; r < 2; ++r) {
                const int c = c0 + 32 * r + lane;
                const bool in = 32 * r < a.bps && c < s.cap;
                p_il[r] = in ? a.idx[(size_t)u * s.cap + c] : -1;
                p_ilm[r] = in && c > 0 ? a.idx[(size_t)u * s.cap + c - 1] : -1;
                p_sl[r] = in ? a.score[(size_t)u * s.cap + c] : 0.f;
            }
        };
        preload(blockIdx.x);
        for (int item = blockIdx.x; ok && item < a.items; item += gridDim.x) {
            const int u = item / a.S, sp = item % a.S;
            const int hs = u % s.Hsel, b = u / s.Hsel;
            const int g = perq ? hs / s.G : hs;
            const int cnt = max(0, min(p_cnt, s.cap));
            const int c_il[2] = {p_il[0], p_il[1]}, c_ilm[2] = {p_ilm[0], p_ilm[1]};
            const float c_sl[2] = {p_sl[0], p_sl[1]};
            const int local = (seq_n(s, b) - 1) / 64;
            const int c0 = sp * a.bps;
            const int n = max(0, min(cnt, c0 + a.bps) - c0);
            const int kvbase = (b * s.Hkv + g) * s.N;
            const float s_loc = cnt > 0 ? a.score[(size_t)u * s.cap + cnt - 1] : 0.f;
            const int gi0 = gi;
            for (int r = 0; ok && r < n; r += 32) {
                // lane-parallel: block id and gate of entries r + lane
                const int ri = r >> 5;
                int myblk = -1;
                float mygate = 0.f;
                if (r + lane < n) {
                    const int c = c0 + r + lane;
                    const int blk = c_il[ri];
                    const bool good = blk >= 0 && blk <= local && (c == 0 || c_ilm[ri] < blk);
                    if (!good) set_status(a.status, kStatusBadIndex);
                    myblk = good ? blk : -1;
                    const bool forced = (blk == local && (s.flags & SA_LOCAL)) || (blk == 0 && (s.flags & SA_SINK));
                    // gated: log2-unit gate; hierarchical: log2-unit retrieval score
                    mygate = hier ? c_sl[ri] * kLog2e
                                  : (((s.flags & SA_GATE) && !forced) ? log_sigmoid(c_sl[ri] - s_loc) * kLog2e : 0.f);
                }
            const int m = min(32, n - r);
                for (int j = 0; j < m; ++j) {
                    const int blk = __shfl_sync(0xffffffffu, myblk, j);
                    const float gate = __shfl_sync(0xffffffffu, mygate, j);
                    const int c = r + j;
                    if (lane == 0) {
                        const int st = gi % kNST;
                        if (gi >= kNST && !wait_bar(su32(&bars[kNST + st]), ((gi / kNST) - 1) & 1, abort_flag, a.status))
                            ok = false;
                        if (ok) {
                            meta[st] = make_int4(blk, __float_as_int(gate), item,
                                                 (c < kNW ? F_FIRST : 0) | (c + kNW >= n ? F_LAST : 0));
                            const uint32_t full = su32(&bars[st]);
                            asm volatile("mbarrier.arrive.expect_tx.shared::cta.b64 _, [%0], %1;" ::"r"(full),
                                         "r"(kStageBytes) : "memory");
                            const int y = kvbase + max(0, blk) * 64;
                            SA_CHECK_START(a.status, max(0, blk) * 64, s.N);
                            const uint32_t dst = sb + st * kStageBytes;
#pragma unroll
                            for (int ch = 0; ch < 2; ++ch) {
                                asm volatile(
                                    "cp.async.bulk.tensor.2d.shared::cluster.global.mbarrier::complete_tx::bytes [%0], "
                                    "[%1, {%3, %4}], [%2];" ::"r"(dst + ch * kHalf),
                                    "l"(reinterpret_cast<uint64_t>(&tmK)), "r"(full), "r"(64 * ch), "r"(y)
                                    : "memory");
                                asm volatile(
                                    "cp.async.bulk.tensor.2d.shared::cluster.global.mbarrier::complete_tx::bytes [%0], "
                                    "[%1, {%3, %4}], [%2];" ::"r"(dst + kBlockBytes + ch * kHalf),
                                    "l"(reinterpret_cast<uint64_t>(&tmV)), "r"(full), "r"(64 * ch), "r"(y)
                                    : "memory");
                            }
                            issued = gi + 1;
                        }
                    }
                    ok = __shfl_sync(0xffffffffu, ok, 0);
                    if (!ok) break;
                    ++gi;
                }
            }
            if (!ok) break;
            // the next item's list, while this item's last blocks are in flight
            preload(item + gridDim.x);
            if (n < kNW) {
                // consumer warps that get no block of this item: empty records
                int nempty = 0;
                for (int w = 0; w < kNW; ++w) {
                    bool covered = false;
                    for (int c = 0; c < n; ++c) covered |= (gi0 + c) % kNW == w;
                    if (covered) continue;
                    ++nempty;
                    float *rec = a.part + (((size_t)item * kNW + w) * HP) * kRec;
                    for (int hh = lane; hh < HP; hh += 32) rec[(size_t)hh * kRec] = -CUDART_INF_F;
                }
                count_records(a, u, nempty);
            }
        }
        // one end record per consumer warp (no data: a plain arrival completes the stage)
        for (int w = 0; ok && w < kNW; ++w, ++gi) {
            if (lane == 0) {
                const int st = gi % kNST;
                if (gi >= kNST && !wait_bar(su32(&bars[kNST + st]), ((gi / kNST) - 1) & 1, abort_flag, a.status))
                    ok = false;
                if (ok) {
                    meta[st] = make_int4(-1, 0, -1, F_END);
                    asm volatile("mbarrier.arrive.shared::cta.b64 _, [%0];" ::"r"(su32(&bars[st])) : "memory");
                }
            }
            ok = __shfl_sync(0xffffffffu, ok, 0);
        }
        if (lane == 0 && *abort_flag) {
            // let the copies in flight land before the CTA exits
            volatile int never = 0;
            for (int li = max(0, issued - kNST); li < issued; ++li)
                wait_bar(su32(&bars[li % kNST]), (li / kNST) & 1, &never, a.status);
        }
        return;
    }

    // ---- consumer warps ------------------------------------------------------
    const int cw = warp - 1;
    const int gq = lane >> 2, tq = lane & 3;
    const float qk_scale = s.scale * kLog2e;
    float m_r[2] = {-CUDART_INF_F, -CUDART_INF_F}, l_r[2] = {0.f, 0.f};
    float oacc[16][4];
    uint32_t qa[8][4];
    int nseq = 0;
    for (int gi = cw;; gi += kNW) {
        const int st = gi % kNST;
        const bool ok = wait_bar(su32(&bars[st]), (gi / kNST) & 1, abort_flag, a.status);
        if (!__all_sync(0xffffffffu, ok)) break;
        const int4 md = meta[st];
        if (md.w & F_END) break;
        const int item = md.z, u = item / a.S;
        const int hs = u % s.Hsel, b = u / s.Hsel;
        const int h0 = perq ? hs : hs * s.G;
        if (md.w & F_FIRST) {
            // a new item for this warp: its query fragments and a fresh state
            nseq = seq_n(s, b);
#pragma unroll
            for (int ks = 0; ks < 8; ++ks) {
#pragma unroll
                for (int rr = 0; rr < 2; ++rr) {
                    const int row = gq + 8 * rr;
                    const bool valid = row < HP;
                    const __nv_bfloat16 *qr =
                        a.q + ((size_t)b * s.Hq + h0 + (valid ? row : 0)) * 128 + 16 * ks + 2 * tq;
                    qa[ks][rr] = valid ? *reinterpret_cast<const uint32_t *>(qr) : 0u;           // a0 / a1
                    qa[ks][2 + rr] = valid ? *reinterpret_cast<const uint32_t *>(qr + 8) : 0u;   // a2 / a3
                }
            }
            m_r[0] = m_r[1] = -CUDART_INF_F;
            l_r[0] = l_r[1] = 0.f;
#pragma unroll
            for (int i = 0; i < 16; ++i) oacc[i][0] = oacc[i][1] = oacc[i][2] = oacc[i][3] = 0.f;
        }
        const uint32_t kb = sb + st * kStageBytes, vb = kb + kBlockBytes;
        const int blk = md.x;
        const int nk = blk < 0 ? 0 : min(64, nseq - blk * 64);
        // S = q K^T over 8 key n-tiles
        float sacc[8][4];
#pragma unroll
        for (int nt = 0; nt < 8; ++nt) {
            sacc[nt][0] = sacc[nt][1] = sacc[nt][2] = sacc[nt][3] = 0.f;
            const int key = 8 * nt + (lane & 7);
#pragma unroll
            for (int pch = 0; pch < 4; ++pch) {
                const int dim0 = 32 * pch + 8 * (lane >> 3);
                uint32_t r0, r1, r2, r3;
                ldsm_x4(kb + (dim0 >> 6) * kHalf + swz(key, (dim0 & 63) >> 3), r0, r1, r2, r3);
                mma16816(sacc[nt], qa[2 * pch][0], qa[2 * pch][1], qa[2 * pch][2], qa[2 * pch][3], r0, r1);
                mma16816(sacc[nt], qa[2 * pch + 1][0], qa[2 * pch + 1][1], qa[2 * pch + 1][2], qa[2 * pch + 1][3],
                         r2, r3);
            }
        }
        // logits (log2 units), masks, block max per row
        const float gl = __int_as_float(md.y);
        float bm[2] = {-CUDART_INF_F, -CUDART_INF_F};
#pragma unroll
        for (int nt = 0; nt < 8; ++nt)
#pragma unroll
            for (int e = 0; e < 4; ++e) {
                const int key = 8 * nt + 2 * tq + (e & 1);
                const float z = key < nk ? fmaf(sacc[nt][e], qk_scale, hier ? 0.f : gl) : -CUDART_INF_F;
                sacc[nt][e] = z;
                bm[e >> 1] = fmaxf(bm[e >> 1], z);
            }
#pragma unroll
        for (int rr = 0; rr < 2; ++rr) {
            bm[rr] = fmaxf(bm[rr], __shfl_xor_sync(0xffffffffu, bm[rr], 1));
            bm[rr] = fmaxf(bm[rr], __shfl_xor_sync(0xffffffffu, bm[rr], 2));
        }
        float corr[2], ref[2], fsc[2] = {1.f, 1.f};
        if (!hier) {
#pragma unroll
            for (int rr = 0; rr < 2; ++rr) {
                const float nm = fmaxf(m_r[rr], bm[rr]);
                corr[rr] = m_r[rr] == -CUDART_INF_F ? 0.f : ex2f(m_r[rr] - nm);
                m_r[rr] = nm;
                ref[rr] = nm == -CUDART_INF_F ? 0.f : nm;
            }
        } else {
#pragma unroll
            for (int rr = 0; rr < 2; ++rr) ref[rr] = bm[rr] == -CUDART_INF_F ? 0.f : bm[rr];
        }
        float ps[2] = {0.f, 0.f};
#pragma unroll
        for (int nt = 0; nt < 8; ++nt)
#pragma unroll
            for (int e = 0; e < 4; ++e) {
                const float p = ex2f(sacc[nt][e] - ref[e >> 1]);
                sacc[nt][e] = p;
                ps[e >> 1] += p;
            }
        if (!hier) {
#pragma unroll
            for (int rr = 0; rr < 2; ++rr) l_r[rr] = l_r[rr] * corr[rr] + ps[rr];   // lane-partial sums
        } else {
#pragma unroll
            for (int rr = 0; rr < 2; ++rr) {
                float lb = ps[rr];
                lb += __shfl_xor_sync(0xffffffffu, lb, 1);
                lb += __shfl_xor_sync(0xffffffffu, lb, 2);
                if (lb > 0.f) {
                    const float nM = fmaxf(m_r[rr], gl);
                    corr[rr] = m_r[rr] == -CUDART_INF_F ? 0.f : ex2f(m_r[rr] - nM);
                    const float wb = ex2f(gl - nM);
                    l_r[rr] = l_r[rr] * corr[rr] + wb;      // full (not lane-partial) weight sum
                    m_r[rr] = nM;
                    fsc[rr] = wb / lb;
                } else {
                    corr[rr] = 1.f;
                    fsc[rr] = 0.f;
                }
            }
        }
#pragma unroll
        for (int nd = 0; nd < 16; ++nd) {
            oacc[nd][0] *= corr[0];
            oacc[nd][1] *= corr[0];
            oacc[nd][2] *= corr[1];
            oacc[nd][3] *= corr[1];
        }
        // O += P V : 4 key k-steps x 16 dim n-tiles
#pragma unroll
        for (int kk = 0; kk < 4; ++kk) {
            const uint32_t pa0 = pack_bf16(sacc[2 * kk][0] * fsc[0], sacc[2 * kk][1] * fsc[0]);
            const uint32_t pa1 = pack_bf16(sacc[2 * kk][2] * fsc[1], sacc[2 * kk][3] * fsc[1]);
            const uint32_t pa2 = pack_bf16(sacc[2 * kk + 1][0] * fsc[0], sacc[2 * kk + 1][1] * fsc[0]);
            const uint32_t pa3 = pack_bf16(sacc[2 * kk + 1][2] * fsc[1], sacc[2 * kk + 1][3] * fsc[1]);
            const int key = 16 * kk + 8 * ((lane >> 3) & 1) + (lane & 7);
#pragma unroll
            for (int np = 0; np < 8; ++np) {
                const int dim0 = 16 * np + 8 * (lane >> 4);
                uint32_t r0, r1, r2, r3;
                ldsm_x4_t(vb + (dim0 >> 6) * kHalf + swz(key, (dim0 & 63) >> 3), r0, r1, r2, r3);
                mma16816(oacc[2 * np], pa0, pa1, pa2, pa3, r0, r1);
                mma16816(oacc[2 * np + 1], pa0, pa1, pa2, pa3, r2, r3);
            }
        }
        __syncwarp();
        if (lane == 0) asm volatile("mbarrier.arrive.shared::cta.b64 _, [%0];" ::"r"(su32(&bars[kNST + st])) : "memory");
        if (md.w & F_LAST) {
            // this warp's state for the item -> its partial record
            float lr[2] = {l_r[0], l_r[1]};
            if (!hier) {
#pragma unroll
                for (int rr = 0; rr < 2; ++rr) {
                    lr[rr] += __shfl_xor_sync(0xffffffffu, lr[rr], 1);
                    lr[rr] += __shfl_xor_sync(0xffffffffu, lr[rr], 2);
                }
            }
            float *rec = a.part + (((size_t)item * kNW + cw) * HP) * kRec;
#pragma unroll
            for (int rr = 0; rr < 2; ++rr) {
                const int hh = gq + 8 * rr;
                if (hh >= HP) continue;
                float *rh = rec + (size_t)hh * kRec;
                if (tq == 0) {
                    rh[0] = m_r[rr];
                    rh[1] = lr[rr];
                }
#pragma unroll
                for (int nd = 0; nd < 16; ++nd)
                    *reinterpret_cast<float2 *>(rh + 2 + 8 * nd + 2 * tq) = make_float2(oacc[nd][2 * rr], oacc[nd][2 * rr + 1]);
            }
            count_records(a, u, 1);
        }
    }
}

PFN_cuTensorMapEncodeTiled_v12000 g_enc = nullptr;
std::once_flag g_enc_once;

}  // namespace

bool decode_mma_supported(const Shape &s) {
    if (!(s.dtype == SA_BF16 && s.d == 128 && s.bs == 64 && s.heads_per <= 16)) return false;
    const char *e = getenv("SPARSE_ATTN_DECODE_PATH");
    return !(e && strcmp(e, "simt") == 0);
}

int decode_mma_records(int S) { return S * kNW; }

size_t decode_mma_partial_bytes(const Shape &s, int S) {
    return (((size_t)s.B * s.Hsel * S * kNW * s.heads_per * kRec * sizeof(float)) + 255) & ~(size_t)255;
}


// Items as large as possible (fewer partial records to write and merge) while
// the grid still fills three quarters of the slots (three CTAs per SM), with
// k items per CTA and grid = ceil(items / k) so every CTA gets k or k - 1.
// The split count (and with it the workspace) is fixed from the 148 SMs of a
// B200; the grid follows the device.
static int dm_grid(long long items, int sms) {
    const long long slots = 3LL * max(1, sms);
    const long long k = (items + slots - 1) / slots;
    return (int)((items + k - 1) / k);
}

void decode_mma_geometry(const Shape &s, int &S, int &bps) {
    const int units = s.B * s.Hsel;
    for (int want = min(s.cap, kMaxBps);; --want) {
        S = (s.cap + want - 1) / want;
        bps = (s.cap + S - 1) / S;
        S = (s.cap + bps - 1) / bps;
        if (want <= 2 || 4 * dm_grid((long long)units * S, 148) >= 3 * 3 * 148) break;
    }
}

cudaError_t launch_decode_mma(const Shape &s, const void *q, const void *K, const void *V, const int32_t *idx,
                              const float *score, const int32_t *count, unsigned *status, unsigned *ucnt,
                              float *part, cudaStream_t st, int &R_out, const unsigned *ready, unsigned epoch) {
    std::call_once(g_enc_once, [] {
        void *fn = nullptr;
        cudaDriverEntryPointQueryResult qr;
        if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &fn, cudaEnableDefault, &qr) == cudaSuccess &&
            qr == cudaDriverEntryPointSuccess)
            g_enc = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(fn);
    });
    if (!g_enc) return cudaErrorNotSupported;
    CUtensorMap mk, mv;
    const cuuint64_t rows = (cuuint64_t)s.B * s.Hkv * s.N;
    cuuint64_t dims[2] = {128, rows};
    cuuint64_t strides[1] = {256};
    cuuint32_t box[2] = {64, 64};
    cuuint32_t estr[2] = {1, 1};
    if (g_enc(&mk, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, const_cast<void *>(K), dims, strides, box, estr,
              CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
              CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) != CUDA_SUCCESS ||
        g_enc(&mv, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, const_cast<void *>(V), dims, strides, box, estr,
              CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
              CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) != CUDA_SUCCESS)
        return cudaErrorInvalidValue;
    DmArgs a{};
    a.s = s;
    a.q = (const __nv_bfloat16 *)q;
    a.idx = idx;
    a.score = score;
    a.count = count;
    a.status = status;
    a.part = part;
    a.ucnt = ucnt;
    a.ready = ready;
    a.epoch = epoch;
    decode_mma_geometry(s, a.S, a.bps);
    a.items = s.B * s.Hsel * a.S;
    const int grid = dm_grid(a.items, sm_count());
    R_out = decode_mma_records(a.S);
    cudaError_t e = cudaFuncSetAttribute(decode_mma_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)kSmemD);
    if (e != cudaSuccess) return e;
    e = launch_pdl(decode_mma_kernel, dim3((unsigned)grid), dim3(kThreadsD), kSmemD, st, mk, mv, a);
    note_launch();
    return e != cudaSuccess ? e : cudaGetLastError();
}

}  // namespace sa
