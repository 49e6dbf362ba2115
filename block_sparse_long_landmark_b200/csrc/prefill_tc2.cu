// prefill_tc2.cu -- persistent tensor-core block-sparse prefill (gated, plain
// or hierarchical) for bf16, d = 128, block 64 or 128, query groups of at
// least 256 rows.
//
// Computes what prefill_tc.cu computes ([SAS] "Ключевые факты" / "Как это
// применить": blockwise softmax attention over the kept blocks only, the
// selector's gate log_sigmoid(s_b - s_local) added to the logits of selected
// blocks, forced sink / local blocks gated by 0), with a layout built for
// one CTA per SM:
//
//   * a work unit is 256 query rows of one (batch, kv-head, block): the four
//     query heads of a block-64 tile or two heads of a block-128 tile, all of
//     which share one kept list, so each K/V key tile is loaded once for
//     256 rows;
//   * the unit is two M=128 Q tiles, each with its own softmax warpgroup,
//     S buffer and O accumulator in tensor memory (4 x 128 columns = all
//     512).  While one warpgroup turns S into P, the tensor core runs the
//     other tile's PV and QK, so the two warpgroups take turns on it;
//   * key tiles are 128 keys (two kept blocks of 64, or one of 128), which
//     halves the per-tile hand-off cost against 64-key tiles;
//   * the grid is one CTA per SM, each looping over units: the next unit's
//     list and Q tiles load while the current one runs, and a warpgroup's
//     epilogue overlaps the other's last tile.
//
// Warp roles (12 warps):
//   warp 0      loads each unit's list into shared memory (all lanes), then
//               issues the TMA loads: Q tiles, K and V key tiles (2-stage rings)
//   warp 1      TMEM owner and MMA issuer: the warp runs the schedule in
//               lockstep, one elected lane issues each tcgen05.mma
//   warps 2-3   idle
//   warps 4-7   softmax for Q tile 0, warps 8-11 for Q tile 1; thread = row
// Registers: launched at 168; the first warpgroup drops to 56 and the two
// softmax warpgroups rise to 224: 128 x 56 + 256 x 224 = 384 x 168.
//
// Per Q tile q and key tile g the MMA warp issues, in this order,
//   O_q += P_q(g-1) V_(g-1)   then   S_q = Q_q K_g^T
// (P_q is written over the first 64 columns of S_q and read from TMEM; it is
// handed over in four 32-key quarters, so the PV of one quarter runs while the
// softmax exponentiates the next), so
// when S_q(g) is ready, the PV before it has completed too: the lazy O
// rescale (when a row max grows by more than 2^8) never waits on the tensor
// core.
//
// Hierarchical mode ([HiLS]: each kept block gets its own softmax and the
// blocks are mixed by softmax_b(s_b) of their retrieval scores) uses the same
// pipeline: per block, P = 2^(x - max_b) * 2^(s_b - M) / l_b with M the list's
// largest retrieval score, so O needs no rescaling; all of a tile's
// exponentials are taken before its first quarter is handed over, since the
// weights need each block's sum.
//
// Every mbarrier wait is bounded; on expiry the CTA records kStatusTimeout,
// stops, lets its copies land, frees TMEM and exits.
#include <math_constants.h>

#include <cstdlib>
#include <cstring>

#include "bounds.cuh"
#include "common.cuh"
#include "tc_ptx.cuh"

namespace sa {
namespace {

using namespace tc;

constexpr int kThreads2 = 384;
constexpr int kRegsLaunch2 = 168, kRegsLow2 = 56, kRegsHigh2 = 224;
static_assert(128 * kRegsLow2 + 256 * kRegsHigh2 <= kThreads2 * kRegsLaunch2, "register split");
constexpr int kRows = 256;                          // query rows per unit
constexpr uint32_t kChunk2 = 128 * 128;             // 128 rows x 64 bf16 (one swizzle atom wide)
constexpr uint32_t kTile2 = 2 * kChunk2;            // 128 rows x 128 bf16
constexpr int kStages2 = 2;
constexpr uint32_t kQOff2 = 0;                      // Q tiles 0 and 1
constexpr uint32_t kKOff2 = 2 * kTile2;             // K ring
constexpr uint32_t kVOff2 = kKOff2 + kStages2 * kTile2;
constexpr uint32_t kBarOff2 = kVOff2 + kStages2 * kTile2;
constexpr int kMaxList2 = 258;
constexpr int kGateRows = 4;                        // per-head gate rows (lists per query head)
// [2 slots] blk[kMaxList2], gate[kGateRows][kMaxList2]
constexpr uint32_t kListOff2 = kBarOff2 + 512;
constexpr uint32_t kListBytes = 4 * kMaxList2 * (1 + kGateRows);
// per-query-head lists: the unit's entries before they are merged (blk, gate, head, first)
constexpr uint32_t kMergeOff2 = kListOff2 + 2 * kListBytes;
constexpr uint32_t kMergeBytes = 16 * kMaxList2 + 8 * kGateRows;   // + per-head list start and count
constexpr uint32_t kSmem2 = kMergeOff2 + kMergeBytes + 64 + 1024;   // + counts + alignment slack
static_assert(kSmem2 <= 227 * 1024, "shared memory");

enum {
    C_Q = 0,                    // Q tiles landed (one phase per unit with work)
    C_QFREE = 1,                // every QK of the unit done: Q may be overwritten
    C_KF = 2,                   // [2] K tile landed
    C_VF = C_KF + kStages2,     // [2] V tile landed
    C_KE = C_VF + kStages2,     // [2] K stage free (both QKs done)
    C_VE = C_KE + kStages2,     // [2] V stage free (both PVs done)
    C_S = C_VE + kStages2,      // [2 Q tiles] S ready
    C_P = C_S + 2,              // [2 Q tiles][4 quarters] P of 32 keys written, 128 arrivals
    C_OD = C_P + 8,             // [2 Q tiles] last PV of the unit done
    C_L = C_OD + 2,             // [2 slots] list loaded
    C_LF = C_L + 2,             // [2 slots] list released, 8 arrivals (one per softmax warp)
    C_END = C_LF + 2,
    NBAR2
};
static_assert(8 * NBAR2 + 8 <= 512, "barrier area");

struct Tc2Args {
    Shape s;
    const int32_t *idx;
    const float *score;
    const int32_t *count;
    __nv_bfloat16 *O;
    float *lse;
    unsigned *status;
    int npair;   // units per (batch, kv-head, block)
    int hc;      // query heads per unit
    int units;
    unsigned long long wait_ns;   // limit of every bounded wait
    int stall_tile;               // test hook: the K load of this key tile (per CTA) is never issued; -1 = off
};

struct Unit {
    int b, g, j, h0;
    size_t lu;   // (b, g, j) list row
};

// Unit order: the units of one (batch, kv-head) are contiguous, so the CTAs
// running at any moment read the K/V of one or two heads and their tiles are
// re-read from L2 (all heads' K/V together would not fit); within a head the
// block index runs from the end, so its longest lists go first.
__device__ __forceinline__ Unit unit_at(const Tc2Args &a, int u) {
    const Shape &s = a.s;
    const int per_g = s.nb * a.npair;
    Unit w;
    const int bg = u / per_g;
    int r = u % per_g;
    w.j = s.nb - 1 - r / a.npair;
    const int pair = r % a.npair;
    w.g = bg % s.Hkv;
    w.b = bg / s.Hkv;
    w.h0 = w.g * s.G + pair * a.hc;
    w.lu = ((size_t)w.b * s.Hkv + w.g) * s.nb + w.j;
    return w;
}

// 128-key tiles of a list of cnt blocks
__device__ __forceinline__ int key_tiles(const Shape &s, int cnt) { return s.bs == 64 ? (cnt + 1) >> 1 : cnt; }


template <bool kHier>
__global__ void __launch_bounds__(kThreads2, 1)
prefill_tc2_kernel(const __grid_constant__ CUtensorMap tmQ, const __grid_constant__ CUtensorMap tmK,
                   const __grid_constant__ CUtensorMap tmV, Tc2Args a) {
    constexpr float kLog2e = 1.4426950408889634f;
    constexpr float kLn2 = 0.6931471805599453f;
    const Shape &s = a.s;
    extern __shared__ unsigned char smem_raw[];
    unsigned char *smem = reinterpret_cast<unsigned char *>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                                            ~uintptr_t(1023));
    const uint32_t sbase = smem_u32(smem);
    uint64_t *bars = reinterpret_cast<uint64_t *>(smem + kBarOff2);
    volatile int *abort_flag = reinterpret_cast<volatile int *>(smem + kBarOff2 + 8 * NBAR2);
    uint32_t *tmem_slot = reinterpret_cast<uint32_t *>(smem + kBarOff2 + 8 * NBAR2 + 4);
    int *cnt_s = reinterpret_cast<int *>(smem + kMergeOff2 + kMergeBytes);   // [2 slots]
    auto blk_of = [&](int slot) { return reinterpret_cast<int *>(smem + kListOff2 + slot * kListBytes); };
    auto gate_of = [&](int slot) {
        return reinterpret_cast<float *>(smem + kListOff2 + slot * kListBytes + 4 * kMaxList2);
    };
    auto bar = [&](int i) { return smem_u32(&bars[i]); };
    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;

    // ---- set-up -----------------------------------------------------------
    if (tid == 0) {
        for (int i = 0; i < NBAR2; ++i)
            mbar_init(bar(i), (i >= C_P && i < C_P + 8) ? 128 : (i == C_LF || i == C_LF + 1) ? 8 : 1);
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
        asm volatile("setmaxnreg.dec.sync.aligned.u32 %0;" ::"n"(kRegsLow2));
        if (lane == 0) {
            asm volatile("prefetch.tensormap [%0];" ::"l"(reinterpret_cast<uint64_t>(&tmQ)) : "memory");
            asm volatile("prefetch.tensormap [%0];" ::"l"(reinterpret_cast<uint64_t>(&tmK)) : "memory");
            asm volatile("prefetch.tensormap [%0];" ::"l"(reinterpret_cast<uint64_t>(&tmV)) : "memory");
        }
        bool ok = true;
        int gt = 0, nq = 0, ul = 0;   // key tiles, Q loads and units so far
        // copies issued and not yet seen complete: the last Q load (its phase),
        // and per ring stage the last key tile whose K / V load went out (-1:
        // none).  A stage is reused only after its previous copy was consumed,
        // so each barrier has at most this one phase outstanding.
        int qlast = -1, klast[kStages2], vlast[kStages2];
        for (int i = 0; i < kStages2; ++i) klast[i] = vlast[i] = -1;
        for (int u = blockIdx.x; u < a.units; u += gridDim.x, ++ul) {
            const Unit w = unit_at(a, u);
            const int slot = ul & 1;
            if (ul >= 2)
                ok = mbar_wait(bar(C_LF + slot), ((ul >> 1) - 1) & 1, abort_flag, a.status, a.wait_ns);
            if (!__all_sync(0xffffffffu, ok)) { ok = false; break; }
            // the unit's list: block ids (bad entries -> -1) and log2-unit gates
            int *blk_s = blk_of(slot);
            float *gate_s = gate_of(slot);
            int cnt;
            if (!(s.flags & SA_SELECT_PER_QHEAD)) {
                cnt = max(0, min(a.count[w.lu], s.cap));
                const int32_t *il = a.idx + w.lu * s.cap;
                const float *sl = a.score + w.lu * s.cap;
                const float s_loc = cnt > 0 ? sl[cnt - 1] : 0.f;
                for (int e = lane; e < cnt; e += 32) {
                    const int blk = il[e];
                    const bool good = blk >= 0 && blk <= w.j && (e == 0 || il[e - 1] < blk);
                    if (!good) set_status(a.status, kStatusBadIndex);
                    blk_s[e] = good ? blk : -1;
                    const bool forced = (blk == w.j && (s.flags & SA_LOCAL)) || (blk == 0 && (s.flags & SA_SINK));
                    gate_s[e] = kHier ? sl[e] * kLog2e
                                : ((s.flags & SA_GATE) && !forced) ? log_sigmoid(sl[e] - s_loc) * kLog2e : 0.f;
                }
            } else {
                // one list per query head: the unit's rows (a.hc heads) read the
                // union of their heads' lists, ascending; gate row hh holds head
                // hh's gate of each union entry, -inf where that head did not
                // keep the block (its keys then drop out of that head's softmax)
                int *mb = reinterpret_cast<int *>(smem + kMergeOff2);     // entry -> block (-1 bad)
                float *mg = reinterpret_cast<float *>(mb + kMaxList2);     // entry -> gate
                int *mh = reinterpret_cast<int *>(mg + kMaxList2);         // entry -> head in unit
                int *mf = mh + kMaxList2;                                  // entry -> first of its block
                int *hst = mf + kMaxList2;                                 // head -> first entry
                int *hcn = hst + kGateRows;                                // head -> entries
                int cn = 0;                                                // this lane's head count (lane < hc)
                if (lane < a.hc)
                    cn = max(0, min(a.count[((size_t)w.b * s.Hq + w.h0 + lane) * s.nb + w.j], s.cap));
                int start = cn;                                            // exclusive prefix over heads
#pragma unroll
                for (int o = 1; o < 32; o <<= 1) {
                    const int t = __shfl_up_sync(0xffffffffu, start, o);
                    if (lane >= o) start += t;
                }
                start -= cn;
                const int E = __shfl_sync(0xffffffffu, start + cn, a.hc - 1);
                if (lane < a.hc) {
                    hst[lane] = start;
                    hcn[lane] = cn;
                }
                __syncwarp();
                for (int f = lane; f < E; f += 32) {
                    int hh = 0;
                    for (int x = 1; x < a.hc; ++x) hh += f >= hst[x] ? 1 : 0;
                    mh[f] = hh;
                    {
                        const int st = hst[hh], c = hcn[hh];
                        const int e = f - st;
                        const size_t lu = ((size_t)w.b * s.Hq + w.h0 + hh) * s.nb + w.j;
                        const int32_t *il = a.idx + lu * s.cap;
                        const float *sl = a.score + lu * s.cap;
                        const int blk = il[e];
                        const bool good = blk >= 0 && blk <= w.j && (e == 0 || il[e - 1] < blk);
                        if (!good) set_status(a.status, kStatusBadIndex);
                        const bool forced = (blk == w.j && (s.flags & SA_LOCAL)) || (blk == 0 && (s.flags & SA_SINK));
                        mb[f] = good ? blk : -1;
                        mg[f] = ((s.flags & SA_GATE) && !forced) ? log_sigmoid(sl[e] - sl[c - 1]) * kLog2e : 0.f;
                    }
                }
                __syncwarp();
                // first entry of each block (lowest head), then its rank among the distinct blocks
                for (int f = lane; f < E; f += 32) {
                    const int blk = mb[f];
                    bool first = blk >= 0;
                    for (int x = 0; x < f && first; ++x) first = mb[x] != blk;
                    mf[f] = first ? 1 : 0;
                }
                __syncwarp();
                int nd = 0;
                for (int f = lane; f < E; f += 32) nd += mf[f];
                cnt = __reduce_add_sync(0xffffffffu, nd);
                for (int x = lane; x < a.hc * kMaxList2; x += 32)
                    if (x % kMaxList2 < cnt) gate_s[x] = -CUDART_INF_F;
                __syncwarp();
                for (int f = lane; f < E; f += 32) {
                    const int blk = mb[f];
                    if (blk < 0) continue;
                    int rank = 0;
                    for (int x = 0; x < E; ++x) rank += (mf[x] && mb[x] < blk) ? 1 : 0;
                    if (mf[f]) blk_s[rank] = blk;
                    gate_s[mh[f] * kMaxList2 + rank] = mg[f];
                }
            }
            if (lane == 0) cnt_s[slot] = cnt;
            __syncwarp();
            if (lane == 0) mbar_arrive(bar(C_L + slot));
            const int T = key_tiles(s, cnt);
            if (lane == 0 && T > 0) {
                // Q tiles: rows of heads h0 .. h0+3 (block 64) or h0, h0+1 (block 128)
                if (nq >= 1) ok = mbar_wait(bar(C_QFREE), (nq - 1) & 1, abort_flag, a.status, a.wait_ns);
                if (ok) {
                    qlast = nq;
                    mbar_expect_tx(bar(C_Q), 2 * kTile2);
                    for (int q = 0; q < 2; ++q)
                        for (int c = 0; c < 2; ++c)
                            for (int e = 0; e < 2; ++e) {
                                const int y = s.bs == 64 ? (w.b * s.Hq + w.h0 + 2 * q + e) * s.N + w.j * 64
                                                         : (w.b * s.Hq + w.h0 + q) * s.N + w.j * 128 + 64 * e;
                                SA_CHECK_START(a.status, s.bs == 64 ? w.h0 + 2 * q + e : w.h0 + q, s.Hq);
                                SA_CHECK_START(a.status, s.bs == 64 ? w.j * 64 : w.j * 128 + 64 * e, s.nb * s.bs);
                                tma_load_2d(sbase + kQOff2 + q * kTile2 + c * kChunk2 + e * 8192, &tmQ, bar(C_Q),
                                            64 * c, y);
                            }
                }
                // key tiles: two 64-row halves each (two blocks of 64, or one block of 128)
                const int kvbase = (w.b * s.Hkv + w.g) * s.N;
                for (int t = 0; ok && t < T; ++t) {
                    const int gg = gt + t, st = gg % kStages2, use = gg / kStages2;
                    int y0, y1;
                    if (s.bs == 64) {
                        // an odd list's last tile repeats its block in the second half (masked later)
                        y0 = kvbase + max(0, blk_s[2 * t]) * 64;
                        y1 = kvbase + max(0, blk_s[min(2 * t + 1, cnt - 1)]) * 64;
                    } else {
                        y0 = kvbase + max(0, blk_s[t]) * 128;
                        y1 = y0 + 64;
                    }
                    if (gg >= kStages2 &&
                        !(ok = mbar_wait(bar(C_KE + st), (use - 1) & 1, abort_flag, a.status, a.wait_ns)))
                        break;
                    SA_CHECK_START(a.status, y0 - kvbase, s.N);
                    SA_CHECK_START(a.status, y1 - kvbase, s.bs == 64 ? s.N : s.nb * s.bs);   // a block's second half: padded extent
                    if (gg != a.stall_tile) {
                        mbar_expect_tx(bar(C_KF + st), kTile2);
                        for (int c = 0; c < 2; ++c) {
                            const uint32_t d = sbase + kKOff2 + st * kTile2 + c * kChunk2;
                            tma_load_2d(d, &tmK, bar(C_KF + st), 64 * c, y0);
                            tma_load_2d(d + 8192, &tmK, bar(C_KF + st), 64 * c, y1);
                        }
                        klast[st] = gg;
                    }
                    if (gg >= kStages2 &&
                        !(ok = mbar_wait(bar(C_VE + st), (use - 1) & 1, abort_flag, a.status, a.wait_ns)))
                        break;
                    mbar_expect_tx(bar(C_VF + st), kTile2);
                    for (int c = 0; c < 2; ++c) {
                        const uint32_t d = sbase + kVOff2 + st * kTile2 + c * kChunk2;
                        tma_load_2d(d, &tmV, bar(C_VF + st), 64 * c, y0);
                        tma_load_2d(d + 8192, &tmV, bar(C_VF + st), 64 * c, y1);
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
            // let the copies in flight land before the CTA exits (bounded)
            volatile int never = 0;
            if (qlast >= 0) mbar_wait(bar(C_Q), qlast & 1, &never, a.status, a.wait_ns);
            for (int st = 0; st < kStages2; ++st) {
                if (klast[st] >= 0)
                    mbar_wait(bar(C_KF + st), (klast[st] / kStages2) & 1, &never, a.status, a.wait_ns);
                if (vlast[st] >= 0)
                    mbar_wait(bar(C_VF + st), (vlast[st] / kStages2) & 1, &never, a.status, a.wait_ns);
            }
        }
    } else if (warp == 1) {
        // ---- MMA issuer -----------------------------------------------------
        // The whole warp runs this loop (waits, descriptor arithmetic) in
        // lockstep; one elected lane issues each MMA and commit.
        asm volatile("setmaxnreg.dec.sync.aligned.u32 %0;" ::"n"(kRegsLow2));
        constexpr uint32_t idq = idesc_bf16(false, 128), idp = idesc_bf16(true, 128);
        // S_q = Q_q K^T for key tile gg (8 MMAs of K = 16 over d = 128);
        // descriptor start addresses advance in 16-byte units (offset >> 4)
        auto qk = [&](int q, int gg) {
            const uint64_t da = desc_k_sw128(sbase + kQOff2 + q * kTile2);
            const uint64_t db = desc_k_sw128(sbase + kKOff2 + (gg % kStages2) * kTile2);
#pragma unroll
            for (int k = 0; k < 8; ++k) {
                const uint32_t off = ((k >> 2) * kChunk2 + (k & 3) * 32) >> 4;
                mma_ss_w(tmem + q * 128, da + off, db + off, idq, k > 0);
            }
            mma_commit_w(bar(C_S + q));
        };
        // O_q += P_q V for keys 32h .. 32h+31 of key tile gg; P_q (bf16) is the
        // first 64 columns of S_q, handed over in quarters
        auto pv = [&](int q, int gg, int h, bool acc) {
            const uint64_t db = desc_mn_sw128(sbase + kVOff2 + (gg % kStages2) * kTile2, kChunk2);
#pragma unroll
            for (int k = 2 * h; k < 2 * h + 2; ++k)
                mma_ts_w(tmem + 256 + q * 128, tmem + q * 128 + 8 * k, db + ((k * 2048) >> 4), idp, acc || k > 0);
        };
        auto wait = [&](int i, int parity) {
            return __all_sync(0xffffffffu, mbar_wait(bar(i), parity, abort_flag, a.status, a.wait_ns));
        };
        bool ok = true;
        int gt = 0, nq = 0, ul = 0;
        for (int u = blockIdx.x; ok && u < a.units; u += gridDim.x, ++ul) {
            const int slot = ul & 1;
            if (!(ok = wait(C_L + slot, (ul >> 1) & 1))) break;
            const int T = key_tiles(s, cnt_s[slot]);
            if (T == 0) continue;
            if (!(ok = wait(C_Q, nq & 1))) break;
            if (!(ok = wait(C_KF + gt % kStages2, (gt / kStages2) & 1))) break;
            tc_fence_after();
            qk(0, gt);
            qk(1, gt);
            mma_commit_w(bar(C_KE + gt % kStages2));
            if (T == 1) mma_commit_w(bar(C_QFREE));
            for (int t = 0; ok && t < T; ++t) {
                const int gg = gt + t;
                if (!(ok = wait(C_P, gg & 1))) break;
                if (!(ok = wait(C_VF + gg % kStages2, (gg / kStages2) & 1))) break;
                tc_fence_after();
                pv(0, gg, 0, t > 0);
                for (int h = 1; ok && h < 4; ++h) {
                    if (!(ok = wait(C_P + h, gg & 1))) break;
                    tc_fence_after();
                    pv(0, gg, h, true);
                }
                if (!ok) break;
                if (t == T - 1) mma_commit_w(bar(C_OD));
                if (t + 1 < T) {
                    const int g1 = gg + 1;
                    if (!(ok = wait(C_KF + g1 % kStages2, (g1 / kStages2) & 1))) break;
                    tc_fence_after();
                    qk(0, g1);
                }
                for (int h = 0; ok && h < 4; ++h) {
                    if (!(ok = wait(C_P + 4 + h, gg & 1))) break;
                    tc_fence_after();
                    pv(1, gg, h, t > 0 || h > 0);
                }
                if (!ok) break;
                mma_commit_w(bar(C_VE + gg % kStages2));
                if (t == T - 1) mma_commit_w(bar(C_OD + 1));
                if (t + 1 < T) {
                    qk(1, gg + 1);
                    mma_commit_w(bar(C_KE + (gg + 1) % kStages2));
                    if (t + 2 == T) mma_commit_w(bar(C_QFREE));
                }
            }
            gt += T;
            ++nq;
        }
        // drain: every MMA issued above has completed once this arrives
        // (waited on even after an abort: TMEM is freed only after it)
        mma_commit_w(bar(C_END));
        volatile int never = 0;
        mbar_wait(bar(C_END), 0, &never, a.status, a.wait_ns);
    } else if (warp < 4) {
        asm volatile("setmaxnreg.dec.sync.aligned.u32 %0;" ::"n"(kRegsLow2));
    } else {
        asm volatile("setmaxnreg.inc.sync.aligned.u32 %0;" ::"n"(kRegsHigh2));
        // ---- softmax warpgroups --------------------------------------------
        const int q = (warp - 4) >> 2;                   // Q tile of this warpgroup
        const int qq = warp & 3;                         // TMEM lane quarter of this warp
        const int r = 32 * qq + lane;                    // row within the Q tile
        const uint32_t lane_off = (uint32_t)(32 * qq) << 16;
        const uint32_t tS = tmem + lane_off + q * 128, tO = tmem + lane_off + 256 + q * 128;
        const bool causal = s.flags & SA_CAUSAL;
        constexpr bool hier = kHier;
        const float qk_scale = s.scale * kLog2e;
        bool ok = true;
        int gt = 0, nq = 0, ul = 0;
        for (int u = blockIdx.x; ok && u < a.units; u += gridDim.x, ++ul) {
            const Unit w = unit_at(a, u);
            const int slot = ul & 1;
            ok = mbar_wait(bar(C_L + slot), (ul >> 1) & 1, abort_flag, a.status, a.wait_ns);
            if (!__all_sync(0xffffffffu, ok)) { ok = false; break; }
            const int cnt = cnt_s[slot];
            const int *blk_s = blk_of(slot);
            const int T = key_tiles(s, cnt);
            int head, ri;
            if (s.bs == 64) { head = w.h0 + 2 * q + (r >> 6); ri = r & 63; }
            else { head = w.h0 + q; ri = r; }
            // per-query-head lists: this row's head has its own gate row
            const float *gate_s = gate_of(slot) + ((s.flags & SA_SELECT_PER_QHEAD) ? (head - w.h0) * kMaxList2 : 0);
            const int qi = w.j * s.bs + ri;              // query position of this row
            float m_run = -CUDART_INF_F, l = 0.f;
            // hierarchical mode ([HiLS]): every block gets its own softmax and
            // the block outputs are weighted by softmax_b(s_b).  With M the
            // largest retrieval score of the list, block b enters O as
            // P_b V_b * 2^(s_b - M) / l_b and l sums 2^(s_b - M), so O is never
            // rescaled and the result is O / l, with LSE = M + log2 l.
            if constexpr (hier) {
                for (int e = 0; e < cnt; ++e)
                    if (blk_s[e] >= 0) m_run = fmaxf(m_run, gate_s[e]);
            }
            for (int t = 0; t < T; ++t) {
                ok = mbar_wait(bar(C_S + q), (gt + t) & 1, abort_flag, a.status, a.wait_ns);
                if (!__all_sync(0xffffffffu, ok)) { ok = false; break; }
                tc_fence_after();
                float x[128];
#pragma unroll
                for (int c = 0; c < 4; ++c) tmem_ld32(tS + 32 * c, x + 32 * c);
                tmem_wait_ld();
                reg_fence<128>(x);
                // per 64-key half: its block, gate and masks (a bad entry, an
                // odd list's empty half, the ragged end, causality in the local block)
                float gh[2], mh[2], raw[2];
#pragma unroll
                for (int h = 0; h < 2; ++h) {
                    int blk, t0;
                    float gl;
                    if (s.bs == 64) {
                        const int e = 2 * t + h;
                        blk = e < cnt ? blk_s[e] : -1;
                        gl = e < cnt ? gate_s[e] : 0.f;
                        t0 = blk * 64;
                    } else {
                        blk = blk_s[t];
                        gl = gate_s[t];
                        t0 = blk * 128 + 64 * h;
                    }
                    float *xh = x + 64 * h;
                    if (blk < 0 || t0 + 64 > s.N || (causal && blk == w.j)) {
#pragma unroll
                        for (int k = 0; k < 64; ++k) {
                            const int key = t0 + k;
                            const bool vis = blk >= 0 && key < s.N && !(causal && blk == w.j && key > qi);
                            xh[k] = vis ? xh[k] : -CUDART_INF_F;
                        }
                    }
                    // four independent chains of 3-input maxima
                    float mq[4];
#pragma unroll
                    for (int e = 0; e < 4; ++e) mq[e] = fmaxf(xh[2 * e], xh[2 * e + 1]);
#pragma unroll
                    for (int k = 8; k < 64; k += 8)
#pragma unroll
                        for (int e = 0; e < 4; ++e) mq[e] = fmax3(mq[e], xh[k + 2 * e], xh[k + 2 * e + 1]);
                    const float mm = fmaxf(fmax3(mq[0], mq[1], mq[2]), mq[3]);
                    raw[h] = mm;
                    mh[h] = mm == -CUDART_INF_F ? -CUDART_INF_F : fmaf(mm, qk_scale, gl);
                    gh[h] = gl;
                }
                if constexpr (hier) {
                    // per-block softmax: one block per 64-key half (block 64), each
                    // half handed over as soon as its weight is known; or one block
                    // per tile (block 128), handed over after both halves
                    const float2 sc2 = make_float2(qk_scale, qk_scale);
                    const bool one = s.bs == 128;
                    const float mt = fmaxf(raw[0], raw[1]);
                    float lsum0 = 0.f;
#pragma unroll
                    for (int h = 0; h < 2; ++h) {
                        const float mb = one ? mt : raw[h];
                        const float nb2 = mb == -CUDART_INF_F ? 0.f : -mb * qk_scale;
                        const float2 b2 = make_float2(nb2, nb2);
                        float2 acc = make_float2(0.f, 0.f);
#pragma unroll
                        for (int k = 0; k < 32; ++k) {
                            const float2 z = ffma2(make_float2(x[64 * h + 2 * k], x[64 * h + 2 * k + 1]), sc2, b2);
                            const float2 pp = make_float2(ex2(z.x), ex2(z.y));
                            x[64 * h + 2 * k] = pp.x;
                            x[64 * h + 2 * k + 1] = pp.y;
                            acc = fadd2(acc, pp);
                        }
                        const float lh = acc.x + acc.y;
                        if (one && h == 0) {
                            lsum0 = lh;
                            continue;
                        }
                        const float lb = one ? lsum0 + lh : lh;
                        const float wb = lb > 0.f ? ex2(gh[h] - m_run) : 0.f;
                        const float fq = lb > 0.f ? wb / lb : 0.f;
                        l += wb;
                        // quarters of this half (both halves when the tile is one block)
#pragma unroll
                        for (int c = 0; c < 4; ++c) {
                            if (!one && (c >> 1) != h) continue;
                            uint32_t pk[16];
#pragma unroll
                            for (int k = 0; k < 16; ++k) {
                                __nv_bfloat162 h2 = __floats2bfloat162_rn(x[32 * c + 2 * k] * fq,
                                                                          x[32 * c + 2 * k + 1] * fq);
                                pk[k] = *reinterpret_cast<uint32_t *>(&h2);
                            }
                            tmem_st16(tS + 16 * c, pk);
                            tmem_wait_st();
                            tc_fence_before();
                            mbar_arrive(bar(C_P + 4 * q + c));
                        }
                    }
                    continue;
                }
                const float mx = fmaxf(mh[0], mh[1]);
                if (t == 0) {
                    m_run = mx;
                } else {
                    const bool need = mx > m_run + 8.f;
                    if (__any_sync(0xffffffffu, need)) {
                        // the PV before this S has completed: O_q is stable
                        const float corr = need ? ex2(m_run - mx) : 1.f;
                        if (need) {
                            l *= corr;
                            m_run = mx;
                        }
#pragma unroll
                        for (int cc = 0; cc < 4; ++cc) {
                            float o[32];
                            tmem_ld32(tO + 32 * cc, o);
                            tmem_wait_ld();
                            reg_fence<32>(o);
#pragma unroll
                            for (int k = 0; k < 32; ++k) o[k] *= corr;
                            tmem_st32(tO + 32 * cc, reinterpret_cast<const uint32_t *>(o));
                        }
                        tmem_wait_st();
                    }
                }
                // p = 2^(x * scale + gate - ref), written as bf16 pairs over S columns 0..63
                // each 32-key quarter is handed to the MMA warp as soon as it is
                // written, so its PV runs while the next quarter is exponentiated
                // (pairs of elements go through the packed fp32 pipe: one FMA and
                // one add per two keys)
                const float ref = m_run == -CUDART_INF_F ? 0.f : m_run;
                const float2 sc2 = make_float2(qk_scale, qk_scale);
                float2 ls2a = make_float2(0.f, 0.f), ls2b = make_float2(0.f, 0.f);
#pragma unroll
                for (int c = 0; c < 4; ++c) {
                    const float bias = gh[c >> 1] - ref;
                    const float2 b2 = make_float2(bias, bias);
                    uint32_t pk[16];
#pragma unroll
                    for (int k = 0; k < 16; ++k) {
                        const float2 z = ffma2(make_float2(x[32 * c + 2 * k], x[32 * c + 2 * k + 1]), sc2, b2);
                        const float2 pp = make_float2(ex2(z.x), ex2(z.y));
                        if (k & 1) ls2b = fadd2(ls2b, pp);
                        else ls2a = fadd2(ls2a, pp);
                        __nv_bfloat162 h2 = __floats2bfloat162_rn(pp.x, pp.y);
                        pk[k] = *reinterpret_cast<uint32_t *>(&h2);
                    }
                    tmem_st16(tS + 16 * c, pk);
                    tmem_wait_st();
                    tc_fence_before();
                    mbar_arrive(bar(C_P + 4 * q + c));
                }
                l += (ls2a.x + ls2a.y) + (ls2b.x + ls2b.y);
            }
            if (!ok) break;
            // ---- epilogue: O_q / l -> bf16, LSE ----------------------------
            if (T > 0) {
                ok = mbar_wait(bar(C_OD + q), nq & 1, abort_flag, a.status, a.wait_ns);
                if (!__all_sync(0xffffffffu, ok)) { ok = false; break; }
                tc_fence_after();
            }
            const bool row_ok = qi < s.N;
            __nv_bfloat16 *orow = a.O + (((size_t)w.b * s.Hq + head) * s.N + (row_ok ? qi : 0)) * 128;
            const float inv = l > 0.f ? 1.f / l : 0.f;
            {
                // all 128 columns in one TMEM round trip
                float o[128];
                if (T > 0) {
#pragma unroll
                    for (int cc = 0; cc < 4; ++cc) tmem_ld32(tO + 32 * cc, o + 32 * cc);
                    tmem_wait_ld();
                    reg_fence<128>(o);
                } else {
#pragma unroll
                    for (int k = 0; k < 128; ++k) o[k] = 0.f;
                }
                if (row_ok) {
#pragma unroll
                    for (int v = 0; v < 128; v += 8) {
                        float f[8];
#pragma unroll
                        for (int k = 0; k < 8; ++k) f[k] = o[v + k] * inv;
                        store16(orow + v, f);
                    }
                }
            }
            if (row_ok)
                a.lse[((size_t)w.b * s.Hq + head) * s.N + qi] = l > 0.f ? (m_run + log2f(l)) * kLn2 : -CUDART_INF_F;
            __syncwarp();
            if (lane == 0) mbar_arrive(bar(C_LF + slot));
            gt += T;
            if (T > 0) ++nq;
        }
    }

    // ---- teardown -----------------------------------------------------------
    tc_fence_before();
    __syncthreads();
    if (warp == 1) {
        tc_fence_after();
        asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(tmem), "n"(512));
    }
}



}  // namespace

bool prefill_tc2_supported(const Shape &s) {
    if (s.dtype != SA_BF16 || s.d != 128) return false;
    if (s.bs != 64 && s.bs != 128) return false;
    if ((s.G * s.bs) % kRows) return false;
    if (s.cap > kMaxList2) return false;
    // per-query-head lists: the union of a unit's heads must fit one list (gated or plain mode)
    if ((s.flags & SA_SELECT_PER_QHEAD) && ((s.flags & SA_HIER) || (kRows / s.bs) * s.cap > kMaxList2))
        return false;
    const char *e = getenv("SPARSE_ATTN_PREFILL_PATH");
    if (e && (strcmp(e, "simt") == 0 || strcmp(e, "tc1") == 0)) return false;
    return true;
}

cudaError_t launch_prefill_tc2(const Shape &s, const void *Q, const void *K, const void *V, const int32_t *idx,
                               const float *score, const int32_t *count, void *O, float *lse, unsigned *status,
                               cudaStream_t st) {
    // The register split above assumes the kernel is launched at exactly
    // kRegsLaunch2 registers per thread; anything else could stall the
    // warpgroups' register exchange, so refuse to launch.
    void (*kern)(CUtensorMap, CUtensorMap, CUtensorMap, Tc2Args) =
        (s.flags & SA_HIER) ? prefill_tc2_kernel<true> : prefill_tc2_kernel<false>;
    cudaFuncAttributes fa;
    cudaError_t e = cudaFuncGetAttributes(&fa, kern);
    if (e != cudaSuccess) return e;
    if (fa.numRegs != kRegsLaunch2) return cudaErrorInvalidDeviceFunction;
    CUtensorMap mq, mk, mv;
    const uint64_t qrows = (uint64_t)s.B * s.Hq * s.N, krows = (uint64_t)s.B * s.Hkv * s.N;
    if (!make_map_d128(&mq, Q, qrows, 64) || !make_map_d128(&mk, K, krows, 64) ||
        !make_map_d128(&mv, V, krows, 64))
        return cudaErrorInvalidValue;
    Tc2Args a{};
    a.s = s;
    a.idx = idx;
    a.score = score;
    a.count = count;
    a.O = (__nv_bfloat16 *)O;
    a.lse = lse;
    a.status = status;
    a.hc = kRows / s.bs;
    a.npair = s.G / a.hc;
    a.wait_ns = tc::kWaitNs;
    a.stall_tile = -1;
    // Test hook for the bounded waits: SPARSE_ATTN_TEST_STALL=<t> makes every
    // CTA skip the K load of its key tile t (nothing is left in flight for
    // it), so the MMA warp's wait on that tile runs out after 1 ms; the CTA
    // then records kStatusTimeout, lets its other copies land, frees TMEM
    // and exits.
    if (const char *st = getenv("SPARSE_ATTN_TEST_STALL")) {
        a.stall_tile = atoi(st);
        a.wait_ns = 1000000ull;
    }
    a.units = s.B * s.Hkv * s.nb * a.npair;
    const int sms = sm_count();
    if (sms <= 0) return cudaErrorNoDevice;
    e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)kSmem2);
    if (e != cudaSuccess) return e;
    const unsigned grid = (unsigned)min(a.units, sms);
    kern<<<grid, kThreads2, kSmem2, st>>>(mq, mk, mv, a);
    note_launch();
    return cudaGetLastError();
}

}  // namespace sa
