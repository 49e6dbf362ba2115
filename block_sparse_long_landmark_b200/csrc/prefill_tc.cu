// prefill_tc.cu -- tensor-core (tcgen05 + TMEM + TMA) gated block-sparse
// prefill for bf16, d = 128, block 64 or 128.
//
// [SAS] "Ключевые факты" / "Как это применить": FlashAttention-style blockwise
// attention over the kept blocks only, the square matrix never materialised;
// the selector's gate log_sigmoid(s_b - s_local) is added to the logits of
// selected blocks inside the softmax (forced sink / local blocks get 0).
//
// One CTA = one M=128 tile: 128 query rows of one (batch, kv-head, tile) that
// share the tile's kept list (GQA: with block 64 the rows of 2 query heads,
// with block 128 those of 1; the other heads of the group are neighbouring
// CTAs, which find the same K/V tiles in L2).  Two CTAs run on every SM, each
// with half the tensor memory, so one CTA's start and end overlap the other's
// main loop.  Key tiles are 64 keys: one kept block of 64, or half of a block
// of 128.
//
// Warp roles (8 warps = 2 warpgroups):
//   warp 0      TMA producer: Q once, then K and V key tiles into 2-stage rings
//   warp 1      TMEM owner + single-thread tcgen05.mma issuer
//   warps 2-3   idle
//   warps 4-7   softmax; thread = one query row = one TMEM lane
// Registers: launched at 128 per thread (two CTAs, 4 warps per SM
// sub-partition); the first warpgroup gives back down to 56 and the softmax
// warpgroup takes 200: 128 x 56 + 128 x 200 = 256 x 128, the launch's total.
// TMEM (256 columns): S buffers A and B (64 fp32 columns each) and O (128).
// P (bf16) is written over the first 32 columns of its S buffer and read by
// the PV MMA straight from TMEM.  S is double-buffered: while the softmax
// warpgroup works on key tile i, the tensor core already holds S(i+1) and,
// once P(i) is in, runs  O += P(i) V_i ; S(i+2) = Q K_(i+2)^T.
// The running max is rescaled lazily: O is corrected in TMEM only when a
// row's max grows by more than 2^8.
//
// Every mbarrier wait is bounded (about two seconds of %globaltimer); on
// expiry the CTA records kStatusTimeout, drains, frees TMEM and exits.
#include <math_constants.h>

#include <cstdlib>
#include <cstring>

#include "bounds.cuh"
#include "common.cuh"
#include "tc_ptx.cuh"

namespace sa {
namespace {

constexpr int kThreads = 256;
constexpr int kRegsLaunch = 128, kRegsProducer = 56, kRegsSoftmax = 200;
static_assert(128 * kRegsProducer + 128 * kRegsSoftmax <= kThreads * kRegsLaunch, "register split");
constexpr int kStages = 2;                      // per ring (K and V)
constexpr uint32_t kQChunk = 128 * 128;         // 128 rows x 64 bf16 (one 128-byte swizzle column)
constexpr uint32_t kQTile = 2 * kQChunk;        // the M tile: 128 rows x 128 bf16
constexpr uint32_t kKChunk = 64 * 128;          // 64 keys x 64 bf16
constexpr uint32_t kKTile = 2 * kKChunk;        // a key tile: 64 keys x 128 bf16
constexpr uint32_t kQOff = 0;
constexpr uint32_t kKOff = kQTile;              // kStages K tiles
constexpr uint32_t kVOff = kKOff + kStages * kKTile;
constexpr uint32_t kBarOff = kVOff + kStages * kKTile;
constexpr int kMaxList = 258;
constexpr uint32_t kSmemBytes = kBarOff + 1024 + 8 * kMaxList + 2048;   // + alignment slack
constexpr uint32_t kTmemCols = 256;

// barrier slots (uint64 each)
enum {
    B_Q = 0,
    B_KF = 1,                   // [kStages] K tile landed
    B_VF = B_KF + kStages,      // [kStages] V tile landed
    B_KE = B_VF + kStages,      // [kStages] K tile consumed (QK done)
    B_VE = B_KE + kStages,      // [kStages] V tile consumed (PV done)
    B_S = B_VE + kStages,       // [2 buffers] S ready
    B_P = B_S + 2,              // [2 buffers] P ready, 128 arrivals each
    B_O = B_P + 2,              // one phase per PV
    B_END = B_O + 1,
    NBAR
};

struct TcArgs {
    Shape s;
    const int32_t *idx;
    const float *score;
    const int32_t *count;
    __nv_bfloat16 *O;
    float *lse;
    unsigned *status;
    int npair;   // CTAs per (batch, kv-head, tile)
    int hc;      // query heads per CTA
};

using namespace tc;

// ---------------------------------------------------------------------------
// kernel
// ---------------------------------------------------------------------------
__global__ void __launch_bounds__(kThreads, 2)
prefill_tc_kernel(const __grid_constant__ CUtensorMap tmQ, const __grid_constant__ CUtensorMap tmK,
                  const __grid_constant__ CUtensorMap tmV, TcArgs a) {
    constexpr float kLog2e = 1.4426950408889634f;
    constexpr float kLn2 = 0.6931471805599453f;
    const Shape &s = a.s;
    extern __shared__ unsigned char smem_raw[];
    unsigned char *smem = reinterpret_cast<unsigned char *>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                                            ~uintptr_t(1023));
    const uint32_t sbase = smem_u32(smem);
    uint64_t *bars = reinterpret_cast<uint64_t *>(smem + kBarOff);
    volatile int *abort_flag = reinterpret_cast<volatile int *>(smem + kBarOff + 8 * NBAR);
    uint32_t *tmem_slot = reinterpret_cast<uint32_t *>(smem + kBarOff + 8 * NBAR + 4);
    int *blk_s = reinterpret_cast<int *>(smem + kBarOff + 1024);
    float *gate_s = reinterpret_cast<float *>(smem + kBarOff + 1024 + 4 * kMaxList);
    auto bar = [&](int i) { return smem_u32(&bars[i]); };

    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    // CTA -> (batch, kv-head, tile, head group); larger tiles first
    int u = blockIdx.x;
    const int pair = u % a.npair;
    u /= a.npair;
    const int j = s.nb - 1 - (u % s.nb);
    u /= s.nb;
    const int g = u % s.Hkv;
    const int b = u / s.Hkv;
    const int h0 = g * s.G + pair * a.hc;          // first query head of this CTA
    const size_t lu = ((size_t)b * s.Hkv + g) * s.nb + j;
    const int cnt = max(0, min(a.count[lu], s.cap));
    const int sub = s.bs / 64;                     // 64-key tiles per kept block
    const int T = cnt * sub;                       // key tiles

    // ---- set-up -----------------------------------------------------------
    if (tid == 0) {
        for (int i = 0; i < NBAR; ++i) mbar_init(bar(i), (i == B_P || i == B_P + 1) ? 128 : 1);
        *abort_flag = 0;
        asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
    }
    if (tid < cnt) {
        const int32_t *il = a.idx + lu * s.cap;
        const float *sl = a.score + lu * s.cap;
        const int blk = il[tid];
        const bool ok = blk >= 0 && blk <= j && (tid == 0 || il[tid - 1] < blk);
        if (!ok) set_status(a.status, kStatusBadIndex);
        blk_s[tid] = ok ? blk : -1;
        const bool forced = (blk == j && (s.flags & SA_LOCAL)) || (blk == 0 && (s.flags & SA_SINK));
        // gated: the log2-unit gate of the block; hierarchical: its log2-unit retrieval score
        gate_s[tid] = (s.flags & SA_HIER) ? sl[tid] * kLog2e
                      : ((s.flags & SA_GATE) && !forced) ? log_sigmoid(sl[tid] - sl[cnt - 1]) * kLog2e : 0.f;
    }
    if (warp == 1) {
        asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(smem_u32(tmem_slot)),
                     "n"(kTmemCols));
        asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;");
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = *tmem_slot;
    const float qk_scale = s.scale * kLog2e;

    if (warp == 0) {
        // ---- TMA producer -------------------------------------------------
        asm volatile("setmaxnreg.dec.sync.aligned.u32 %0;" ::"n"(kRegsProducer));
        if (lane == 0 && T > 0) {
            asm volatile("prefetch.tensormap [%0];" ::"l"(reinterpret_cast<uint64_t>(&tmQ)) : "memory");
            asm volatile("prefetch.tensormap [%0];" ::"l"(reinterpret_cast<uint64_t>(&tmK)) : "memory");
            asm volatile("prefetch.tensormap [%0];" ::"l"(reinterpret_cast<uint64_t>(&tmV)) : "memory");
            mbar_expect_tx(bar(B_Q), kQTile);
            for (int c = 0; c < 2; ++c)
                for (int e = 0; e < 2; ++e) {
                    // block 64: rows of heads h0 and h0+1; block 128: rows 0-63 and 64-127 of head h0
                    const int y = s.bs == 64 ? ((b * s.Hq + h0 + e) * s.N) + j * 64
                                             : ((b * s.Hq + h0) * s.N) + j * 128 + 64 * e;
                    SA_CHECK_START(a.status, s.bs == 64 ? h0 + e : h0, s.Hq);
                    SA_CHECK_START(a.status, j * s.bs, s.nb * s.bs);
                    tma_load_2d(sbase + kQOff + c * kQChunk + e * 8192, &tmQ, bar(B_Q), 64 * c, y);
                }
            const int kvbase = (b * s.Hkv + g) * s.N;
            int nk = 0, nv = 0;   // K and V tiles issued
            for (int t = 0; t < T; ++t) {
                const int st = t % kStages, use = t / kStages;
                const int blk = max(0, blk_s[t / sub]);
                const int y = kvbase + blk * s.bs + (t % sub) * 64;
                SA_CHECK_START(a.status, blk * s.bs, s.N);
                if (t >= kStages && !mbar_wait(bar(B_KE + st), (use - 1) & 1, abort_flag, a.status)) break;
                mbar_expect_tx(bar(B_KF + st), kKTile);
                for (int ch = 0; ch < 2; ++ch)
                    tma_load_2d(sbase + kKOff + st * kKTile + ch * kKChunk, &tmK, bar(B_KF + st), 64 * ch, y);
                nk = t + 1;
                if (t >= kStages && !mbar_wait(bar(B_VE + st), (use - 1) & 1, abort_flag, a.status)) break;
                mbar_expect_tx(bar(B_VF + st), kKTile);
                for (int ch = 0; ch < 2; ++ch)
                    tma_load_2d(sbase + kVOff + st * kKTile + ch * kKChunk, &tmV, bar(B_VF + st), 64 * ch, y);
                nv = t + 1;
            }
            if (*abort_flag) {
                // let the copies in flight land before the CTA exits (bounded)
                volatile int never = 0;
                mbar_wait(bar(B_Q), 0, &never, a.status);
                for (int t = max(0, nk - kStages); t < nk; ++t)
                    mbar_wait(bar(B_KF + t % kStages), (t / kStages) & 1, &never, a.status);
                for (int t = max(0, nv - kStages); t < nv; ++t)
                    mbar_wait(bar(B_VF + t % kStages), (t / kStages) & 1, &never, a.status);
            }
        }
    } else if (warp == 1) {
        // ---- MMA issuer ---------------------------------------------------
        asm volatile("setmaxnreg.dec.sync.aligned.u32 %0;" ::"n"(kRegsProducer));
        if (lane == 0 && T > 0) {
            constexpr uint32_t idq = idesc_bf16(false, 64), idp = idesc_bf16(true, 128);
            bool ok = mbar_wait(bar(B_Q), 0, abort_flag, a.status);
            tc_fence_after();
            const uint32_t qa = sbase + kQOff;
            // S(t) = Q K_t^T into buffer t & 1; frees K stage when done
            auto qk = [&](int t) {
                const int st = t % kStages;
                const uint32_t kb = sbase + kKOff + st * kKTile;
                const uint32_t dS = tmem + (t & 1) * 64;
#pragma unroll
                for (int k = 0; k < 8; ++k)
                    mma_ss(dS, desc_k_sw128(qa + (k >> 2) * kQChunk + (k & 3) * 32),
                           desc_k_sw128(kb + (k >> 2) * kKChunk + (k & 3) * 32), idq, k > 0);
                mma_commit(bar(B_S + (t & 1)));
                mma_commit(bar(B_KE + st));
            };
            // O += P(t) V_t, P read from the first 32 columns of S buffer t & 1
            auto pv = [&](int t) {
                const int st = t % kStages;
                const uint32_t vb = sbase + kVOff + st * kKTile;
                const uint32_t aP = tmem + (t & 1) * 64, dO = tmem + 128;
#pragma unroll
                for (int k = 0; k < 4; ++k)
                    mma_ts(dO, aP + 8 * k, desc_mn_sw128(vb + k * 2048, kKChunk), idp, (t > 0 || k > 0));
                mma_commit(bar(B_O));
                mma_commit(bar(B_VE + st));
            };
            for (int t = 0; ok && t < min(2, T); ++t) {
                if (!(ok = mbar_wait(bar(B_KF + t % kStages), (t / kStages) & 1, abort_flag, a.status))) break;
                tc_fence_after();
                qk(t);
            }
            for (int i = 0; ok && i < T; ++i) {
                if (!(ok = mbar_wait(bar(B_P + (i & 1)), (i >> 1) & 1, abort_flag, a.status))) break;
                if (!(ok = mbar_wait(bar(B_VF + i % kStages), (i / kStages) & 1, abort_flag, a.status))) break;
                tc_fence_after();
                pv(i);
                const int t2 = i + 2;
                if (t2 < T) {
                    if (!(ok = mbar_wait(bar(B_KF + t2 % kStages), (t2 / kStages) & 1, abort_flag, a.status))) break;
                    tc_fence_after();
                    qk(t2);
                }
            }
            // drain: every MMA issued above has completed once this arrives
            // (waited on even after an abort: TMEM is freed only after it)
            mma_commit(bar(B_END));
            volatile int never = 0;
            mbar_wait(bar(B_END), 0, &never, a.status);
        }
    } else if (warp < 4) {
        asm volatile("setmaxnreg.dec.sync.aligned.u32 %0;" ::"n"(kRegsProducer));
    } else {
        // ---- softmax warpgroup ----------------------------------------------
        asm volatile("setmaxnreg.inc.sync.aligned.u32 %0;" ::"n"(kRegsSoftmax));
        const int q4 = warp & 3;                         // TMEM lane quarter of this warp
        const int r = 32 * q4 + lane;                    // row within the M tile
        const uint32_t lane_off = (uint32_t)(32 * q4) << 16;
        const uint32_t tM = tmem + lane_off, tO = tM + 128;
        int head, ri;
        if (s.bs == 64) { head = h0 + (r >> 6); ri = r & 63; }
        else { head = h0; ri = r; }
        const int qi = j * s.bs + ri;                    // query position of this row
        const bool causal = s.flags & SA_CAUSAL;
        float m_run = -CUDART_INF_F, l = 0.f;
        bool ok = true;
        // hierarchical mode ([HiLS]): every block gets its own softmax, and the
        // block outputs are weighted by softmax_b(s_b).  With M the largest
        // retrieval score of the list (known before the first tile), block b
        // enters O as P_b V_b * 2^(s_b - M) / l_b and W sums 2^(s_b - M), so
        // O never needs rescaling and the result is O / W.
        const bool hier = s.flags & SA_HIER;
        float mh = -CUDART_INF_F;
        if (hier) {
            for (int c = 0; c < cnt; ++c)
                if (blk_s[c] >= 0) mh = fmaxf(mh, gate_s[c]);
            m_run = mh;
        }
        for (int i = 0; i < T; ++i) {
            const uint32_t tS = tM + (i & 1) * 64;
            ok = mbar_wait(bar(B_S + (i & 1)), (i >> 1) & 1, abort_flag, a.status);
            if (!__all_sync(0xffffffffu, ok)) { ok = false; break; }
            tc_fence_after();
            float x[64];
            tmem_ld32(tS, x);
            tmem_ld32(tS + 32, x + 32);
            tmem_wait_ld();
            reg_fence<64>(x);
            const int c = i / sub;
            const int blk = blk_s[c];
            const float gl = gate_s[c];
            const int t0 = blk * s.bs + (i % sub) * 64;  // first key of this tile
            // masks: a bad list entry, the ragged end of the sequence, causality in the local block
            const bool masked = blk < 0 || t0 + 64 > s.N || (causal && blk == j);
            if (masked) {
#pragma unroll
                for (int k = 0; k < 64; ++k) {
                    const int t = t0 + k;
                    const bool vis = blk >= 0 && t < s.N && !(causal && blk == j && t > qi);
                    x[k] = vis ? x[k] : -CUDART_INF_F;
                }
            }
            // row max: eight independent chains, then a three-level tree
            float mq[8];
#pragma unroll
            for (int e = 0; e < 8; ++e) mq[e] = x[e];
#pragma unroll
            for (int k = 8; k < 64; k += 8)
#pragma unroll
                for (int e = 0; e < 8; ++e) mq[e] = fmaxf(mq[e], x[k + e]);
#pragma unroll
            for (int w = 4; w > 0; w >>= 1)
#pragma unroll
                for (int e = 0; e < w; ++e) mq[e] = fmaxf(mq[e], mq[e + w]);
            float mx = mq[0];
            mx = mx == -CUDART_INF_F ? mx : fmaf(mx, qk_scale, gl);
            if (hier) {
                // this block's own softmax (scores without gate), weighted by its retrieval score
                const float mb = mx == -CUDART_INF_F ? 0.f : mx - gl;   // mx carried the score: drop it
                float lb = 0.f;
#pragma unroll
                for (int k = 0; k < 64; ++k) {
                    x[k] = ex2(fmaf(x[k], qk_scale, -mb));
                    lb += x[k];
                }
                const float wb = lb > 0.f ? ex2(gl - mh) : 0.f;
                const float f = lb > 0.f ? wb / lb : 0.f;
                l += wb;
                uint32_t pk[32];
#pragma unroll
                for (int k = 0; k < 32; ++k) {
                    __nv_bfloat162 h2 = __floats2bfloat162_rn(x[2 * k] * f, x[2 * k + 1] * f);
                    pk[k] = *reinterpret_cast<uint32_t *>(&h2);
                }
                tmem_st32(tS, pk);
                tmem_wait_st();
                tc_fence_before();
                mbar_arrive(bar(B_P + (i & 1)));
                continue;
            }
            const float m_new = fmaxf(m_run, mx);
            if (i == 0) {
                m_run = m_new;
            } else {
                const bool need = m_new > m_run + 8.f;
                if (__any_sync(0xffffffffu, need)) {
                    // PV(i-2) is done (S(i) was computed after it), so PV(i-1)
                    // is either running or done: parity (i-1) is unambiguous
                    ok = mbar_wait(bar(B_O), (i - 1) & 1, abort_flag, a.status);
                    if (!__all_sync(0xffffffffu, ok)) { ok = false; break; }
                    tc_fence_after();
                    const float corr = need ? ex2(m_run - m_new) : 1.f;
                    if (need) {
                        l *= corr;
                        m_run = m_new;
                    }
#pragma unroll
                    for (int cc = 0; cc < 4; ++cc) {
                        float o[32];
                        tmem_ld32(tO + 32 * cc, o);
                        tmem_wait_ld();
                        reg_fence<32>(o);
                        uint32_t w[32];
#pragma unroll
                        for (int k = 0; k < 32; ++k) w[k] = __float_as_uint(o[k] * corr);
                        tmem_st32(tO + 32 * cc, w);
                    }
                    tmem_wait_st();
                }
            }
            // p = 2^(x * scale + gate - ref): one FFMA and one ex2 per element
            const float bias = gl - (m_run == -CUDART_INF_F ? 0.f : m_run);
            uint32_t pk[32];
            float ls = 0.f;
#pragma unroll
            for (int k = 0; k < 32; ++k) {
                const float p0 = ex2(fmaf(x[2 * k], qk_scale, bias)), p1 = ex2(fmaf(x[2 * k + 1], qk_scale, bias));
                ls += p0 + p1;
                __nv_bfloat162 h2 = __floats2bfloat162_rn(p0, p1);
                pk[k] = *reinterpret_cast<uint32_t *>(&h2);
            }
            l += ls;
            tmem_st32(tS, pk);
            tmem_wait_st();
            tc_fence_before();
            mbar_arrive(bar(B_P + (i & 1)));
        }
        // ---- epilogue: O / l -> bf16, LSE ---------------------------------
        // O is final once the MMA thread's drain barrier (committed after its
        // last MMA) completes: a single phase, so no parity can alias.  The
        // per-PV barrier would not do here -- up to two of its phases may
        // still be pending, and a parity wait cannot tell them apart.
        const bool have = T > 0 && ok;
        if (have) {
            ok = mbar_wait(bar(B_END), 0, abort_flag, a.status);
            ok = __all_sync(0xffffffffu, ok);
            tc_fence_after();
        }
        const bool row_ok = qi < s.N;
        __nv_bfloat16 *orow = a.O + (((size_t)b * s.Hq + head) * s.N + (row_ok ? qi : 0)) * 128;
        const float inv = (l > 0.f) ? 1.f / l : 0.f;
#pragma unroll
        for (int cc = 0; cc < 4; ++cc) {
            float o[32];
            if (have && ok) {
                tmem_ld32(tO + 32 * cc, o);
                tmem_wait_ld();
                reg_fence<32>(o);
            } else {
#pragma unroll
                for (int k = 0; k < 32; ++k) o[k] = 0.f;
            }
            if (row_ok) {
#pragma unroll
                for (int v = 0; v < 32; v += 8) {
                    float f[8];
#pragma unroll
                    for (int k = 0; k < 8; ++k) f[k] = o[v + k] * inv;
                    store16(orow + 32 * cc + v, f);
                }
            }
        }
        if (row_ok)
            a.lse[((size_t)b * s.Hq + head) * s.N + qi] =
                (l > 0.f && ok) ? (m_run + log2f(l)) * kLn2 : -CUDART_INF_F;
    }

    // ---- teardown -----------------------------------------------------------
    tc_fence_before();
    __syncthreads();
    if (warp == 1) {
        tc_fence_after();
        asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(tmem), "n"(kTmemCols));
    }
}

// ---------------------------------------------------------------------------
// host side
// ---------------------------------------------------------------------------
}  // namespace

bool prefill_tc_supported(const Shape &s) {
    if (s.dtype != SA_BF16 || s.d != 128) return false;
    if (s.flags & SA_SELECT_PER_QHEAD) return false;
    if ((s.flags & SA_HIER) && s.bs != 64) return false;   // hierarchical: one block per key tile
    if (s.bs != 64 && s.bs != 128) return false;
    const int hc = 128 / s.bs;   // query heads per CTA
    if (s.G % hc) return false;
    if (s.cap > kMaxList) return false;
    const char *e = getenv("SPARSE_ATTN_PREFILL_PATH");
    if (e && strcmp(e, "simt") == 0) return false;
    return true;
}

cudaError_t launch_prefill_tc(const Shape &s, const void *Q, const void *K, const void *V, const int32_t *idx,
                              const float *score, const int32_t *count, void *O, float *lse, unsigned *status,
                              cudaStream_t st) {
    // The register split assumes a launch at exactly kRegsLaunch registers
    // per thread; anything else could stall the register exchange.
    cudaFuncAttributes fa;
    cudaError_t fe = cudaFuncGetAttributes(&fa, prefill_tc_kernel);
    if (fe != cudaSuccess) return fe;
    if (fa.numRegs != kRegsLaunch) return cudaErrorInvalidDeviceFunction;
    CUtensorMap mq, mk, mv;
    const uint64_t qrows = (uint64_t)s.B * s.Hq * s.N, krows = (uint64_t)s.B * s.Hkv * s.N;
    if (!make_map_d128(&mq, Q, qrows, 64) || !make_map_d128(&mk, K, krows, 64) ||
        !make_map_d128(&mv, V, krows, 64))
        return cudaErrorInvalidValue;
    TcArgs a{};
    a.s = s;
    a.idx = idx;
    a.score = score;
    a.count = count;
    a.O = (__nv_bfloat16 *)O;
    a.lse = lse;
    a.status = status;
    a.hc = 128 / s.bs;
    a.npair = s.G / a.hc;
    cudaError_t e = cudaFuncSetAttribute(prefill_tc_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                         (int)kSmemBytes);
    if (e != cudaSuccess) return e;
    const unsigned grid = (unsigned)((size_t)s.B * s.Hkv * s.nb * a.npair);
    prefill_tc_kernel<<<grid, kThreads, kSmemBytes, st>>>(mq, mk, mv, a);
    note_launch();
    return cudaGetLastError();
}

}  // namespace sa
