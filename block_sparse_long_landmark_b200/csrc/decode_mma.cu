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
// once.  A CTA (unit, split) owns up to `bps` kept blocks of one (batch,
// kv-head) list.  Warp 0 streams them with cp.async.bulk.tensor (128-byte
// swizzle) into a shared-memory ring with one stage per consumer warp (three
// CTAs fit an SM); consumer warps take whole blocks round-robin and compute,
// with mma.sync m16n8k16 bf16 tiles,
//   S[16 x 64] = q[16 x 128] K_b^T     (rows = the group's query heads, padded)
//   O[16 x 128] += P[16 x 64] V_b      (P straight from S's registers)
// keeping a per-warp online softmax.  The warps' states are merged in shared
// memory and the CTA leaves (max, sum, acc) per head for the split merge, or
// the final output when the list fits one CTA.
#include <cuda.h>
#include <cudaTypedefs.h>
#include <math_constants.h>

#include <cstdlib>
#include <cstring>
#include <mutex>

#include "common.cuh"

namespace sa {
namespace {

constexpr int kNW = 2;                          // consumer warps
constexpr int kThreadsD = 32 * (kNW + 1);
constexpr int kNST = 2;                         // ring stages
// Block li goes to stage li % kNST and to consumer warp li % kNW.  With
// kNST a multiple of kNW every stage has a single consumer warp, which waits
// on its phases strictly in order; a shared stage would let one warp wait on a
// parity two phases ahead of the barrier and pass before its data landed.
static_assert(kNST % kNW == 0, "each ring stage must belong to one consumer warp");
constexpr uint32_t kHalf = 64 * 128;            // one 64-row x 64-col bf16 box (8 KB)
constexpr uint32_t kBlockBytes = 2 * kHalf;     // 64 x 128 bf16 (16 KB)
constexpr uint32_t kStageBytes = 2 * kBlockBytes;  // K + V
constexpr uint32_t kBarOffD = kNST * kStageBytes;
constexpr int kMaxBps = 64;
constexpr uint32_t kSmemD = kBarOffD + 256 + 8 * kMaxBps + 1024;
constexpr unsigned long long kWaitNsD = 2000000000ull;

struct DmArgs {
    Shape s;
    const __nv_bfloat16 *q;
    const int32_t *idx;
    const float *score;
    const int32_t *count;
    __nv_bfloat16 *o;
    float *lse;
    unsigned *status;
    float *part;
    int S, bps;
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

__global__ void __launch_bounds__(kThreadsD, 3)
decode_mma_kernel(const __grid_constant__ CUtensorMap tmK, const __grid_constant__ CUtensorMap tmV, DmArgs a) {
    constexpr float kLog2e = 1.4426950408889634f;
    constexpr float kLn2 = 0.6931471805599453f;
    const Shape &s = a.s;
    extern __shared__ unsigned char dsm_raw[];
    unsigned char *sm = reinterpret_cast<unsigned char *>((reinterpret_cast<uintptr_t>(dsm_raw) + 1023) &
                                                          ~uintptr_t(1023));
    const uint32_t sb = su32(sm);
    uint64_t *bars = reinterpret_cast<uint64_t *>(sm + kBarOffD);      // full[kNST], empty[kNST]
    volatile int *abort_flag = reinterpret_cast<volatile int *>(sm + kBarOffD + 8 * 2 * kNST);
    int *blk_s = reinterpret_cast<int *>(sm + kBarOffD + 256);
    float *gate_s = reinterpret_cast<float *>(sm + kBarOffD + 256 + 4 * kMaxBps);

    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const int u = blockIdx.x / a.S, split = blockIdx.x % a.S;
    const int hs = u % s.Hsel, b = u / s.Hsel;
    const bool perq = s.flags & SA_SELECT_PER_QHEAD;
    const int g = perq ? hs / s.G : hs;
    const int h0 = perq ? hs : hs * s.G;
    const int HP = s.heads_per;
    const int32_t *il = a.idx + (size_t)u * s.cap;
    const float *sl = a.score + (size_t)u * s.cap;
    const int cnt = max(0, min(a.count[u], s.cap));
    const int nseq = seq_n(s, b);                       // this sequence's context length
    const int local = (nseq - 1) / 64;
    const int c0 = split * a.bps, c1 = min(cnt, c0 + a.bps);
    const int nloc = max(0, c1 - c0);
    const bool hier = s.flags & SA_HIER;

    if (tid == 0) {
        for (int i = 0; i < kNST; ++i) {
            asm volatile("mbarrier.init.shared::cta.b64 [%0], 1;" ::"r"(su32(&bars[i])));
            asm volatile("mbarrier.init.shared::cta.b64 [%0], 1;" ::"r"(su32(&bars[kNST + i])));
        }
        *abort_flag = 0;
        asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
    }
    for (int li = tid; li < nloc; li += kThreadsD) {
        const int c = c0 + li;
        const int blk = il[c];
        const bool ok = blk >= 0 && blk <= local && (c == 0 || il[c - 1] < blk);
        if (!ok) set_status(a.status, kStatusBadIndex);
        blk_s[li] = ok ? blk : -1;
        const bool forced = (blk == local && (s.flags & SA_LOCAL)) || (blk == 0 && (s.flags & SA_SINK));
        // gated: log2-unit gate; hierarchical: log2-unit retrieval score
        gate_s[li] = hier ? sl[c] * kLog2e
                          : (((s.flags & SA_GATE) && !forced) ? log_sigmoid(sl[c] - sl[cnt - 1]) * kLog2e : 0.f);
    }
    __syncthreads();

    float *mrg = reinterpret_cast<float *>(sm);   // merge area, reuses the ring after the loop
    if (warp == 0) {
        // ---- producer -------------------------------------------------------
        if (lane == 0) {
            const int kvbase = (b * s.Hkv + g) * s.N;
            int issued = 0;
            for (int li = 0; li < nloc; ++li) {
                const int st = li % kNST;
                if (li >= kNST &&
                    !wait_bar(su32(&bars[kNST + st]), ((li / kNST) - 1) & 1, abort_flag, a.status))
                    break;
                const uint32_t full = su32(&bars[st]);
                asm volatile("mbarrier.arrive.expect_tx.shared::cta.b64 _, [%0], %1;" ::"r"(full), "r"(kStageBytes)
                             : "memory");
                const int y = kvbase + max(0, blk_s[li]) * 64;
                const uint32_t dst = sb + st * kStageBytes;
#pragma unroll
                for (int ch = 0; ch < 2; ++ch) {
                    asm volatile(
                        "cp.async.bulk.tensor.2d.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1, {%3, "
                        "%4}], [%2];" ::"r"(dst + ch * kHalf),
                        "l"(reinterpret_cast<uint64_t>(&tmK)), "r"(full), "r"(64 * ch), "r"(y)
                        : "memory");
                    asm volatile(
                        "cp.async.bulk.tensor.2d.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1, {%3, "
                        "%4}], [%2];" ::"r"(dst + kBlockBytes + ch * kHalf),
                        "l"(reinterpret_cast<uint64_t>(&tmV)), "r"(full), "r"(64 * ch), "r"(y)
                        : "memory");
                }
                issued = li + 1;
            }
            if (*abort_flag) {
                volatile int never = 0;
                for (int li = max(0, issued - kNST); li < issued; ++li)
                    wait_bar(su32(&bars[li % kNST]), (li / kNST) & 1, &never, a.status);
            }
        }
        __syncwarp();
    }
    // consumer state (rows g and g+8 of the 16-row tile = query heads)
    const int gq = lane >> 2, tq = lane & 3;
    float m_r[2] = {-CUDART_INF_F, -CUDART_INF_F}, l_r[2] = {0.f, 0.f};
    float oacc[16][4];
#pragma unroll
    for (int i = 0; i < 16; ++i) oacc[i][0] = oacc[i][1] = oacc[i][2] = oacc[i][3] = 0.f;
    if (warp > 0) {
        const int cw = warp - 1;
        // q fragments: rows = heads h0 + row (row < HP), 8 k-steps of 16 dims
        uint32_t qa[8][4];
#pragma unroll
        for (int ks = 0; ks < 8; ++ks) {
#pragma unroll
            for (int rr = 0; rr < 2; ++rr) {
                const int row = gq + 8 * rr;
                const bool valid = row < HP;
                const __nv_bfloat16 *qr = a.q + ((size_t)b * s.Hq + h0 + (valid ? row : 0)) * 128 + 16 * ks + 2 * tq;
                const uint32_t lo = valid ? *reinterpret_cast<const uint32_t *>(qr) : 0u;
                const uint32_t hi = valid ? *reinterpret_cast<const uint32_t *>(qr + 8) : 0u;
                qa[ks][rr] = lo;       // a0 (row g) / a1 (row g+8)
                qa[ks][2 + rr] = hi;   // a2 / a3
            }
        }
        const float qk_scale = s.scale * kLog2e;
        bool ok = true;
        for (int li = cw; li < nloc && ok; li += kNW) {
            const int st = li % kNST;
            ok = wait_bar(su32(&bars[st]), (li / kNST) & 1, abort_flag, a.status);
            if (!__all_sync(0xffffffffu, ok)) { ok = false; break; }
            const uint32_t kb = sb + st * kStageBytes, vb = kb + kBlockBytes;
            const int blk = blk_s[li];
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
                    mma16816(sacc[nt], qa[2 * pch + 1][0], qa[2 * pch + 1][1], qa[2 * pch + 1][2],
                             qa[2 * pch + 1][3], r2, r3);
                }
            }
            // logits (log2 units), masks, block max per row
            const float gl = gate_s[li];
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
        }
        if (!hier) {
#pragma unroll
            for (int rr = 0; rr < 2; ++rr) {
                l_r[rr] += __shfl_xor_sync(0xffffffffu, l_r[rr], 1);
                l_r[rr] += __shfl_xor_sync(0xffffffffu, l_r[rr], 2);
            }
        }
    }
    // ---- merge the consumer warps (all CTA threads reach the barriers) ------
    __syncthreads();
    // layout: per warp cw: m[16], l[16], O[16][128]
    constexpr int kWarpFloats = 32 + 16 * 128;
    if (warp > 0) {
        float *w = mrg + (warp - 1) * kWarpFloats;
        if (tq == 0) {
            w[gq] = m_r[0];
            w[gq + 8] = m_r[1];
            w[16 + gq] = l_r[0];
            w[16 + gq + 8] = l_r[1];
        }
#pragma unroll
        for (int nd = 0; nd < 16; ++nd) {
            const int dim = 8 * nd + 2 * tq;
            w[32 + gq * 128 + dim] = oacc[nd][0];
            w[32 + gq * 128 + dim + 1] = oacc[nd][1];
            w[32 + (gq + 8) * 128 + dim] = oacc[nd][2];
            w[32 + (gq + 8) * 128 + dim + 1] = oacc[nd][3];
        }
    }
    __syncthreads();
    for (int e = tid; e < HP * 128; e += kThreadsD) {
        const int hh = e >> 7, dim = e & 127;
        float M = -CUDART_INF_F;
        for (int w = 0; w < kNW; ++w) M = fmaxf(M, mrg[w * kWarpFloats + hh]);
        float L = 0.f, O = 0.f;
        if (M != -CUDART_INF_F) {
            for (int w = 0; w < kNW; ++w) {
                const float *ww = mrg + w * kWarpFloats;
                if (ww[hh] == -CUDART_INF_F) continue;
                const float f = ex2f(ww[hh] - M);
                L = fmaf(ww[16 + hh], f, L);
                O = fmaf(ww[32 + hh * 128 + dim], f, O);
            }
        }
        if (a.S == 1) {
            a.o[((size_t)b * s.Hq + h0 + hh) * 128 + dim] = __float2bfloat16_rn(L > 0.f ? O / L : 0.f);
            if (dim == 0)
                a.lse[(size_t)b * s.Hq + h0 + hh] = L > 0.f ? (M + log2f(L)) * kLn2 : -CUDART_INF_F;
        } else {
            float *pp = a.part + (((size_t)u * a.S + split) * HP + hh) * 130;
            pp[2 + dim] = O;
            if (dim == 0) {
                pp[0] = M;
                pp[1] = L;
            }
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

size_t decode_mma_partial_bytes(const Shape &s, int S) {
    return (((size_t)s.B * s.Hsel * S * s.heads_per * 130 * sizeof(float)) + 255) & ~(size_t)255;
}

void decode_mma_geometry(const Shape &s, int &S, int &bps) {
    const int units = s.B * s.Hsel;
    const int want = (3 * 3 * 148 + units - 1) / units;      // about three waves of 3 CTAs per SM
    S = max(1, min(want, (s.cap + 5) / 6));
    bps = (s.cap + S - 1) / S;
    if (bps > kMaxBps) bps = kMaxBps;
    S = (s.cap + bps - 1) / bps;
}

cudaError_t launch_decode_mma(const Shape &s, const void *q, const void *K, const void *V, const int32_t *idx,
                              const float *score, const int32_t *count, void *o, float *lse, unsigned *status,
                              float *part, cudaStream_t st, int &S_out) {
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
    a.o = (__nv_bfloat16 *)o;
    a.lse = lse;
    a.status = status;
    a.part = part;
    decode_mma_geometry(s, a.S, a.bps);
    S_out = a.S;
    cudaError_t e = cudaFuncSetAttribute(decode_mma_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)kSmemD);
    if (e != cudaSuccess) return e;
    decode_mma_kernel<<<(unsigned)(s.B * s.Hsel * a.S), kThreadsD, kSmemD, st>>>(mk, mv, a);
    note_launch();
    return cudaGetLastError();
}

}  // namespace sa
