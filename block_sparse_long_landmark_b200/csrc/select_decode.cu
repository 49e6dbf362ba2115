// select_decode.cu -- decode selection with a warp per chunk of candidates.
//
// [SAS] opening section / "Ключевые факты": a light selector scores the
// context blocks and a hard top-K keeps the best; the current block is
// always kept.  The Latent Sparse Attention post ("Индекс перестаёт
// перебирать весь контекст"): the start of the context is always added.
//
// Decode scans every landmark of a sequence once per step, so the step is a
// stream of landmarks from HBM.  Here each warp owns a chunk of 256
// candidate blocks of one (batch, selection head): it averages the unit's
// query heads (every lane its own 16-byte slice), streams the chunk's
// landmarks with 16-byte loads (a VPR-lane group per row, eight rows per
// group in flight), scores them in fp32 and takes the chunk's top-K with
// the warp-level bitwise select (warp_select.cuh) -- no block-wide barrier,
// so one warp's selection overlaps the other warps' streaming.  Warp 0 then
// merges the CTA's eight chunk lists; when a unit spans several CTAs, each
// leaves its list in the workspace and the unit's last CTA to finish merges
// them.  The candidates sit in index order throughout and every select takes
// equal keys at the lower position, so the result is the exact top-K by
// (score desc, index asc) whatever the split.
#include <cstdlib>
#include <cstring>

#include "common.cuh"
#include "warp_select.cuh"

namespace sa {
namespace {

constexpr int kSdThreads = 256;
constexpr int kSdWarps = kSdThreads / 32;
constexpr int kSdChunk = 256;        // candidates per warp
constexpr int kSdMaxMerge = 4096;    // candidates the cross-CTA merge holds in shared memory

struct SdArgs {
    Shape s;
    const void *q;        // [B,Hq,d]
    const void *L;        // [B,Hkv,nb,d]
    int32_t *idx;
    float *score;
    int32_t *count;
    unsigned *status;
    uint32_t *pkey;       // [units][C][top_k] per-CTA candidates (keys)
    int32_t *pidx;        // [units][C][top_k] per-CTA candidates (block ids)
    int32_t *pcnt;        // [units][C] candidates per CTA
    float *special;       // [units][2]: s_0, s_local
    unsigned *done;       // [units] CTAs finished; back to 0 by the merging CTA
    int C;                // CTAs per unit
};

struct SdSmem {
    float s_special[2];
    int nv[kSdWarps];
    int last;
};

// Final list of unit u: [0 (sink)] + selected (ascending) + [local].
__device__ void write_list(const SdArgs &a, int u, int local, const int *sel_idx, const uint32_t *sel_key, int nsel,
                           float s0, float sloc) {
    const Shape &s = a.s;
    int32_t *idx = a.idx + (size_t)u * s.cap;
    float *sc = a.score + (size_t)u * s.cap;
    const bool sink = s.flags & SA_SINK;
    const bool loc = (s.flags & SA_LOCAL) && !(sink && local == 0);
    const int off = sink ? 1 : 0;
    const int cnt = off + nsel + (loc ? 1 : 0);
    for (int i = threadIdx.x & 31; i < s.cap; i += 32) {
        int bi = -1;
        float sv = 0.f;
        if (i < cnt) {
            if (sink && i == 0) { bi = 0; sv = s0; }
            else if (loc && i == cnt - 1) { bi = local; sv = sloc; }
            else { bi = sel_idx[i - off]; sv = key_to_float(sel_key[i - off]); }
        }
        idx[i] = bi;
        sc[i] = sv;
    }
    if ((threadIdx.x & 31) == 0) a.count[u] = cnt;
}

template <typename T, int VPR>
__global__ void __launch_bounds__(kSdThreads, 4) select_decode_kernel(SdArgs a) {
    constexpr int EPV = Vec<T>::n;
    constexpr int RPW = 32 / VPR;            // rows per warp step
    constexpr int U = 8;                     // steps in flight
    const Shape &s = a.s;
    const int D = VPR * EPV;
    extern __shared__ __align__(16) unsigned char smraw[];
    SdSmem &sm = *reinterpret_cast<SdSmem *>(smraw);
    uint32_t *keys = reinterpret_cast<uint32_t *>(smraw + ((sizeof(SdSmem) + 15) & ~15));   // [8][256]
    int *wpos = reinterpret_cast<int *>(keys + kSdWarps * kSdChunk);                          // [8][256]
    uint32_t *mkey = reinterpret_cast<uint32_t *>(wpos + kSdWarps * kSdChunk);                // [merge]
    int *midx = reinterpret_cast<int *>(mkey + max(kSdWarps, a.C) * s.top_k);                // [merge]
    int *mpos = midx + max(kSdWarps, a.C) * s.top_k;                                          // [top_k]

    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int u = blockIdx.x / a.C, cta = blockIdx.x % a.C;
    const int hs = u % s.Hsel, b = u / s.Hsel;
    const bool perq = s.flags & SA_SELECT_PER_QHEAD;
    const int g = perq ? hs / s.G : hs;
    const int hq0 = perq ? hs : hs * s.G;
    const int local = (seq_n(s, b) - 1) / s.bs;
    const int first = (s.flags & SA_SINK) ? 1 : 0;
    const int ncand = max(0, local - first);
    const int c0 = first + (cta * kSdWarps + warp) * kSdChunk;      // this warp's first candidate
    const int n = max(0, min(local, c0 + kSdChunk) - c0);

    // the unit's pooled query: lane group member cv holds elements cv*EPV ..
    const int sub = lane / VPR, cv = lane % VPR;
    float qv[EPV];
#pragma unroll
    for (int i = 0; i < EPV; ++i) qv[i] = 0.f;
    for (int hh = 0; hh < s.heads_per; ++hh) {
        float f[EPV];
        load16((const T *)a.q + ((size_t)b * s.Hq + hq0 + hh) * D + cv * EPV, f);
#pragma unroll
        for (int i = 0; i < EPV; ++i) qv[i] += f[i];
    }
#pragma unroll
    for (int i = 0; i < EPV; ++i) qv[i] /= (float)s.heads_per;
    const T *Lg = (const T *)a.L + ((size_t)b * s.Hkv + g) * s.nb * D;

    // ---- this warp's chunk: scores, then its top-K -------------------------
    uint32_t *kw = keys + warp * kSdChunk;
    int *pw = wpos + warp * kSdChunk;
    bool nan_seen = false;
    for (int r0 = 0; r0 < n; r0 += RPW * U) {
        uint4 raw[U];
#pragma unroll
        for (int uu = 0; uu < U; ++uu) {
            const int r = min(r0 + sub + RPW * uu, n - 1);
            raw[uu] = *reinterpret_cast<const uint4 *>(Lg + (size_t)(c0 + r) * D + cv * EPV);
        }
#pragma unroll
        for (int uu = 0; uu < U; ++uu) {
            float f[EPV];
            load16(reinterpret_cast<const T *>(&raw[uu]), f);
            float dot = 0.f;
#pragma unroll
            for (int i = 0; i < EPV; ++i) dot = fmaf(qv[i], f[i], dot);
#pragma unroll
            for (int o = VPR / 2; o > 0; o >>= 1) dot += __shfl_xor_sync(0xffffffffu, dot, o);
            const int r = r0 + sub + RPW * uu;
            if (cv == 0 && r < n) {
                const float sc = s.scale * dot;
                nan_seen |= isnan(sc);
                kw[r] = ord_key(sc);
            }
        }
    }
    __syncwarp();
    const int nsel = warp_topk_positions<8>(kw, n, s.top_k, pw);
    // the warp's list (ascending block ids) into the CTA's merge area
    for (int i = lane; i < nsel; i += 32) {
        mkey[warp * s.top_k + i] = kw[pw[i]];
        midx[warp * s.top_k + i] = c0 + pw[i];
    }
    if (lane == 0) sm.nv[warp] = nsel;
    // the sink and local scores (one warp of the unit's first CTA)
    if (cta == 0 && warp == 0) {
#pragma unroll
        for (int e = 0; e < 2; ++e) {
            const int blk = e == 0 ? 0 : local;
            float f[EPV];
            load16(Lg + (size_t)blk * D + cv * EPV, f);
            float dot = 0.f;
#pragma unroll
            for (int i = 0; i < EPV; ++i) dot = fmaf(qv[i], f[i], dot);
#pragma unroll
            for (int o = VPR / 2; o > 0; o >>= 1) dot += __shfl_xor_sync(0xffffffffu, dot, o);
            if (lane == 0) {
                sm.s_special[e] = s.scale * dot;
                nan_seen |= isnan(s.scale * dot);
            }
        }
    }
    if (nan_seen) set_status(a.status, kStatusNaN);
    __syncthreads();

    // ---- warp 0: the CTA's list, then the unit's ---------------------------
    if (warp != 0) return;
    // pack the lists in warp (= index) order; a list only moves down (the
    // lists before it hold at most top_k entries each), read before written
    int ntot = 0;
    for (int w = 0; w < kSdWarps; ++w) {
        const int m = sm.nv[w];
        for (int i0 = 0; i0 < m; i0 += 32) {
            const int i = i0 + lane;
            uint32_t k = 0u;
            int id = 0;
            if (i < m) {
                k = mkey[w * s.top_k + i];
                id = midx[w * s.top_k + i];
            }
            __syncwarp();
            if (i < m) {
                mkey[ntot + i] = k;
                midx[ntot + i] = id;
            }
            __syncwarp();
        }
        ntot += m;
    }
    const int nc = warp_topk_positions<8>(mkey, ntot, s.top_k, mpos);
    if (a.C == 1) {
        // one CTA per unit: its list is the unit's
        int *sel_idx = wpos;                    // reuse: this CTA's other buffers are free now
        uint32_t *sel_key = keys;
        for (int i = lane; i < nc; i += 32) {
            sel_idx[i] = midx[mpos[i]];
            sel_key[i] = mkey[mpos[i]];
        }
        __syncwarp();
        write_list(a, u, local, sel_idx, sel_key, nc, sm.s_special[0], sm.s_special[1]);
        return;
    }
    {
        uint32_t *pk = a.pkey + ((size_t)u * a.C + cta) * s.top_k;
        int32_t *pi = a.pidx + ((size_t)u * a.C + cta) * s.top_k;
        for (int i = lane; i < nc; i += 32) {
            pk[i] = mkey[mpos[i]];
            pi[i] = midx[mpos[i]];
        }
        if (lane == 0) {
            a.pcnt[(size_t)u * a.C + cta] = nc;
            if (cta == 0) {
                a.special[(size_t)u * 2] = sm.s_special[0];
                a.special[(size_t)u * 2 + 1] = sm.s_special[1];
            }
        }
    }
    // the unit's last CTA to finish merges (writes fenced before the count)
    __threadfence();
    __syncwarp();
    int last = 0;
    if (lane == 0) last = atomicAdd(a.done + u, 1u) == (unsigned)(a.C - 1);
    last = __shfl_sync(0xffffffffu, last, 0);
    if (!last) return;
    __threadfence();
    ntot = 0;
    for (int c = 0; c < a.C; ++c) {
        const int m = __ldcg(a.pcnt + (size_t)u * a.C + c);
        for (int i = lane; i < m; i += 32) {
            const size_t src = ((size_t)u * a.C + c) * s.top_k + i;
            mkey[ntot + i] = __ldcg(a.pkey + src);
            midx[ntot + i] = __ldcg(a.pidx + src);
        }
        ntot += m;
    }
    __syncwarp();
    const int nf = warp_topk_positions<0>(mkey, ntot, s.top_k, mpos);
    int *sel_idx = wpos;
    uint32_t *sel_key = keys;
    for (int i = lane; i < nf; i += 32) {
        sel_idx[i] = midx[mpos[i]];
        sel_key[i] = mkey[mpos[i]];
    }
    __syncwarp();
    write_list(a, u, local, sel_idx, sel_key, nf, __ldcg(a.special + (size_t)u * 2),
               __ldcg(a.special + (size_t)u * 2 + 1));
    if (lane == 0) a.done[u] = 0u;
    (void)ncand;
}

}  // namespace

// Geometry: warp-chunks per unit cover the largest candidate count (the
// full context), grouped eight to a CTA.
static void sd_geometry(const Shape &s, int &C) {
    const int first = (s.flags & SA_SINK) ? 1 : 0;
    const int ncand = max(1, (s.N - 1) / s.bs - first);
    const int W = (ncand + kSdChunk - 1) / kSdChunk;
    C = (W + kSdWarps - 1) / kSdWarps;
}

bool select_force_chunked() {
    const char *e = getenv("SPARSE_ATTN_SELECT_PATH");
    return e && strcmp(e, "chunked") == 0;
}

bool select_decode_supported(const Shape &s) {
    if (s.top_k < 1 || s.top_k > kSdChunk) return false;
    int C;
    sd_geometry(s, C);
    return C == 1 || (long long)C * s.top_k <= kSdMaxMerge;
}

size_t select_decode_workspace(const Shape &s) {
    int C;
    sd_geometry(s, C);
    if (C == 1) return 0;
    const size_t units = (size_t)s.B * s.Hsel;
    return units * C * s.top_k * 8 + units * C * 4 + units * 2 * 4 + 4 * 256;
}

static size_t sd_smem(const Shape &s, int C) {
    const size_t merge = (size_t)max(kSdWarps, C) * s.top_k;
    return ((sizeof(SdSmem) + 15) & ~(size_t)15) + (size_t)kSdWarps * kSdChunk * 8 + merge * 8 + (size_t)s.top_k * 4;
}

template <typename T>
static cudaError_t run_sd(const Shape &s, const void *q, const void *L, int32_t *idx, float *score, int32_t *count,
                          void *ws, cudaStream_t st) {
    SdArgs a{};
    a.s = s;
    a.q = q;
    a.L = L;
    a.idx = idx;
    a.score = score;
    a.count = count;
    a.status = (unsigned *)ws;
    sd_geometry(s, a.C);
    const size_t units = (size_t)s.B * s.Hsel;
    if (a.C > 1) {
        char *p = (char *)ws + ws_layout(s).scratch;
        auto take = [&](size_t bytes) {
            char *r = p;
            p += (bytes + 255) & ~(size_t)255;
            return r;
        };
        a.pkey = (uint32_t *)take(units * a.C * s.top_k * 4);
        a.pidx = (int32_t *)take(units * a.C * s.top_k * 4);
        a.pcnt = (int32_t *)take(units * a.C * 4);
        a.special = (float *)take(units * 2 * 4);
        a.done = (unsigned *)((char *)ws + ws_layout(s).sel_decode);
    }
    const int vpr = s.d * (int)sizeof(T) / 16;
    void (*kern)(SdArgs) = nullptr;
    switch (vpr) {
        case 8: kern = select_decode_kernel<T, 8>; break;
        case 16: kern = select_decode_kernel<T, 16>; break;
        case 32: kern = select_decode_kernel<T, 32>; break;
        default: return cudaErrorInvalidValue;
    }
    const size_t smem = sd_smem(s, a.C);
    cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    if (e != cudaSuccess) return e;
    kern<<<(unsigned)(units * a.C), kSdThreads, smem, st>>>(a);
    note_launch();
    return cudaGetLastError();
}

cudaError_t launch_select_decode(const Shape &s, const void *q, const void *L, int32_t *idx, float *score,
                                 int32_t *count, void *ws, cudaStream_t st) {
    return s.dtype == SA_BF16 ? run_sd<__nv_bfloat16>(s, q, L, idx, score, count, ws, st)
                              : run_sd<float>(s, q, L, idx, score, count, ws, st);
}

}  // namespace sa
