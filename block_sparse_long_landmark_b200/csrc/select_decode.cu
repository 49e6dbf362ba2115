// select_decode.cu -- decode selection with a warp per chunk of candidates.
//
// [SAS] opening section / "Ключевые факты": a light selector scores the
// context blocks and a hard top-K keeps the best; the current block is
// always kept.  The Latent Sparse Attention post ("Индекс перестаёт
// перебирать весь контекст"): the start of the context is always added.
//
// Decode scans every landmark of a sequence once per step, so the step is a
// stream of landmarks from HBM.  A CTA owns 2048 (or 4096) consecutive
// candidate blocks of one (batch, selection head): a producer warp streams
// their landmarks in 32 KB stages through a ring of bulk copies in shared
// memory, and eight scoring warps each take an eighth of every stage.  Each
// lane holds a 16-byte slice of the unit's pooled query and scores eight
// 16-byte slices per stage; the partial dots are summed by a reduce-scatter
// across the lanes of a row, so every lane ends with one full score.  Once the
// stream is over the eight warps take the CTA's top-K together with a
// bounded-candidate select (block_select.cuh).  When a unit spans several
// CTAs, each leaves its top-K in the workspace ordered by (key desc, block
// asc); the unit's last CTA to finish ranks every entry in the unit by its
// index in its own list plus a binary search in each other list, keeps ranks
// below K and orders them by block.  Every select takes equal keys at the
// lower block, so the result is the exact top-K by (score desc, index asc)
// whatever the split.
#include <cstdlib>
#include <cstring>

#include "block_select.cuh"
#include "bounds.cuh"
#include "common.cuh"
#include "tc_ptx.cuh"

namespace sa {
namespace {

constexpr int kSdWarps = 8;          // scoring warps; warp 8 streams
constexpr int kSdThreads = 32 * (kSdWarps + 1);
constexpr int kSdChunk = 256;        // candidates per scoring warp, or twice that
constexpr int kSdMaxMerge = 4096;    // list entries the cross-CTA merge holds
constexpr int kSdMaxC = 64;          // CTAs per unit, at most
constexpr int kSdStage = 32768;      // bytes per ring stage: eight 16-byte slices per scoring lane
constexpr int kSdStages = 3;        // ring stages with 256 candidates per warp; 2 with 512
__host__ __device__ constexpr int sd_stages(int CH) { return CH == kSdChunk ? kSdStages : 2; }
__host__ __device__ constexpr uint32_t sd_ring_bytes(int CH) { return (uint32_t)sd_stages(CH) * kSdStage; }

struct SdArgs {
    Shape s;
    const void *q;        // [B,Hq,d]
    const void *L;        // [B,Hkv,nb,d]
    int32_t *idx;
    float *score;
    int32_t *count;
    unsigned *status;
    uint32_t *pkey;       // [units][C][top_k] each CTA's top-K keys, by (key desc, block asc)
    int32_t *pidx;        // [units][C][top_k] their block ids
    int32_t *pcnt;        // [units][C] how many
    float *special;       // [units][2]: s_0, s_local
    unsigned *done;       // [units] CTAs finished; back to 0 by the merging CTA
    unsigned *ready;      // [units] epoch of the latest list, or null (not published)
    unsigned epoch;
    int C;                // CTAs per unit
};

struct SdSmem {
    float s_special[2];
    int abort_flag;
    int last;
    int ccnt[kSdMaxC];          // the unit's CTAs: list lengths
    int coff[kSdMaxC + 1];      // and where each list starts
    uint64_t full[kSdStages], empty[kSdStages];
};

// Shared memory: header, keys [8 * CH], the ring [stages][32 KB].  Once the
// stream is over the ring holds the select's state, the positions it returns,
// the final list and the cross-CTA merge's keys and block ids.
__host__ __device__ constexpr size_t sd_off_keys() { return (sizeof(SdSmem) + 127) & ~(size_t)127; }
__host__ __device__ constexpr size_t sd_off_ring(int CH) { return sd_off_keys() + (size_t)kSdWarps * CH * 4; }
__host__ __device__ constexpr size_t sd_smem_bytes(int CH) { return sd_off_ring(CH) + sd_ring_bytes(CH); }
// offsets inside the ring once the stream is over
constexpr size_t kSdXKey = 0;                                   // [kSdMaxMerge] keys
constexpr size_t kSdXIdx = kSdXKey + (size_t)kSdMaxMerge * 4;   // [kSdMaxMerge] block ids
constexpr size_t kSdBs = kSdXIdx + (size_t)kSdMaxMerge * 4;     // BsSmem
constexpr size_t kSdPos = kSdBs + ((sizeof(BsSmem) + 15) & ~(size_t)15);   // [kSdChunk] positions
constexpr size_t kSdSelKey = kSdPos + (size_t)kSdChunk * 4;     // [kSdChunk] final keys
constexpr size_t kSdSelIdx = kSdSelKey + (size_t)kSdChunk * 4;  // [kSdChunk] final block ids
constexpr size_t kSdAfter = kSdSelIdx + (size_t)kSdChunk * 4;
static_assert(kSdAfter <= sd_ring_bytes(2 * kSdChunk) && kSdAfter <= sd_ring_bytes(kSdChunk),
              "the select's state fits the ring");

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

// The unit's list is written (by the calling warp): store the call's epoch
// with release order, for a decode step that waits on it unit by unit.
__device__ __forceinline__ void publish_list(const SdArgs &a, int u) {
    if (!a.ready) return;
    __threadfence();
    __syncwarp();
    if ((threadIdx.x & 31) == 0)
        asm volatile("st.release.gpu.global.u32 [%0], %1;" ::"l"(a.ready + u), "r"(a.epoch) : "memory");
}

// How many of list[0..n) (16-byte aligned) are below x; four per shared load.
__device__ __forceinline__ int count_below(const int *list, int n, int x) {
    const int4 *l4 = reinterpret_cast<const int4 *>(list);
    int c0 = 0, c1 = 0;
    const int n4 = n >> 2;
#pragma unroll 4
    for (int i4 = 0; i4 < n4; ++i4) {
        const int4 y = l4[i4];
        c0 += (y.x < x) + (y.z < x);
        c1 += (y.y < x) + (y.w < x);
    }
    for (int i = n4 << 2; i < n; ++i) c0 += list[i] < x;
    return c0 + c1;
}

// fp32 slice of a 16-byte group of elements
__device__ __forceinline__ void slice_f32(const uint4 &u, const __nv_bfloat16 *, float *f) {
    const uint32_t w[4] = {u.x, u.y, u.z, u.w};
#pragma unroll
    for (int i = 0; i < 4; ++i) {
        f[2 * i] = __uint_as_float(w[i] << 16);
        f[2 * i + 1] = __uint_as_float(w[i] & 0xffff0000u);
    }
}
__device__ __forceinline__ void slice_f32(const uint4 &u, const float *, float *f) {
    f[0] = __uint_as_float(u.x);
    f[1] = __uint_as_float(u.y);
    f[2] = __uint_as_float(u.z);
    f[3] = __uint_as_float(u.w);
}

template <typename T, int VPR, int CH>
__global__ void __launch_bounds__(kSdThreads, 2) select_decode_kernel(SdArgs a) {
    constexpr int NST = sd_stages(CH);
    using namespace tc;
    constexpr int EPV = Vec<T>::n;
    constexpr int RB = VPR * 16;                    // bytes per row
    constexpr int RPL = 32 / VPR;                   // rows per 16-byte load step of the warp
    constexpr int ROWS = kSdStage / RB;             // rows per stage
    constexpr int RW = ROWS / kSdWarps;             // rows per scoring warp per stage
    constexpr int NL = RW / RPL;                    // load steps (partial dots) per lane per stage
    constexpr int SPAN = VPR / NL;                  // lanes that end with the same row's score
    static_assert(NL == 8 && SPAN >= 1, "stage geometry");
    const Shape &s = a.s;
    const int D = VPR * EPV;
    extern __shared__ __align__(128) unsigned char smraw[];
    SdSmem &sm = *reinterpret_cast<SdSmem *>(smraw);
    uint32_t *keys = reinterpret_cast<uint32_t *>(smraw + sd_off_keys());      // [8 * CH]
    unsigned char *ring = smraw + sd_off_ring(CH);                              // [stages][32 KB]

    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int u = blockIdx.x / a.C, cta = blockIdx.x % a.C;
    const int hs = u % s.Hsel, b = u / s.Hsel;
    const bool perq = s.flags & SA_SELECT_PER_QHEAD;
    const int g = perq ? hs / s.G : hs;
    const int hq0 = perq ? hs : hs * s.G;
    const int local = (seq_n(s, b) - 1) / s.bs;
    const int first = (s.flags & SA_SINK) ? 1 : 0;
    const int cc0 = first + cta * kSdWarps * CH;                    // the CTA's first candidate
    const int ncta = max(0, min(local, cc0 + kSdWarps * CH) - cc0);

    // the attention launch that follows may start as this grid's CTAs are placed
    asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
    if (threadIdx.x == 0) {
        for (int i = 0; i < NST; ++i) {
            mbar_init(smem_u32(&sm.full[i]), 1);
            mbar_init(smem_u32(&sm.empty[i]), kSdWarps);
        }
        sm.abort_flag = 0;
        asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
    }
    __syncthreads();

    const T *Lg = (const T *)a.L + ((size_t)b * s.Hkv + g) * s.nb * D;
    const size_t cbytes = (size_t)ncta * RB;                        // the CTA's landmark bytes
    const int nst = (int)((cbytes + kSdStage - 1) / kSdStage);
    bool nan_seen = false;
    float qv[EPV];
    const int sub = lane / VPR, cv = lane % VPR;
    if (warp == kSdWarps) {
        // ---- producer: the CTA's landmarks, stage by stage --------------------
        if (lane == 0) {
            const unsigned char *src = reinterpret_cast<const unsigned char *>(Lg + (size_t)cc0 * D);
            int issued = 0;
            for (int i = 0; i < nst; ++i) {
                const int st = i % NST;
                if (i >= NST &&
                    !mbar_wait(smem_u32(&sm.empty[st]), ((i / NST) - 1) & 1, &sm.abort_flag, a.status))
                    break;
                const uint32_t bytes = (uint32_t)min((size_t)kSdStage, cbytes - (size_t)i * kSdStage);
                SA_CHECK_SPAN(a.status, (long long)cc0 * RB + (long long)i * kSdStage, bytes, (long long)s.nb * RB);
                mbar_expect_tx(smem_u32(&sm.full[st]), bytes);
                bulk_load(smem_u32(ring + st * kSdStage), src + (size_t)i * kSdStage, bytes, smem_u32(&sm.full[st]));
                issued = i + 1;
            }
            if (sm.abort_flag) {
                // let the copies in flight land before the ring is reused
                volatile int never = 0;
                for (int i = max(0, issued - NST); i < issued; ++i)
                    mbar_wait(smem_u32(&sm.full[i % NST]), (i / NST) & 1, &never, a.status);
            }
        }
    } else {
        // ---- scoring warps -------------------------------------------------------
        // the unit's pooled query: lane group member cv holds elements cv*EPV ..
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
        // the sink and local scores (warp 0 of the unit's first CTA, while the
        // first stage is in flight)
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
        for (int i = 0; i < nst; ++i) {
            const int st = i % NST;
            const bool ok = mbar_wait(smem_u32(&sm.full[st]), (i / NST) & 1, &sm.abort_flag, a.status);
            if (!__all_sync(0xffffffffu, ok)) break;
            const unsigned char *stg = ring + st * kSdStage + warp * RW * RB;
            float v[NL];
#pragma unroll
            for (int l = 0; l < NL; ++l) {
                const uint4 raw = *reinterpret_cast<const uint4 *>(stg + (l * RPL + sub) * RB + cv * 16);
                float f[EPV];
                slice_f32(raw, (const T *)nullptr, f);
                float dot = 0.f;
#pragma unroll
                for (int e = 0; e < EPV; ++e) dot = fmaf(qv[e], f[e], dot);
                v[l] = dot;
            }
            __syncwarp();
            if (lane == 0) mbar_arrive(smem_u32(&sm.empty[st]));
            // reduce-scatter over the VPR lanes of a row: each halving step keeps
            // half of the rows and adds the partner's partials for them
#pragma unroll
            for (int m = VPR / 2, cnt = NL; cnt > 1; m >>= 1, cnt >>= 1) {
                const bool upper = cv & m;
#pragma unroll
                for (int k = 0; k < cnt / 2; ++k) {
                    const float send = upper ? v[k] : v[k + cnt / 2];
                    const float keep = upper ? v[k + cnt / 2] : v[k];
                    v[k] = keep + __shfl_xor_sync(0xffffffffu, send, m);
                }
            }
#pragma unroll
            for (int m = SPAN / 2; m > 0; m >>= 1) v[0] += __shfl_xor_sync(0xffffffffu, v[0], m);
            // the row this lane's score belongs to, as an offset in the CTA's candidates
            const int r = i * ROWS + warp * RW + (cv / SPAN) * RPL + sub;
            if (cv % SPAN == 0 && r < ncta) {
                const float sc = s.scale * v[0];
                nan_seen |= isnan(sc);
                keys[r] = ord_key(sc);
            }
        }
    }
    if (nan_seen) set_status(a.status, kStatusNaN);
    __syncthreads();
    // ---- the CTA's top-K: the eight scoring warps together ------------------
    // (the producer leaves; the rest synchronise on named barrier 1)
    if (warp == kSdWarps) return;
    constexpr int NT = kSdWarps * 32;
    BsSmem &bs = *reinterpret_cast<BsSmem *>(ring + kSdBs);
    int *pos = reinterpret_cast<int *>(ring + kSdPos);
    uint32_t *sel_key = reinterpret_cast<uint32_t *>(ring + kSdSelKey);
    int *sel_idx = reinterpret_cast<int *>(ring + kSdSelIdx);
    const int nc = block_topk32<kSdWarps, CH / 32>(keys, ncta, s.top_k, pos, bs, 1, CH / 32);
    if (a.C == 1) {
        // one CTA per unit: its list is the unit's
        for (int i = threadIdx.x; i < nc; i += NT) {
            sel_idx[i] = cc0 + pos[i];
            sel_key[i] = keys[pos[i]];
        }
        named_bar_sync<NT>(1);
        if (warp == 0) {
            write_list(a, u, local, sel_idx, sel_key, nc, sm.s_special[0], sm.s_special[1]);
            publish_list(a, u);
        }
        return;
    }
    {
        // several CTAs per unit: this CTA's list into the workspace, ordered by
        // (key desc, block asc) -- each entry's rank among the list's entries
        uint32_t *pk = a.pkey + ((size_t)u * a.C + cta) * s.top_k;
        int32_t *pi = a.pidx + ((size_t)u * a.C + cta) * s.top_k;
        for (int i = threadIdx.x; i < nc; i += NT) sel_key[i] = keys[pos[i]];
        named_bar_sync<NT>(1);
        for (int i = threadIdx.x; i < nc; i += NT) {
            const uint32_t x = sel_key[i];
            const int rk = rank_in(sel_key, nc, x, i);
            pk[rk] = x;
            pi[rk] = cc0 + pos[i];
        }
        if (threadIdx.x == 0) {
            a.pcnt[(size_t)u * a.C + cta] = nc;
            if (cta == 0) {
                a.special[(size_t)u * 2] = sm.s_special[0];
                a.special[(size_t)u * 2 + 1] = sm.s_special[1];
            }
        }
    }
    // the unit's last CTA to finish merges (every thread's writes fenced
    // before the count)
    __threadfence();
    named_bar_sync<NT>(1);
    if (threadIdx.x == 0) sm.last = atomicAdd(a.done + u, 1u) == (unsigned)(a.C - 1);
    named_bar_sync<NT>(1);
    if (!sm.last) return;
    __threadfence();
    // the sink and local scores, loaded before the lists so the loads overlap
    float sp0 = 0.f, sp1 = 0.f;
    if (warp == 0) {
        sp0 = __ldcg(a.special + (size_t)u * 2);
        sp1 = __ldcg(a.special + (size_t)u * 2 + 1);
    }
    // The unit's lists, end to end in CTA order, each by (key desc, block asc).
    // An entry's rank in the unit is its index in its own list plus, in every
    // other list, the entries above it: keys > x, and keys == x too in the
    // lists of earlier CTAs (lower blocks) -- a binary search per list.
    uint32_t *xkey = reinterpret_cast<uint32_t *>(ring + kSdXKey);     // [C][top_k]
    int *xidx = reinterpret_cast<int *>(ring + kSdXIdx);
    // every list slot and every count in one round of loads
    const int K = s.top_k, slots = a.C * K;
    if (threadIdx.x < a.C) sm.ccnt[threadIdx.x] = __ldcg(a.pcnt + (size_t)u * a.C + threadIdx.x);
    for (int e = threadIdx.x; e < slots; e += NT) {
        xkey[e] = __ldcg(a.pkey + (size_t)u * slots + e);
        xidx[e] = __ldcg(a.pidx + (size_t)u * slots + e);
    }
    named_bar_sync<NT>(1);
    int total = 0;
    for (int c = 0; c < a.C; ++c) total += sm.ccnt[c];
    for (int e = threadIdx.x; e < slots; e += NT) {
        const int c = e / K, i0 = e - c * K;
        if (i0 >= sm.ccnt[c]) continue;
        const uint32_t x = xkey[e];
        int rk = i0;
        for (int c2 = 0; c2 < a.C && rk < K; ++c2) {
            if (c2 == c) continue;
            // first entry of list c2 not above x (descending keys)
            int lo = c2 * K, hi = c2 * K + sm.ccnt[c2];
            while (lo < hi) {
                const int mid = (lo + hi) >> 1;
                const uint32_t y = xkey[mid];
                if (y > x || (c2 < c && y == x)) lo = mid + 1;
                else hi = mid;
            }
            rk += lo - c2 * K;
        }
        if (rk < K) {       // the unit's top-K, slot = rank
            sel_key[rk] = x;
            pos[rk] = xidx[e];
        }
    }
    named_bar_sync<NT>(1);
    // the kept entries by ascending block
    const int nf = min(total, K);
    for (int i = threadIdx.x; i < nf; i += NT) {
        const int blk = pos[i];
        const int at = count_below(pos, nf, blk);
        sel_idx[at] = blk;
        xkey[at] = sel_key[i];
    }
    named_bar_sync<NT>(1);
    for (int i = threadIdx.x; i < nf; i += NT) sel_key[i] = xkey[i];
    named_bar_sync<NT>(1);
    if (warp == 0) {
        write_list(a, u, local, sel_idx, sel_key, nf, sp0, sp1);
        publish_list(a, u);
        if (lane == 0) a.done[u] = 0u;
    }
}

}  // namespace

// Geometry: scoring-warp chunks of 256 candidates (512 when that turns more
// than one wave of CTAs -- two per SM -- into one) cover the largest candidate
// count (the full context), grouped eight to a CTA.
static void sd_geometry(const Shape &s, int &C, int &CH) {
    const int first = (s.flags & SA_SINK) ? 1 : 0;
    const int ncand = max(1, (s.N - 1) / s.bs - first);
    const long long units = (long long)s.B * s.Hsel, slots = 2LL * 148;
    auto ctas = [&](int ch) { return (ncand + kSdWarps * ch - 1) / (kSdWarps * ch); };
    CH = (units * ctas(kSdChunk) > slots && units * ctas(2 * kSdChunk) <= slots) ? 2 * kSdChunk : kSdChunk;
    C = ctas(CH);
}

bool select_force_chunked() {
    const char *e = getenv("SPARSE_ATTN_SELECT_PATH");
    return e && strcmp(e, "chunked") == 0;
}

bool select_decode_supported(const Shape &s) {
    if (s.top_k < 1 || s.top_k > kSdChunk) return false;
    int C, CH;
    sd_geometry(s, C, CH);
    return C == 1 || (C <= kSdMaxC && (long long)C * s.top_k <= kSdMaxMerge);
}

size_t select_decode_workspace(const Shape &s) {
    int C, CH;
    sd_geometry(s, C, CH);
    if (C == 1) return 0;
    const size_t units = (size_t)s.B * s.Hsel;
    return units * C * s.top_k * 8 + units * C * 4 + units * 2 * 4 + 4 * 256;
}

static size_t sd_smem(int CH) { return sd_smem_bytes(CH); }

template <typename T>
static cudaError_t run_sd(const Shape &s, const void *q, const void *L, int32_t *idx, float *score, int32_t *count,
                          void *ws, cudaStream_t st, unsigned *ready, unsigned epoch) {
    SdArgs a{};
    a.s = s;
    a.q = q;
    a.L = L;
    a.idx = idx;
    a.score = score;
    a.count = count;
    a.status = (unsigned *)ws;
    a.ready = ready;
    a.epoch = epoch;
    int CH;
    sd_geometry(s, a.C, CH);
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
        case 8: kern = CH == kSdChunk ? select_decode_kernel<T, 8, kSdChunk> : select_decode_kernel<T, 8, 2 * kSdChunk>; break;
        case 16: kern = CH == kSdChunk ? select_decode_kernel<T, 16, kSdChunk> : select_decode_kernel<T, 16, 2 * kSdChunk>; break;
        case 32: kern = CH == kSdChunk ? select_decode_kernel<T, 32, kSdChunk> : select_decode_kernel<T, 32, 2 * kSdChunk>; break;
        default: return cudaErrorInvalidValue;
    }
    const size_t smem = sd_smem(CH);
    cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    if (e != cudaSuccess) return e;
    kern<<<(unsigned)(units * a.C), kSdThreads, smem, st>>>(a);
    note_launch();
    return cudaGetLastError();
}

cudaError_t launch_select_decode(const Shape &s, const void *q, const void *L, int32_t *idx, float *score,
                                 int32_t *count, void *ws, cudaStream_t st, unsigned *ready, unsigned epoch) {
    return s.dtype == SA_BF16 ? run_sd<__nv_bfloat16>(s, q, L, idx, score, count, ws, st, ready, epoch)
                              : run_sd<float>(s, q, L, idx, score, count, ws, st, ready, epoch);
}

}  // namespace sa
