// select.cu -- pooled-query scoring against block landmarks and hard top-K.
//
// [SAS] opening section / "Ключевые факты": a light selector scores context
// units and a hard top-K keeps the best; the current block is always kept.
// The Latent Sparse Attention post ("Индекс перестаёт перебирать весь
// контекст"): the start of the context is always added as well.
//
// One unit = (batch, kv-head, query tile) in prefill or (batch, kv-head) in
// decode (per q-head with SA_SELECT_PER_QHEAD).  A CTA pools the unit's query
// (mean over its query heads and the tile's rows), scores one chunk of the
// candidate blocks (s_b = scale * <qbar, L_b>, fp32), and radix-selects the
// chunk's top-K on 32-bit order-preserving keys of the fp32 score; equal
// scores go to the lower block index (the candidates sit in index order and
// ties are ranked by position).  With one chunk per unit the CTA writes the
// final list; otherwise each chunk leaves its top-K in the workspace and a
// merge kernel picks the unit's top-K from them.  Either way the result is
// the exact top-K of the whole candidate set, independent of the split.
#include "common.cuh"

namespace sa {

constexpr int kSelThreads = 256;
constexpr int kMaxChunk = 8192;

struct SelArgs {
    Shape s;
    const void *Q;       // prefill Q [B,Hq,N,d] or decode q [B,Hq,d]
    const void *L;       // [B,Hkv,nb,d]
    int32_t *idx;
    float *score;
    int32_t *count;
    unsigned *status;
    uint32_t *part_key;  // [units][S][top_k]
    int32_t *part_idx;   // [units][S][top_k]
    float *special;      // [units][2]: s_0, s_local
    int S;               // chunks per unit
    int CH;              // candidates per chunk
    int decode;
    int ntiles;          // prefill: nb; decode: 1
    int mode;            // kFinal or kPartial
    unsigned *done;      // kPartial: [units] chunks finished; back to 0 after each call
};

// What a chunk CTA leaves behind: the unit's final list (one chunk per
// unit) or its chunk's top-K; in the second case the unit's last chunk CTA
// to finish merges the chunks' lists into the final one.
enum { kFinal = 0, kPartial = 1 };

struct SelSmem {
    float qbar[256];
    int hist[256];
    int tmp[8];
    int sel_digit, sel_above;
    float s_special[2];
    int last;
};

// Decodes a unit number into (batch, selection head, tile) and its local block.
__device__ __forceinline__ void unit_coords(const SelArgs &a, int u, int &b, int &hs, int &j, int &local) {
    j = u % a.ntiles;
    int r = u / a.ntiles;
    hs = r % a.s.Hsel;
    b = r / a.s.Hsel;
    local = a.decode ? (seq_n(a.s, b) - 1) / a.s.bs : j;
}

// Pooled query of the unit into sm.qbar (fp32).  Every thread participates.
template <typename T, int VPR>
__device__ void pool_query(const SelArgs &a, int b, int hs, int j, SelSmem &sm, float *red) {
    constexpr int EPV = Vec<T>::n;
    constexpr int NG = kSelThreads / VPR;
    const Shape &s = a.s;
    const int d = VPR * EPV;
    const int h0 = (s.flags & SA_SELECT_PER_QHEAD) ? hs : hs * s.G;
    const int nh = s.heads_per;
    const int r0 = a.decode ? 0 : j * s.bs;
    const int nrows = a.decode ? 1 : min(s.bs, s.N - r0);
    const int R = nh * nrows;
    const int cv = threadIdx.x % VPR, rg = threadIdx.x / VPR;
    float acc[EPV];
#pragma unroll
    for (int i = 0; i < EPV; ++i) acc[i] = 0.f;
    const T *Q = (const T *)a.Q;
    // U rows in flight per thread: pooling streams the tile's queries from HBM
    constexpr int U = 8;
    for (int r0u = rg; r0u < R; r0u += NG * U) {
        uint4 raw[U];
#pragma unroll
        for (int uu = 0; uu < U; ++uu) {
            const int r = r0u + NG * uu;
            const int rc = r < R ? r : r0u;
            const int hh = h0 + rc / nrows, row = r0 + rc % nrows;
            const T *p = a.decode ? Q + ((size_t)b * s.Hq + hh) * d : Q + (((size_t)b * s.Hq + hh) * s.N + row) * d;
            raw[uu] = *reinterpret_cast<const uint4 *>(p + cv * EPV);
        }
#pragma unroll
        for (int uu = 0; uu < U; ++uu) {
            if (r0u + NG * uu >= R) break;
            float f[EPV];
            load16(reinterpret_cast<const T *>(&raw[uu]), f);
#pragma unroll
            for (int i = 0; i < EPV; ++i) acc[i] += f[i];
        }
    }
#pragma unroll
    for (int i = 0; i < EPV; ++i) red[rg * d + cv * EPV + i] = acc[i];
    __syncthreads();
    if (threadIdx.x < d) {
        float t = 0.f;
        for (int g = 0; g < NG; ++g) t += red[g * d + threadIdx.x];
        sm.qbar[threadIdx.x] = t / (float)R;
    }
    __syncthreads();
}

// Score of landmark row `blk` for the VPR-lane group this lane belongs to.
template <typename T, int VPR>
__device__ __forceinline__ float group_score(const T *Lrow, const float *qv, float scale) {
    constexpr int EPV = Vec<T>::n;
    const int cv = (threadIdx.x & 31) % VPR;
    float f[EPV];
    load16(Lrow + cv * EPV, f);
    float dot = 0.f;
#pragma unroll
    for (int i = 0; i < EPV; ++i) dot = fmaf(qv[i], f[i], dot);
#pragma unroll
    for (int o = VPR / 2; o > 0; o >>= 1) dot += __shfl_xor_sync(0xffffffffu, dot, o);
    return scale * dot;
}

// Exact top-`k` of keys[0..n) (n > k): returns threshold key T and the number
// of keys equal to T that are taken (the lowest positions first).
__device__ void radix_select(const uint32_t *keys, int n, int k, SelSmem &sm, uint32_t &T, int &take_eq) {
    uint32_t prefix = 0, mask = 0;
    int remaining = k;
    for (int shift = 24; shift >= 0; shift -= 8) {
        sm.hist[threadIdx.x] = 0;
        __syncthreads();
        // warp-aggregated histogram: scores cluster in few top digits, so
        // lanes with the same digit add once per warp instead of once each
        for (int i0 = threadIdx.x - (threadIdx.x & 31); i0 < n; i0 += kSelThreads) {
            const int i = i0 + (threadIdx.x & 31);
            const uint32_t x = i < n ? keys[i] : 0u;
            const bool take = i < n && (x & mask) == prefix;
            const unsigned act = __ballot_sync(0xffffffffu, take);
            if (take) {
                const int digit = (int)((x >> shift) & 255);
                const unsigned same = __match_any_sync(act, digit);
                if ((threadIdx.x & 31) == __ffs(same) - 1) atomicAdd(&sm.hist[digit], __popc(same));
            }
        }
        __syncthreads();
        if (threadIdx.x < 32) {
            const int lane = threadIdx.x;
            const int hi = 255 - 8 * lane;
            int local = 0;
#pragma unroll
            for (int q = 0; q < 8; ++q) local += sm.hist[hi - q];
            int incl = local;
#pragma unroll
            for (int o = 1; o < 32; o <<= 1) {
                int t = __shfl_up_sync(0xffffffffu, incl, o);
                if (lane >= o) incl += t;
            }
            const int excl = incl - local;
            if (excl < remaining && remaining <= incl) {
                int cum = excl;
                for (int q = 0; q < 8; ++q) {
                    const int c = sm.hist[hi - q];
                    if (cum + c >= remaining) {
                        sm.sel_digit = hi - q;
                        sm.sel_above = cum;
                        break;
                    }
                    cum += c;
                }
            }
        }
        __syncthreads();
        remaining -= sm.sel_above;
        prefix |= (uint32_t)sm.sel_digit << shift;
        mask |= 255u << shift;
        __syncthreads();
    }
    T = prefix;
    take_eq = remaining;
}

// Marks the top-k of keys[0..n) and writes their positions, ascending, to
// out_pos[0..min(n,k)).  Returns the number written.
__device__ int topk_positions(const uint32_t *keys, int n, int k, SelSmem &sm, int *out_pos) {
    if (k <= 0 || n <= 0) return 0;
    if (n <= k) {
        for (int i = threadIdx.x; i < n; i += kSelThreads) out_pos[i] = i;
        __syncthreads();
        return n;
    }
    uint32_t T;
    int take_eq;
    radix_select(keys, n, k, sm, T, take_eq);
    const int seg = (n + kSelThreads - 1) / kSelThreads;
    const int i0 = min(n, threadIdx.x * seg), i1 = min(n, i0 + seg);
    int neq = 0;
    for (int i = i0; i < i1; ++i) neq += keys[i] == T;
    int eq_base = block_scan_incl(neq, sm.tmp, nullptr) - neq;
    int nsel = 0;
    {
        int e = eq_base;
        for (int i = i0; i < i1; ++i) {
            const uint32_t x = keys[i];
            const bool take = x > T || (x == T && e < take_eq);
            e += x == T;
            nsel += take;
        }
    }
    int total;
    int pos = block_scan_incl(nsel, sm.tmp, &total) - nsel;
    {
        int e = eq_base;
        for (int i = i0; i < i1; ++i) {
            const uint32_t x = keys[i];
            const bool take = x > T || (x == T && e < take_eq);
            e += x == T;
            if (take) out_pos[pos++] = i;
        }
    }
    __syncthreads();
    return total;
}

// Writes the final kept list of a unit: [0 (sink)] + selected (ascending) +
// [local].  sel_idx/sel_score hold `nsel` selected blocks in ascending order.
__device__ void write_final(const SelArgs &a, int u, int local, const int *sel_idx, const float *sel_score,
                            int nsel, float s0, float slocal) {
    const Shape &s = a.s;
    int32_t *idx = a.idx + (size_t)u * s.cap;
    float *sc = a.score + (size_t)u * s.cap;
    const bool sink = s.flags & SA_SINK;
    const bool loc = (s.flags & SA_LOCAL) && !(sink && local == 0);
    const int off = sink ? 1 : 0;
    const int cnt = off + nsel + (loc ? 1 : 0);
    for (int i = threadIdx.x; i < s.cap; i += kSelThreads) {
        int bi = -1;
        float sv = 0.f;
        if (i < cnt) {
            if (sink && i == 0) { bi = 0; sv = s0; }
            else if (loc && i == cnt - 1) { bi = local; sv = slocal; }
            else { bi = sel_idx[i - off]; sv = sel_score[i - off]; }
        }
        idx[i] = bi;
        sc[i] = sv;
    }
    if (threadIdx.x == 0) a.count[u] = cnt;
}

// Merges the per-chunk top-K lists of unit u (they sit in ascending block
// order, chunk after chunk) into the unit's final list.  Run by the unit's
// last chunk CTA; the partial lists are read past L1 (written by other CTAs).
__device__ void merge_unit(const SelArgs &a, int u, unsigned char *smem_raw) {
    SelSmem &sm = *reinterpret_cast<SelSmem *>(smem_raw);
    const Shape &s = a.s;
    const int M = a.S * s.top_k;
    uint32_t *keys = reinterpret_cast<uint32_t *>(smem_raw + sizeof(SelSmem));
    int *cidx = reinterpret_cast<int *>(keys + M);
    int *pos = cidx + M;
    int *sel_idx = pos + M;
    float *sel_sc = reinterpret_cast<float *>(sel_idx + s.top_k);
    int b, hs, j, local;
    unit_coords(a, u, b, hs, j, local);
    const int first = (s.flags & SA_SINK) ? 1 : 0;
    // chunk c holds nv(c) = min(top_k, its candidates) valid entries, packed
    // in chunk order; the chunk sizes are known, so every thread finds its
    // entry's slot by arithmetic and all loads are in flight together
    auto nv = [&](int c) {
        const int c0 = first + c * a.CH, c1 = min(local, c0 + a.CH);
        return min(s.top_k, max(0, c1 - c0));
    };
    int ntot = 0;
    for (int c = 0; c < a.S; ++c) ntot += nv(c);
    for (int e = threadIdx.x; e < M; e += kSelThreads) {
        const int c = e / s.top_k, i = e - c * s.top_k;
        if (i < nv(c)) {
            int base = 0;
            for (int q = 0; q < c; ++q) base += nv(q);
            const size_t src = ((size_t)u * a.S + c) * s.top_k + i;
            keys[base + i] = __ldcg(a.part_key + src);
            cidx[base + i] = __ldcg(a.part_idx + src);
        }
    }
    __syncthreads();
    const int nsel = topk_positions(keys, ntot, s.top_k, sm, pos);
    for (int i = threadIdx.x; i < nsel; i += kSelThreads) {
        sel_idx[i] = cidx[pos[i]];
        sel_sc[i] = key_to_float(keys[pos[i]]);
    }
    __syncthreads();
    write_final(a, u, local, sel_idx, sel_sc, nsel, __ldcg(a.special + (size_t)u * 2),
                __ldcg(a.special + (size_t)u * 2 + 1));
}

template <typename T, int VPR>
__global__ void __launch_bounds__(kSelThreads, 5) select_chunk_kernel(SelArgs a) {
    constexpr int EPV = Vec<T>::n;
    constexpr int NG = kSelThreads / VPR;
    extern __shared__ __align__(16) unsigned char smem_raw[];
    SelSmem &sm = *reinterpret_cast<SelSmem *>(smem_raw);
    uint32_t *keys = reinterpret_cast<uint32_t *>(smem_raw + sizeof(SelSmem));
    int *pos = reinterpret_cast<int *>(keys + a.CH);
    float *red = reinterpret_cast<float *>(pos + a.CH);

    const Shape &s = a.s;
    const int d = VPR * EPV;
    const int u = blockIdx.x / a.S, chunk = blockIdx.x % a.S;
    int b, hs, j, local;
    unit_coords(a, u, b, hs, j, local);
    const int g = (s.flags & SA_SELECT_PER_QHEAD) ? hs / s.G : hs;
    const int first = (s.flags & SA_SINK) ? 1 : 0;
    const int c0 = first + chunk * a.CH;
    const int c1 = min(local, c0 + a.CH);
    const int n = max(0, c1 - c0);

    float qv[EPV];
    if (a.decode) {
        // one query per head: every lane averages its own slice over the
        // group's heads (no shared memory, no barrier before the scan)
        const int cvq = (threadIdx.x & 31) % VPR;
        const int hq0 = (s.flags & SA_SELECT_PER_QHEAD) ? hs : hs * s.G;
#pragma unroll
        for (int i = 0; i < EPV; ++i) qv[i] = 0.f;
        for (int hh = 0; hh < s.heads_per; ++hh) {
            float f[EPV];
            load16((const T *)a.Q + ((size_t)b * s.Hq + hq0 + hh) * d + cvq * EPV, f);
#pragma unroll
            for (int i = 0; i < EPV; ++i) qv[i] += f[i];
        }
#pragma unroll
        for (int i = 0; i < EPV; ++i) qv[i] /= (float)s.heads_per;
    } else {
        pool_query<T, VPR>(a, b, hs, j, sm, red);
        const int cvq = (threadIdx.x & 31) % VPR;
#pragma unroll
        for (int i = 0; i < EPV; ++i) qv[i] = sm.qbar[cvq * EPV + i];
    }
    const T *Lg = (const T *)a.L + ((size_t)b * s.Hkv + g) * s.nb * d;
    // rows are handed out per warp so that every lane of a warp takes the
    // same trip count (the group reduction shuffles over the full warp)
    constexpr int RPW = 32 / VPR;
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int sub = lane / VPR, cv = lane % VPR;
    bool nan_seen = false;
    // U rows per group in flight: the scan is a pure HBM stream of landmarks
    constexpr int U = 8;
    for (int base = warp * RPW * U; base < n; base += NG * U) {
        uint4 raw[U];
#pragma unroll
        for (int uu = 0; uu < U; ++uu) {
            const int r = min(base + sub + RPW * uu, n - 1);
            raw[uu] = *reinterpret_cast<const uint4 *>(Lg + (size_t)(c0 + r) * d + cv * EPV);
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
            const float sc = s.scale * dot;
            const int r = base + sub + RPW * uu;
            if (cv == 0 && r < n) {
                nan_seen |= isnan(sc);
                keys[r] = ord_key(sc);
            }
        }
    }
    if (chunk == 0 && warp < 2) {
        const int blk = warp == 0 ? 0 : local;   // warp 0: sink score, warp 1: local score
        const float sc = group_score<T, VPR>(Lg + (size_t)blk * d, qv, s.scale);
        if (lane == 0) {
            sm.s_special[warp] = sc;
            nan_seen |= isnan(sc);
        }
    }
    if (nan_seen) set_status(a.status, kStatusNaN);
    __syncthreads();

    const int nsel = topk_positions(keys, n, s.top_k, sm, pos);
    if (a.mode == kFinal) {
        // reuse the pooling buffer for the ascending selected list
        int *sel_idx = reinterpret_cast<int *>(red);
        float *sel_sc = reinterpret_cast<float *>(sel_idx + s.top_k);
        for (int i = threadIdx.x; i < nsel; i += kSelThreads) {
            sel_idx[i] = c0 + pos[i];
            sel_sc[i] = key_to_float(keys[pos[i]]);
        }
        __syncthreads();
        write_final(a, u, local, sel_idx, sel_sc, nsel, sm.s_special[0], sm.s_special[1]);
    } else {
        uint32_t *pk = a.part_key + ((size_t)u * a.S + chunk) * s.top_k;
        int32_t *pi = a.part_idx + ((size_t)u * a.S + chunk) * s.top_k;
        for (int i = threadIdx.x; i < s.top_k; i += kSelThreads) {
            pk[i] = i < nsel ? keys[pos[i]] : 0u;
            pi[i] = i < nsel ? c0 + pos[i] : -1;
        }
        if (chunk == 0 && threadIdx.x < 2) a.special[(size_t)u * 2 + threadIdx.x] = sm.s_special[threadIdx.x];
        // the unit's last chunk to finish merges (writes fenced before the count)
        __threadfence();
        __syncthreads();
        if (threadIdx.x == 0) sm.last = atomicAdd(a.done + u, 1u) == (unsigned)(a.S - 1);
        __syncthreads();
        if (sm.last) {
            __threadfence();
            merge_unit(a, u, smem_raw);
            if (threadIdx.x == 0) a.done[u] = 0u;
        }
    }
}

static void geometry(const Shape &s, bool decode, int &nunits, int &S, int &CH) {
    const int ntiles = decode ? 1 : s.nb;
    nunits = s.B * s.Hsel * ntiles;
    const int local_max = decode ? (s.N - 1) / s.bs : s.nb - 1;
    const int first = (s.flags & SA_SINK) ? 1 : 0;
    const int ncand = max(1, local_max - first);
    S = 1;
    if (decode) {
        // chunks of about 512 candidates: thousands of CTAs keep every SM
        // streaming landmarks while others run their chunk's top-K
        S = max(1, (ncand + 511) / 512);
    }
    S = max(S, (ncand + kMaxChunk - 1) / kMaxChunk);
    CH = (ncand + S - 1) / S;
    if (s.top_k == 0) {   // nothing to rank: only the sink and local scores
        S = 1;
        CH = 0;
    }
}

size_t select_workspace(const Shape &s, bool decode) {
    if (decode && select_decode_supported(s)) return select_decode_workspace(s);
    int nunits, S, CH;
    geometry(s, decode, nunits, S, CH);
    if (S == 1) return 0;
    return (size_t)nunits * S * s.top_k * (sizeof(uint32_t) + sizeof(int32_t)) + (size_t)nunits * 2 * sizeof(float) +
           256;
}

template <typename T>
static cudaError_t run(const Shape &s, bool decode, const void *Q, const void *L, int32_t *idx, float *score,
                       int32_t *count, void *ws, cudaStream_t st) {
    SelArgs a{};
    a.s = s;
    a.Q = Q;
    a.L = L;
    a.idx = idx;
    a.score = score;
    a.count = count;
    a.status = (unsigned *)ws;
    a.decode = decode;
    a.ntiles = decode ? 1 : s.nb;
    int nunits;
    geometry(s, decode, nunits, a.S, a.CH);
    a.mode = a.S == 1 ? kFinal : kPartial;
    if (a.S > 1) {
        char *p = (char *)ws + ws_layout(s).scratch;
        a.part_key = (uint32_t *)p;
        p += (size_t)nunits * a.S * s.top_k * sizeof(uint32_t);
        a.part_idx = (int32_t *)p;
        p += (size_t)nunits * a.S * s.top_k * sizeof(int32_t);
        a.special = (float *)p;
        a.done = (unsigned *)((char *)ws + ws_layout(s).sel_chunk);
    }
    const int vpr = s.d * (int)sizeof(T) / 16;
    const int d = s.d;
    size_t red_bytes = (size_t)(kSelThreads / vpr) * d * sizeof(float);
    red_bytes = max(red_bytes, (size_t)s.top_k * 8);
    size_t smem = sizeof(SelSmem) + (size_t)a.CH * 8 + red_bytes;
    if (a.mode == kPartial)   // the merging CTA reuses the same shared memory
        smem = max(smem, sizeof(SelSmem) + (size_t)a.S * s.top_k * 12 + (size_t)s.top_k * 8);
    void (*kern)(SelArgs) = nullptr;
    switch (vpr) {
        case 8: kern = select_chunk_kernel<T, 8>; break;
        case 16: kern = select_chunk_kernel<T, 16>; break;
        case 32: kern = select_chunk_kernel<T, 32>; break;
        default: return cudaErrorInvalidValue;
    }
    cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    if (e != cudaSuccess) return e;
    kern<<<(unsigned)nunits * a.S, kSelThreads, smem, st>>>(a);
    note_launch();
    e = cudaGetLastError();
    return e;
}

cudaError_t launch_select(const Shape &s, bool decode, const void *Q, const void *L, int32_t *idx, float *score,
                          int32_t *count, void *ws, size_t ws_bytes, cudaStream_t st) {
    (void)ws_bytes;
    // prefill: eight tiles per CTA share one landmark scan (select_tiles.cu)
    if (!decode && select_tiles_supported(s))
        return launch_select_tiles(s, Q, L, idx, score, count, (unsigned *)ws, st);
    // decode: a warp per chunk of candidates (select_decode.cu)
    if (decode && select_decode_supported(s) && !select_force_chunked())
        return launch_select_decode(s, Q, L, idx, score, count, ws, st);
    return s.dtype == SA_BF16 ? run<__nv_bfloat16>(s, decode, Q, L, idx, score, count, ws, st)
                              : run<float>(s, decode, Q, L, idx, score, count, ws, st);
}

}  // namespace sa
