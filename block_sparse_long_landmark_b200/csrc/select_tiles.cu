// select_tiles.cu -- prefill selection for eight consecutive query tiles per
// CTA: the landmarks are read once for all eight, and each warp selects its
// own tile's blocks without block-wide barriers.
//
// Same definition as select.cu ([SAS] opening section and "Ключевые факты":
// a light selector scores the blocks and a hard top-K keeps the best, the
// current block always kept; the Latent Sparse Attention post, "Индекс
// перестаёт перебирать весь контекст": the start of the context always
// added): pooled query = mean of Q over the unit's query heads and the tile's
// rows; s_b = scale * <pooled, L_b> in fp32; top-K of the candidate blocks by
// (score desc, index asc) on order-preserving 32-bit keys.
//
// CTA = (batch, selection head, tiles j0 .. j0+7); warp w owns tile j0 + w.
//   1. warp w pools its tile's queries (16-byte loads, 16 per lane in flight);
//   2. the CTA scans landmark rows 0 .. j0+7 once: a group of VPR lanes holds
//      one row and all eight pooled queries' matching slices, forms the eight
//      dot products and reduce-scatters them (3 halving exchanges + the rest
//      of the butterfly), so every row costs eight shuffles, not 32;
//   3. warp w finds its tile's top-K (bitwise search for the k-th key, then
//      an index-ordered compaction; warp_select.cuh) and writes the list.
#include "common.cuh"
#include "warp_select.cuh"

namespace sa {
namespace {

constexpr int kTpc = 8;          // tiles per CTA (one per warp)
constexpr int kThreadsT = 32 * kTpc;
constexpr int kMaxRows = 4096;   // landmark rows kept in shared memory per tile

struct TilesArgs {
    Shape s;
    const void *Q, *L;
    int32_t *idx;
    float *score;
    int32_t *count;
    unsigned *status;
    int ngroups;                 // ceil(nb / kTpc)
};

template <typename T, int VPR>
__global__ void __launch_bounds__(kThreadsT) select_tiles_kernel(TilesArgs a) {
    constexpr int EPV = Vec<T>::n;
    constexpr int D = VPR * EPV;
    constexpr int RPW = 32 / VPR;                 // landmark rows per warp step
    constexpr int NGR = kThreadsT / VPR;          // lane groups in the CTA
    constexpr int U = 4;                          // rows in flight per group
    const Shape &s = a.s;
    extern __shared__ __align__(16) unsigned char smem_raw[];
    float *qbar = reinterpret_cast<float *>(smem_raw);                     // [kTpc][D]
    int *outp = reinterpret_cast<int *>(qbar + kTpc * D);                  // [kTpc][top_k]
    uint32_t *keys = reinterpret_cast<uint32_t *>(outp + kTpc * max(s.top_k, 1));   // [kTpc][kcap]

    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int grp = blockIdx.x % a.ngroups;
    const int row = blockIdx.x / a.ngroups;       // b * Hsel + hs
    const int hs = row % s.Hsel, b = row / s.Hsel;
    const int j0 = grp * kTpc;
    const int kmax = min(s.nb - 1, j0 + kTpc - 1);
    const int kcap = kmax + 1;
    const bool perq = s.flags & SA_SELECT_PER_QHEAD;
    const int g = perq ? hs / s.G : hs;
    const int h0 = perq ? hs : hs * s.G;
    const int cv = lane % VPR, sub = lane / VPR;

    // ---- 1. pooled query of tile j0 + warp --------------------------------
    {
        const int j = j0 + warp;
        float acc[EPV];
#pragma unroll
        for (int i = 0; i < EPV; ++i) acc[i] = 0.f;
        int R = 0;
        if (j < s.nb) {
            const int r0 = j * s.bs, nrows = min(s.bs, s.N - r0);
            R = s.heads_per * nrows;
            const T *Qb = (const T *)a.Q;
            constexpr int UP = 16;
            for (int base = 0; base < R; base += RPW * UP) {
                uint4 raw[UP];
#pragma unroll
                for (int uu = 0; uu < UP; ++uu) {
                    const int r = min(base + sub + RPW * uu, R - 1);
                    const int hh = h0 + r / nrows, qr = r0 + r % nrows;
                    raw[uu] = *reinterpret_cast<const uint4 *>(Qb + (((size_t)b * s.Hq + hh) * s.N + qr) * D +
                                                               cv * EPV);
                }
#pragma unroll
                for (int uu = 0; uu < UP; ++uu) {
                    if (base + sub + RPW * uu >= R) continue;
                    float f[EPV];
                    load16(reinterpret_cast<const T *>(&raw[uu]), f);
#pragma unroll
                    for (int i = 0; i < EPV; ++i) acc[i] += f[i];
                }
            }
        }
#pragma unroll
        for (int o = VPR; o < 32; o <<= 1)
#pragma unroll
            for (int i = 0; i < EPV; ++i) acc[i] += __shfl_xor_sync(0xffffffffu, acc[i], o);
        if (sub == 0) {
#pragma unroll
            for (int i = 0; i < EPV; ++i) qbar[warp * D + cv * EPV + i] = R > 0 ? acc[i] / (float)R : 0.f;
        }
    }
    __syncthreads();

    // ---- 2. one scan of the landmark rows for all eight tiles -------------
    float qv[kTpc][EPV];
#pragma unroll
    for (int t = 0; t < kTpc; ++t)
#pragma unroll
        for (int i = 0; i < EPV; ++i) qv[t][i] = qbar[t * D + cv * EPV + i];
    const T *Lg = (const T *)a.L + ((size_t)b * s.Hkv + g) * s.nb * D;
    // the tile whose total this lane ends up with after the three halvings
    const int my_t = ((lane & (VPR / 2)) ? 4 : 0) + ((lane & (VPR / 4)) ? 2 : 0) + ((lane & (VPR / 8)) ? 1 : 0);
    const bool writer = (cv % (VPR / 8)) == 0;
    bool nan_seen = false;
    for (int base = warp * RPW * U; base < kcap; base += NGR * U) {
        uint4 raw[U];
#pragma unroll
        for (int uu = 0; uu < U; ++uu) {
            const int k = min(base + sub + RPW * uu, kcap - 1);
            raw[uu] = *reinterpret_cast<const uint4 *>(Lg + (size_t)k * D + cv * EPV);
        }
#pragma unroll
        for (int uu = 0; uu < U; ++uu) {
            float f[EPV];
            load16(reinterpret_cast<const T *>(&raw[uu]), f);
            // eight partial dot products, two elements per packed FMA
            float v[kTpc];
#pragma unroll
            for (int t = 0; t < kTpc; ++t) {
                float2 acc = make_float2(0.f, 0.f);
#pragma unroll
                for (int i = 0; i < EPV; i += 2)
                    acc = ffma2(make_float2(qv[t][i], qv[t][i + 1]), make_float2(f[i], f[i + 1]), acc);
                v[t] = acc.x + acc.y;
            }
            // reduce-scatter 8 values over the VPR lanes of the group
#pragma unroll
            for (int st = 0; st < 3; ++st) {
                const int o = VPR >> (st + 1);
                const int half = 4 >> st;
                const bool upper = (lane & o) != 0;
#pragma unroll
                for (int i = 0; i < 4; ++i) {
                    if (i >= half) break;
                    const float send = upper ? v[i] : v[i + half];
                    const float keep = upper ? v[i + half] : v[i];
                    v[i] = keep + __shfl_xor_sync(0xffffffffu, send, o);
                }
            }
            float tot = v[0];
#pragma unroll
            for (int o = VPR / 16; o > 0; o >>= 1) tot += __shfl_xor_sync(0xffffffffu, tot, o);
            const int k = base + sub + RPW * uu;
            if (writer && k < kcap) {
                const float sc = s.scale * tot;
                nan_seen |= isnan(sc);
                keys[my_t * kcap + k] = ord_key(sc);
            }
        }
    }
    if (nan_seen) set_status(a.status, kStatusNaN);
    __syncthreads();

    // ---- 3. per-warp top-K and the tile's list -----------------------------
    const int j = j0 + warp;
    if (j >= s.nb) return;
    const uint32_t *kw = keys + warp * kcap;
    const int first = (s.flags & SA_SINK) ? 1 : 0;
    const int n = max(0, j - first);
    const uint32_t *cand = kw + first;
    int *op = outp + warp * max(s.top_k, 1);
    const int nsel = warp_topk_positions(cand, n, s.top_k, op);
    __syncwarp();
    const size_t u = ((size_t)b * s.Hsel + hs) * s.nb + j;
    int32_t *idx = a.idx + u * s.cap;
    float *sco = a.score + u * s.cap;
    const bool sink = s.flags & SA_SINK;
    const bool loc = (s.flags & SA_LOCAL) && !(sink && j == 0);
    const int off = sink ? 1 : 0;
    const int cnt = off + nsel + (loc ? 1 : 0);
    for (int i = lane; i < s.cap; i += 32) {
        int bi = -1;
        float sv = 0.f;
        if (i < cnt) {
            if (sink && i == 0) bi = 0;
            else if (loc && i == cnt - 1) bi = j;
            else bi = first + op[i - off];
            sv = key_to_float(kw[bi]);
        }
        idx[i] = bi;
        sco[i] = sv;
    }
    if (lane == 0) a.count[u] = cnt;
}

template <typename T>
cudaError_t run_tiles(const Shape &s, const void *Q, const void *L, int32_t *idx, float *score, int32_t *count,
                      unsigned *status, cudaStream_t st) {
    TilesArgs a{};
    a.s = s;
    a.Q = Q;
    a.L = L;
    a.idx = idx;
    a.score = score;
    a.count = count;
    a.status = status;
    a.ngroups = (s.nb + kTpc - 1) / kTpc;
    const int vpr = s.d * (int)sizeof(T) / 16;
    const int kcap_max = min(s.nb, a.ngroups * kTpc);
    const size_t smem = (size_t)kTpc * s.d * 4 + (size_t)kTpc * max(s.top_k, 1) * 4 + (size_t)kTpc * kcap_max * 4;
    void (*kern)(TilesArgs) = nullptr;
    switch (vpr) {
        case 8: kern = select_tiles_kernel<T, 8>; break;
        case 16: kern = select_tiles_kernel<T, 16>; break;
        case 32: kern = select_tiles_kernel<T, 32>; break;
        default: return cudaErrorNotSupported;
    }
    cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    if (e != cudaSuccess) return e;
    kern<<<(unsigned)(s.B * s.Hsel * a.ngroups), kThreadsT, smem, st>>>(a);
    note_launch();
    return cudaGetLastError();
}

}  // namespace

bool select_tiles_supported(const Shape &s) { return s.nb <= kMaxRows && s.top_k <= 256; }

cudaError_t launch_select_tiles(const Shape &s, const void *Q, const void *L, int32_t *idx, float *score,
                                int32_t *count, unsigned *status, cudaStream_t st) {
    return s.dtype == SA_BF16 ? run_tiles<__nv_bfloat16>(s, Q, L, idx, score, count, status, st)
                              : run_tiles<float>(s, Q, L, idx, score, count, status, st);
}

}  // namespace sa
