// lsa.cu -- flat clustered index of Latent Sparse Attention (decode).
//
// The Latent Sparse Attention post, section "Индекс перестаёт перебирать
// весь контекст": adjacent keys are pooled into items; once a segment of
// items is complete it is clustered by Ward's method and frozen; the index
// keeps each cluster's centre and the positions of its items.  A query is
// scored against every centre (flat variant), the best clusters are expanded
// back to positions, the context start and a recent window are added, and the
// query attends to that set.
//
// Kernel 1 (build): one CTA per (batch, kv-head, complete segment).  Items
// (means of `pool` keys) and Ward's merges in double precision -- the merge
// order is a chain of exact comparisons, taken in the precision the index's
// definition is written in -- down to `clusters` clusters per segment; writes
// each cluster's centre and its item ids.
// Kernel 2 (decode): one CTA per (batch, kv-head).  Pooled query of the
// group's heads; scores of every centre (double); the best `top_clusters` by
// (score desc, cluster id asc); a bitmap of kept positions (sink, window,
// chosen clusters' items); then one warp per query head runs an fp32 online
// softmax over the kept positions.
#include <math_constants.h>

#include "common.cuh"
#include "lsa.cuh"

namespace sa {
namespace {

constexpr int kLsaThreads = 256;

template <typename T>
__global__ void __launch_bounds__(kLsaThreads) lsa_build_kernel(LsaShape s, const void *Kv, double *centres64,
                                                               int32_t *members, int32_t *msize) {
    extern __shared__ double sm[];
    const int D = s.d, S = s.seg;
    double *cent = sm;                                   // [S][D] cluster centres (item means at start)
    double *cost = cent + S * D;                         // [kLsaThreads] per-thread best cost
    int *csize = reinterpret_cast<int *>(cost + kLsaThreads);   // [S]
    int *owner = csize + S;                              // [S] item -> cluster id (its first item's slot)
    int *alive = owner + S;                              // [S]
    int *bpair = alive + S;                              // [kLsaThreads] per-thread best pair
    const int tid = threadIdx.x;
    const int sg = blockIdx.x % s.nseg, bg = blockIdx.x / s.nseg;
    const T *K = (const T *)Kv + (size_t)bg * s.N * D;
    // items of this segment
    for (int x = tid; x < S * D; x += kLsaThreads) {
        const int i = x / D, e = x % D;
        const int t0 = (sg * S + i) * s.pool;
        double acc = 0.0;
        for (int t = 0; t < s.pool; ++t) acc += (double)to_f(K[(size_t)(t0 + t) * D + e]);
        cent[x] = acc / s.pool;
    }
    for (int i = tid; i < S; i += kLsaThreads) {
        csize[i] = 1;
        owner[i] = i;
        alive[i] = 1;
    }
    __syncthreads();
    const int npairs = S * (S - 1) / 2;
    for (int live = S; live > s.clusters; --live) {
        // every thread: its best alive pair (a < b) by (cost, a, b)
        double best = CUDART_INF;
        int bp = 0x7fffffff;
        for (int p = tid; p < npairs; p += kLsaThreads) {
            // pair index -> (a, b), a < b, in row-major order of a
            int a = 0, rem = p;
            while (rem >= S - 1 - a) { rem -= S - 1 - a; ++a; }
            const int b = a + 1 + rem;
            if (!alive[a] || !alive[b]) continue;
            double dist = 0.0;
            for (int e = 0; e < D; ++e) {
                const double df = cent[a * D + e] - cent[b * D + e];
                dist += df * df;
            }
            const double na = csize[a], nb = csize[b];
            double c = na * nb / (na + nb) * dist;
            if (!(c <= CUDART_INF)) c = CUDART_INF;      // NaN ranks as +inf: some alive pair always wins
            const int code = a * S + b;
            if (c < best || (c == best && code < bp)) { best = c; bp = code; }
        }
        cost[tid] = best;
        bpair[tid] = bp;
        __syncthreads();
        for (int w = kLsaThreads / 2; w > 0; w >>= 1) {
            if (tid < w) {
                const double c2 = cost[tid + w];
                const int p2 = bpair[tid + w];
                if (c2 < cost[tid] || (c2 == cost[tid] && p2 < bpair[tid])) {
                    cost[tid] = c2;
                    bpair[tid] = p2;
                }
            }
            __syncthreads();
        }
        const int bp0 = bpair[0];
        if (bp0 < 0 || bp0 >= S * S) break;              // no alive pair (cannot happen while live >= 2)
        const int a = bp0 / S, b = bp0 % S;
        const double na = csize[a], nb = csize[b];
        __syncthreads();
        for (int e = tid; e < D; e += kLsaThreads) cent[a * D + e] = (na * cent[a * D + e] + nb * cent[b * D + e]) / (na + nb);
        for (int i = tid; i < S; i += kLsaThreads)
            if (owner[i] == b) owner[i] = a;
        if (tid == 0) {
            csize[a] += csize[b];
            alive[b] = 0;
        }
        __syncthreads();
    }
    // clusters numbered by their first item (surviving ids are first items)
    if (tid == 0) {
        int c = 0;
        for (int i = 0; i < S; ++i) {
            if (!alive[i]) continue;
            const size_t cid = ((size_t)bg * s.nseg + sg) * s.clusters + c;
            int m = 0;
            for (int x = 0; x < S; ++x)
                if (owner[x] == i) members[cid * S + m++] = sg * S + x;
            for (int x = m; x < S; ++x) members[cid * S + x] = -1;
            msize[cid] = m;
            alive[i] = 1000 + c;          // remember the output slot
            ++c;
        }
    }
    __syncthreads();
    for (int i = 0; i < S; ++i) {
        if (alive[i] < 1000) continue;
        const size_t cid = ((size_t)bg * s.nseg + sg) * s.clusters + (alive[i] - 1000);
        for (int e = tid; e < D; e += kLsaThreads) centres64[cid * D + e] = cent[i * D + e];
    }
}

template <typename T>
__global__ void __launch_bounds__(kLsaThreads) lsa_decode_kernel(LsaShape s, const void *qv, const void *Kv,
                                                                const void *Vv, const double *centres64,
                                                                const int32_t *members, const int32_t *msize,
                                                                double *scores, unsigned *status, void *ov,
                                                                float *lse) {
    extern __shared__ unsigned char smraw[];
    double *qbar = reinterpret_cast<double *>(smraw);                 // [D]
    double *rv = qbar + s.d;                                          // [kLsaThreads]
    int *ri = reinterpret_cast<int *>(rv + kLsaThreads);              // [kLsaThreads]
    int *chosen = ri + kLsaThreads;                                   // [top_clusters]
    unsigned *keep = reinterpret_cast<unsigned *>(chosen + max(1, s.top_clusters));   // [ceil(N / 32)]
    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    const int bg = blockIdx.x, b = bg / s.Hkv, g = bg % s.Hkv;
    const int D = s.d;
    const T *q = (const T *)qv;
    for (int e = tid; e < D; e += kLsaThreads) {
        double acc = 0.0;
        for (int h = 0; h < s.G; ++h) acc += (double)to_f(q[((size_t)b * s.Hq + g * s.G + h) * D + e]);
        qbar[e] = acc / s.G;
    }
    const int nw = (s.N + 31) / 32;
    for (int x = tid; x < nw; x += kLsaThreads) keep[x] = 0u;
    __syncthreads();
    // scores of every centre
    double *sc = scores + (size_t)bg * s.ctotal;
    const double *cb = centres64 + (size_t)bg * s.ctotal * D;
    for (int c = tid; c < s.ctotal; c += kLsaThreads) {
        double acc = 0.0;
        for (int e = 0; e < D; ++e) acc += cb[(size_t)c * D + e] * qbar[e];
        sc[c] = (double)s.scale * acc;
    }
    __syncthreads();
    // the best top_clusters, by (score desc, id asc): repeated arg-max
    const int ntop = min(s.top_clusters, s.ctotal);
    for (int r = 0; r < ntop; ++r) {
        double bv = -CUDART_INF;
        int bi = 0x7fffffff;
        for (int c = tid; c < s.ctotal; c += kLsaThreads) {
            bool taken = false;
            for (int x = 0; x < r; ++x) taken |= chosen[x] == c;
            if (taken) continue;
            const double v = isnan(sc[c]) ? -CUDART_INF : sc[c];   // NaN ranks lowest
            if (v > bv || (v == bv && c < bi)) { bv = v; bi = c; }
        }
        rv[tid] = bv;
        ri[tid] = bi;
        __syncthreads();
        for (int w = kLsaThreads / 2; w > 0; w >>= 1) {
            if (tid < w && (rv[tid + w] > rv[tid] || (rv[tid + w] == rv[tid] && ri[tid + w] < ri[tid]))) {
                rv[tid] = rv[tid + w];
                ri[tid] = ri[tid + w];
            }
            __syncthreads();
        }
        if (tid == 0) chosen[r] = ri[0];
        __syncthreads();
    }
    for (int c = tid; c < s.ctotal; c += kLsaThreads)
        if (isnan(sc[c])) set_status(status, kStatusNaN);
    // kept positions: the chosen clusters' items, the first `sink`, the last `window`
    const int qpos = s.N - 1;
    for (int r = 0; r < ntop; ++r) {
        if (chosen[r] < 0 || chosen[r] >= s.ctotal) {    // every candidate taken: nothing left to expand
            if (tid == 0) set_status(status, kStatusBadIndex);
            continue;
        }
        const size_t cid = (size_t)bg * s.ctotal + chosen[r];
        const int m = min(max(msize[cid], 0), s.seg);
        for (int x = tid; x < m * s.pool; x += kLsaThreads) {
            const int item = members[cid * s.seg + x / s.pool];
            const int t = item * s.pool + x % s.pool;
            if (item < 0 || t >= s.N) {            // not an index this build wrote: skip, report
                set_status(status, kStatusBadIndex);
                continue;
            }
            if (t <= qpos) atomicOr(&keep[t >> 5], 1u << (t & 31));
        }
    }
    for (int t = tid; t < s.N; t += kLsaThreads) {
        if (t < s.sink || (t > qpos - s.window && t <= qpos)) atomicOr(&keep[t >> 5], 1u << (t & 31));
    }
    __syncthreads();
    // one warp per query head: online softmax over the kept positions (fp32)
    const T *K = (const T *)Kv + (size_t)bg * s.N * D;
    const T *V = (const T *)Vv + (size_t)bg * s.N * D;
    constexpr int kMaxEPT = 4;                       // d <= 128
    const int ept = D / 32;
    for (int h = warp; h < s.G; h += kLsaThreads / 32) {
        const int head = g * s.G + h;
        float qh[kMaxEPT], o[kMaxEPT];
        for (int c = 0; c < kMaxEPT; ++c) {
            qh[c] = c < ept ? to_f(q[((size_t)b * s.Hq + head) * D + lane + 32 * c]) : 0.f;
            o[c] = 0.f;
        }
        float m = -CUDART_INF_F, l = 0.f;
        for (int w = 0; w < nw; ++w) {
            unsigned bits = keep[w];
            while (bits) {
                const int t = w * 32 + __ffs(bits) - 1;
                bits &= bits - 1;
                float dot = 0.f;
                for (int c = 0; c < ept; ++c) dot += qh[c] * to_f(K[(size_t)t * D + lane + 32 * c]);
                for (int off = 16; off > 0; off >>= 1) dot += __shfl_xor_sync(0xffffffffu, dot, off);
                const float z = s.scale * dot;
                const float mn = fmaxf(m, z);
                const float corr = expf(m - mn), p = expf(z - mn);
                l = l * corr + p;
                for (int c = 0; c < ept; ++c) o[c] = o[c] * corr + p * to_f(V[(size_t)t * D + lane + 32 * c]);
                m = mn;
            }
        }
        T *oh = (T *)ov + ((size_t)b * s.Hq + head) * D;
        const float inv = l > 0.f ? 1.f / l : 0.f;
        for (int c = 0; c < ept; ++c) from_f(oh[lane + 32 * c], o[c] * inv);
        if (lane == 0) lse[(size_t)b * s.Hq + head] = l > 0.f ? m + logf(l) : -CUDART_INF_F;
    }
}

}  // namespace

size_t lsa_build_smem(const LsaShape &s) {
    return sizeof(double) * ((size_t)s.seg * s.d + kLsaThreads) + sizeof(int) * (3 * (size_t)s.seg + kLsaThreads);
}

cudaError_t launch_lsa_build(const LsaShape &s, const void *K, double *centres, int32_t *members, int32_t *sizes,
                             cudaStream_t st) {
    if (s.nseg == 0) return cudaSuccess;
    const size_t smem = lsa_build_smem(s);
    void (*kern)(LsaShape, const void *, double *, int32_t *, int32_t *) =
        s.dtype == SA_BF16 ? lsa_build_kernel<__nv_bfloat16> : lsa_build_kernel<float>;
    cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    if (e != cudaSuccess) return e;
    kern<<<(unsigned)(s.B * s.Hkv * s.nseg), kLsaThreads, smem, st>>>(s, K, centres, members, sizes);
    note_launch();
    return cudaGetLastError();
}

cudaError_t launch_lsa_decode(const LsaShape &s, const void *q, const void *K, const void *V, const double *centres,
                              const int32_t *members, const int32_t *sizes, double *scores, unsigned *status, void *o,
                              float *lse, cudaStream_t st) {
    const size_t smem = sizeof(double) * ((size_t)s.d + kLsaThreads) +
                        sizeof(int) * (kLsaThreads + (size_t)max(1, s.top_clusters)) +
                        sizeof(unsigned) * (((size_t)s.N + 31) / 32);
    void (*kern)(LsaShape, const void *, const void *, const void *, const double *, const int32_t *, const int32_t *,
                 double *, unsigned *, void *, float *) =
        s.dtype == SA_BF16 ? lsa_decode_kernel<__nv_bfloat16> : lsa_decode_kernel<float>;
    cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    if (e != cudaSuccess) return e;
    kern<<<(unsigned)(s.B * s.Hkv), kLsaThreads, smem, st>>>(s, q, K, V, centres, members, sizes, scores, status, o,
                                                             lse);
    note_launch();
    return cudaGetLastError();
}

}  // namespace sa
