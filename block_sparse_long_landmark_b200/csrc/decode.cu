// decode.cu -- block-sparse decode: one query per sequence over a full KV
// cache, reading only the kept blocks.
//
// [HiLS] "Ключевые факты": sparse access to the KV cache; the Latent Sparse
// Attention post (section "Ускорение видно на слое, но дерево пока требует
// проверки"): the cache itself stays whole, only the reads shrink.  Gated
// mode follows [SAS] "Как это применить" (log gate inside the softmax,
// normalised against the current block); hierarchical mode follows [HiLS]'s
// opening section (per-block softmax, outputs weighted by softmax_b(s_b)).
//
// Split-K over the kept list: CTA (unit, split) reads `bps` kept blocks,
// keeps a per-head running (max, sum, acc) -- in hierarchical mode the max
// and sum run over the retrieval scores and acc sums e^{s_b} * o_b -- and
// leaves the triple in the workspace; a merge kernel combines the splits by
// log-sum-exp.  All query heads of a kv-head group share the blocks they read.
#include <math_constants.h>

#include "bounds.cuh"
#include "common.cuh"

namespace sa {

constexpr int kDecThreads = 256;
constexpr int kMaxPairsPerThread = 4;

struct DecArgs {
    Shape s;
    const void *q, *K, *V;
    const int32_t *idx;
    const float *score;
    const int32_t *count;
    void *o;
    float *lse;
    unsigned *status;
    float *part;   // [units][S][HP][d + 2]
    // tensor-core records: [units] records written (the merge waits until a
    // unit's count reaches S), [units] merge CTAs done; null otherwise
    unsigned *ucnt, *mcnt;
    int S, bps;
};

template <typename T>
__global__ void __launch_bounds__(kDecThreads) decode_split_kernel(DecArgs a) {
    constexpr float kLog2e = 1.4426950408889634f;
    constexpr float kLn2 = 0.6931471805599453f;
    const Shape &s = a.s;
    const int d = s.d, HP = s.heads_per, bs = s.bs;
    const int kstride = d + 16 / (int)sizeof(T);   // padded K rows: conflict-free 16-byte reads
    extern __shared__ __align__(16) unsigned char smem_raw[];
    float *qs = reinterpret_cast<float *>(smem_raw);                 // [HP][d], pre-scaled
    float *pz = qs + HP * d;                                         // [HP][bs]
    float *stat = pz + HP * bs;                                      // [HP][4]: m, l, corr, f
    T *Ks = reinterpret_cast<T *>(stat + HP * 4);                    // [bs][kstride]
    T *Vs = Ks + (size_t)bs * kstride;                               // [bs][d]

    const int u = blockIdx.x / a.S, split = blockIdx.x % a.S;
    const int hs = u % s.Hsel, b = u / s.Hsel;
    const bool perq = s.flags & SA_SELECT_PER_QHEAD;
    const int g = perq ? hs / s.G : hs;
    const int h0 = perq ? hs : hs * s.G;
    const int32_t *idx = a.idx + (size_t)u * s.cap;
    const float *sc = a.score + (size_t)u * s.cap;
    const int cnt = min(a.count[u], s.cap);
    const int nseq = seq_n(s, b);                       // this sequence's context length
    const int local = (nseq - 1) / bs;
    const bool hier = s.flags & SA_HIER, gate_on = s.flags & SA_GATE;
    const float s_local = cnt > 0 ? sc[cnt - 1] : 0.f;

    const T *qg = (const T *)a.q + ((size_t)b * s.Hq + h0) * d;
    for (int e = threadIdx.x; e < HP * d; e += kDecThreads) qs[e] = to_f(qg[e]) * (s.scale * kLog2e);
    if (threadIdx.x < HP) {
        stat[threadIdx.x * 4 + 0] = -CUDART_INF_F;
        stat[threadIdx.x * 4 + 1] = 0.f;
    }
    const int npairs = HP * d / 2;
    float acc[kMaxPairsPerThread][2];
#pragma unroll
    for (int r = 0; r < kMaxPairsPerThread; ++r) acc[r][0] = acc[r][1] = 0.f;

    const T *Kg = (const T *)a.K + ((size_t)b * s.Hkv + g) * (size_t)s.N * d;
    const T *Vg = (const T *)a.V + ((size_t)b * s.Hkv + g) * (size_t)s.N * d;
    const int c0 = split * a.bps, c1 = min(cnt, c0 + a.bps);
    for (int c = c0; c < c1; ++c) {
        const int blk = idx[c];
        const bool bad = blk < 0 || blk > local || (c > 0 && idx[c - 1] >= blk);
        if (bad) {
            if (threadIdx.x == 0) set_status(a.status, kStatusBadIndex);
            continue;
        }
        const bool forced = (blk == local && (s.flags & SA_LOCAL)) || (blk == 0 && (s.flags & SA_SINK));
        const float gate = (gate_on && !forced) ? log_sigmoid(sc[c] - s_local) * kLog2e : 0.f;
        const int t0 = blk * bs, nk = min(bs, nseq - t0);
        SA_CHECK_START(a.status, t0, nseq);
        __syncthreads();
        {
            constexpr int EPV = Vec<T>::n;
            const int vpr = d / EPV;
            const T *ks = Kg + (size_t)t0 * d, *vs = Vg + (size_t)t0 * d;
            for (int e = threadIdx.x; e < nk * vpr; e += kDecThreads) {
                const int t = e / vpr, cv = e % vpr;
                *reinterpret_cast<uint4 *>(Ks + (size_t)t * kstride + cv * EPV) =
                    *reinterpret_cast<const uint4 *>(ks + (size_t)t * d + cv * EPV);
                reinterpret_cast<uint4 *>(Vs)[e] = reinterpret_cast<const uint4 *>(vs)[e];
            }
        }
        __syncthreads();
        // logits (log2 units)
        for (int e = threadIdx.x; e < HP * bs; e += kDecThreads) {
            const int hh = e / bs, t = e % bs;
            float z = -CUDART_INF_F;
            if (t < nk) {
                const T *kr = Ks + (size_t)t * kstride;
                const float *qr = qs + hh * d;
                float dot = 0.f;
                for (int v = 0; v < d; v += Vec<T>::n) {
                    float f[Vec<T>::n];
                    load16(kr + v, f);
#pragma unroll
                    for (int w = 0; w < Vec<T>::n; ++w) dot = fmaf(qr[v + w], f[w], dot);
                }
                z = dot + (hier ? 0.f : gate);
            }
            pz[e] = z;
        }
        __syncthreads();
        // per-head softmax update: one warp per head
        for (int hh = threadIdx.x >> 5; hh < HP; hh += kDecThreads / 32) {
            const int lane = threadIdx.x & 31;
            float bm = -CUDART_INF_F;
            for (int t = lane; t < bs; t += 32) bm = fmaxf(bm, pz[hh * bs + t]);
#pragma unroll
            for (int o = 16; o > 0; o >>= 1) bm = fmaxf(bm, __shfl_xor_sync(0xffffffffu, bm, o));
            float *st = stat + hh * 4;
            const float m_old = st[0];
            if (!hier) {
                const float nm = fmaxf(m_old, bm);
                float ls = 0.f;
                for (int t = lane; t < bs; t += 32) {
                    const float p = nm == -CUDART_INF_F ? 0.f : exp2f(pz[hh * bs + t] - nm);
                    pz[hh * bs + t] = p;
                    ls += p;
                }
#pragma unroll
                for (int o = 16; o > 0; o >>= 1) ls += __shfl_xor_sync(0xffffffffu, ls, o);
                __syncwarp();
                if (lane == 0) {
                    const float corr = m_old == -CUDART_INF_F ? 0.f : exp2f(m_old - nm);
                    st[2] = corr;
                    st[1] = st[1] * corr + ls;
                    st[0] = nm;
                }
            } else {
                float ls = 0.f;
                for (int t = lane; t < bs; t += 32) {
                    const float p = bm == -CUDART_INF_F ? 0.f : exp2f(pz[hh * bs + t] - bm);
                    pz[hh * bs + t] = p;
                    ls += p;
                }
#pragma unroll
                for (int o = 16; o > 0; o >>= 1) ls += __shfl_xor_sync(0xffffffffu, ls, o);
                __syncwarp();
                if (lane == 0) {
                    if (ls > 0.f) {
                        const float sb = sc[c] * kLog2e;
                        const float nM = fmaxf(m_old, sb);
                        const float corr = m_old == -CUDART_INF_F ? 0.f : exp2f(m_old - nM);
                        const float wb = exp2f(sb - nM);
                        st[2] = corr;
                        st[3] = wb / ls;
                        st[1] = st[1] * corr + wb;
                        st[0] = nM;
                    } else {
                        st[2] = 1.f;
                        st[3] = 0.f;
                    }
                }
                __syncwarp();
                const float f = st[3];
                for (int t = lane; t < bs; t += 32) pz[hh * bs + t] *= f;
            }
        }
        __syncthreads();
        // acc = acc * corr + sum_t p_t v_t
#pragma unroll
        for (int r = 0; r < kMaxPairsPerThread; ++r) {
            const int e = threadIdx.x + r * kDecThreads;
            if (e >= npairs) break;
            const int hh = (2 * e) / d, dim = (2 * e) % d;
            const float corr = stat[hh * 4 + 2];
            float a0 = acc[r][0] * corr, a1 = acc[r][1] * corr;
            const float *pr = pz + hh * bs;
            for (int t = 0; t < nk; ++t) {
                const float p = pr[t];
                const float v0 = to_f(Vs[(size_t)t * d + dim]), v1 = to_f(Vs[(size_t)t * d + dim + 1]);
                a0 = fmaf(p, v0, a0);
                a1 = fmaf(p, v1, a1);
            }
            acc[r][0] = a0;
            acc[r][1] = a1;
        }
    }
    __syncthreads();
    if (a.S == 1) {
        T *og = (T *)a.o + ((size_t)b * s.Hq + h0) * d;
#pragma unroll
        for (int r = 0; r < kMaxPairsPerThread; ++r) {
            const int e = threadIdx.x + r * kDecThreads;
            if (e >= npairs) break;
            const int hh = (2 * e) / d, dim = (2 * e) % d;
            const float L = stat[hh * 4 + 1];
            const float inv = L > 0.f ? 1.f / L : 0.f;
            from_f(og[hh * d + dim], acc[r][0] * inv);
            from_f(og[hh * d + dim + 1], acc[r][1] * inv);
        }
        if (threadIdx.x < HP) {
            const float m = stat[threadIdx.x * 4], L = stat[threadIdx.x * 4 + 1];
            a.lse[(size_t)b * s.Hq + h0 + threadIdx.x] = L > 0.f ? (m + log2f(L)) * kLn2 : -CUDART_INF_F;
        }
        return;
    }
    float *pp = a.part + ((size_t)u * a.S + split) * HP * (d + 2);
#pragma unroll
    for (int r = 0; r < kMaxPairsPerThread; ++r) {
        const int e = threadIdx.x + r * kDecThreads;
        if (e >= npairs) break;
        const int hh = (2 * e) / d, dim = (2 * e) % d;
        pp[hh * (d + 2) + 2 + dim] = acc[r][0];
        pp[hh * (d + 2) + 2 + dim + 1] = acc[r][1];
    }
    if (threadIdx.x < HP) {
        pp[threadIdx.x * (d + 2)] = stat[threadIdx.x * 4];
        pp[threadIdx.x * (d + 2) + 1] = stat[threadIdx.x * 4 + 1];
    }
}

// One CTA per (unit, query head of the unit): the unit's R = a.S partial
// records of that head (m, l, acc[d]) combined by log-sum-exp.  Each thread
// takes whole output dimensions: the max M over the records' m, then L and O
// weighted by 2^(m - M), empty records (m = -inf) skipped; up to 16 records
// are read in one round of independent loads.
// Records of the tensor-core decode come with a per-unit count: the launch
// starts while the decode still runs and each CTA waits (bounded) only for
// its own unit's R records; the unit's last merge CTA clears both counters.
// Otherwise the CTA waits for the whole previous launch.
constexpr int kMergeThreads = 128;
constexpr int kMergeRegR = 16;        // records held in registers (more: two passes over them)
constexpr unsigned long long kMergeWaitNs = 2000000000ull;

__device__ __forceinline__ unsigned ld_acquire_u32(const unsigned *p) {
    unsigned v;
    asm volatile("ld.acquire.gpu.global.u32 %0, [%1];" : "=r"(v) : "l"(p) : "memory");
    return v;
}

template <typename T>
__global__ void __launch_bounds__(kMergeThreads) decode_merge_kernel(DecArgs a) {
    constexpr float kLn2 = 0.6931471805599453f;
    __shared__ int gave_up;
    const Shape &s = a.s;
    const int d = s.d, HP = s.heads_per, R = a.S;
    const int u = blockIdx.x / HP, hh = blockIdx.x % HP;   // a unit's heads side by side
    if (a.ucnt) {
        if (threadIdx.x == 0) {
            gave_up = 0;
            unsigned long long t0, t;
            asm volatile("mov.u64 %0, %%globaltimer;" : "=l"(t0));
            while (ld_acquire_u32(a.ucnt + u) < (unsigned)R) {
                // the decode gave up (its own wait ran out): no records will come
                if (*(volatile unsigned *)a.status & kStatusTimeout) { gave_up = 1; break; }
                asm volatile("mov.u64 %0, %%globaltimer;" : "=l"(t));
                if (t - t0 > kMergeWaitNs) {
                    set_status(a.status, kStatusTimeout);
                    gave_up = 1;
                    break;
                }
                __nanosleep(256);
            }
        }
        __syncthreads();
        if (gave_up) return;
    } else {
        asm volatile("griddepcontrol.wait;" ::: "memory");   // the records of the launch before this one
    }
    const int hs = u % s.Hsel, b = u / s.Hsel;
    const int h0 = (s.flags & SA_SELECT_PER_QHEAD) ? hs : hs * s.G;
    const size_t rs = (size_t)HP * (d + 2);                  // record stride
    const float *pp = a.part + (size_t)u * R * rs + (size_t)hh * (d + 2);
    T *orow = (T *)a.o + ((size_t)b * s.Hq + h0 + hh) * d;
    for (int dim = threadIdx.x; dim < d; dim += kMergeThreads) {
        float M = -CUDART_INF_F, L = 0.f, O = 0.f;
        if (R <= kMergeRegR) {
            // every record's (m, l, acc[dim]) in one round of independent loads
            float mr[kMergeRegR], lr[kMergeRegR], ar[kMergeRegR];
#pragma unroll
            for (int r = 0; r < kMergeRegR; ++r) {
                mr[r] = r < R ? __ldcg(pp + r * rs) : -CUDART_INF_F;
                lr[r] = r < R ? __ldcg(pp + r * rs + 1) : 0.f;
                ar[r] = r < R ? __ldcg(pp + r * rs + 2 + dim) : 0.f;
            }
#pragma unroll
            for (int r = 0; r < kMergeRegR; ++r) M = fmaxf(M, mr[r]);
            if (M != -CUDART_INF_F) {
#pragma unroll
                for (int r = 0; r < kMergeRegR; ++r)
                    if (mr[r] != -CUDART_INF_F) {
                        const float w = exp2f(mr[r] - M);
                        L = fmaf(lr[r], w, L);
                        O = fmaf(ar[r], w, O);
                    }
            }
        } else {
            for (int r = 0; r < R; ++r) M = fmaxf(M, __ldcg(pp + r * rs));
            if (M != -CUDART_INF_F) {
#pragma unroll 4
                for (int r = 0; r < R; ++r) {
                    const float m = __ldcg(pp + r * rs);
                    if (m != -CUDART_INF_F) {
                        const float w = exp2f(m - M);
                        L = fmaf(__ldcg(pp + r * rs + 1), w, L);
                        O = fmaf(__ldcg(pp + r * rs + 2 + dim), w, O);
                    }
                }
            }
        }
        from_f(orow[dim], L > 0.f ? O / L : 0.f);
        if (dim == 0) a.lse[(size_t)b * s.Hq + h0 + hh] = L > 0.f ? (M + log2f(L)) * kLn2 : -CUDART_INF_F;
    }
    if (a.ucnt) {
        // every read of this CTA is done; the unit's last merge CTA clears the counters
        __syncthreads();
        if (threadIdx.x == 0 && atomicAdd(a.mcnt + u, 1u) == (unsigned)HP - 1) {
            a.ucnt[u] = 0u;
            a.mcnt[u] = 0u;
        }
    }
}


template <typename T>
static cudaError_t launch_merge(const DecArgs &a, cudaStream_t st, bool pdl) {
    const dim3 grid((unsigned)(a.s.B * a.s.Hsel * a.s.heads_per));
    cudaError_t e = pdl ? launch_pdl(decode_merge_kernel<T>, grid, dim3(kMergeThreads), 0, st, a)
                        : (decode_merge_kernel<T><<<grid, kMergeThreads, 0, st>>>(a), cudaSuccess);
    note_launch();
    return e != cudaSuccess ? e : cudaGetLastError();
}

static void split_geometry(const Shape &s, int &S, int &bps) {
    const int units = s.B * s.Hsel;
    const int want = (2 * 148 + units - 1) / units;
    S = max(1, min(want, s.cap));
    bps = (s.cap + S - 1) / S;
    S = (s.cap + bps - 1) / bps;
}

size_t decode_workspace(const Shape &s) {
    int S, bps;
    if (decode_mma_supported(s)) {
        decode_mma_geometry(s, S, bps);
        return decode_mma_partial_bytes(s, S);
    }
    split_geometry(s, S, bps);
    if (S == 1) return 0;
    return (size_t)s.B * s.Hsel * S * s.heads_per * (s.d + 2) * sizeof(float);
}

template <typename T>
static cudaError_t run(DecArgs a, cudaStream_t st) {
    const Shape &s = a.s;
    if (s.heads_per * s.d / 2 > kMaxPairsPerThread * kDecThreads) return cudaErrorInvalidValue;
    const size_t smem = (size_t)s.heads_per * (s.d + s.bs + 4) * sizeof(float) +
                        (size_t)s.bs * (2 * s.d + 16 / sizeof(T)) * sizeof(T);
    cudaError_t e = cudaFuncSetAttribute(decode_split_kernel<T>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                         (int)smem);
    if (e != cudaSuccess) return e;
    const unsigned units = (unsigned)(s.B * s.Hsel);
    decode_split_kernel<T><<<units * a.S, kDecThreads, smem, st>>>(a);
    note_launch();
    e = cudaGetLastError();
    if (e != cudaSuccess || a.S == 1) return e;
    return launch_merge<T>(a, st, false);
}

cudaError_t launch_decode(const Shape &s, const void *q, const void *K, const void *V, const int32_t *idx,
                          const float *score, const int32_t *count, void *o, float *lse, unsigned *status,
                          unsigned *ucnt, float *part, cudaStream_t st, const unsigned *ready, unsigned epoch) {
    DecArgs a{};
    a.s = s;
    a.q = q;
    a.K = K;
    a.V = V;
    a.idx = idx;
    a.score = score;
    a.count = count;
    a.o = o;
    a.lse = lse;
    a.status = status;
    a.part = part;
    if (decode_mma_supported(s)) {
        // tensor-core item records, counted per unit; the merge launch starts
        // early and takes each unit as soon as its records are in
        int R = 1;
        cudaError_t e = launch_decode_mma(s, q, K, V, idx, score, count, status, ucnt, part, st, R, ready, epoch);
        if (e != cudaSuccess) return e;
        a.S = R;
        a.ucnt = ucnt;
        a.mcnt = ucnt + (size_t)s.B * s.Hsel;
        return launch_merge<__nv_bfloat16>(a, st, true);
    }
    split_geometry(s, a.S, a.bps);
    return s.dtype == SA_BF16 ? run<__nv_bfloat16>(a, st) : run<float>(a, st);
}

}  // namespace sa
