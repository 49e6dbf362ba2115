// backward.cu -- backward pass of gated block-sparse prefill (CUDA cores, fp32).
//
// [SAS] "Как это применить": the selector's score enters the attention as a
// gate log_sigmoid(s_b - s_local) inside the softmax, so the loss reaches the
// selector through it ("Ключевые факты": the top-K choice itself is hard and
// carries no gradient).  With the kept lists of the forward pass fixed:
//
//   P = exp(z - lse),  D_i = <dO_i, O_i>,  dZ = P (dO V^T - D)
//   dQ = scale dZ K,   dK += scale dZ^T Q,  dV += P^T dO
//   dg_c = sum of dZ over the unit's rows and the keys of entry c
//   ds_c = dg_c sigmoid(-(s_c - s_loc)) for gated entries, ds_loc = -sum of them
// and, for the selector (separate entry point):
//   qbar = mean of the unit's rows,  dqbar = scale sum_c ds_c L_c,
//   dQ[rows] += dqbar / R,  dL_c += scale ds_c qbar,  dK[keys of b] += dL_b / n_b
// (the landmarks' rounding to the key precision is taken as the identity).
//
// Kernel A: one CTA per (unit, 64-row chunk of the unit's G * block rows);
// it walks the kept blocks in 32-key chunks: the chunk's K and V in shared
// memory, z and dO.V for 64 x 32 pairs (8 per thread), then dQ (kept in
// registers), dK and dV (fp32 atomics into the caller's buffers).
// Kernel B turns the gate gradients into score gradients per unit.
// Kernel C (selector): per unit, pooled query, dqbar into dQ, dL by atomics.
// Kernel D: dK += dL_b / n_b for every key.
#include <math_constants.h>

#include <algorithm>

#include "backward_tc.cuh"
#include "common.cuh"

namespace sa {
namespace {

constexpr int kBwThreads = 256;
constexpr int kRC = 64;    // query rows per CTA
constexpr int kKC = 32;    // keys per step

struct BwArgs {
    Shape s;
    const void *Q, *K, *V, *O, *dO;
    const float *lse;
    const int32_t *idx;
    const float *score;
    const int32_t *count;
    float *dQ, *dK, *dV, *dgate;   // dgate: [units][cap], summed over row chunks
    unsigned *status;
    int rchunks;
};

template <typename T>
__device__ __forceinline__ float ld1(const T *p) { return to_f(*p); }

// N = 2 or 4 consecutive floats (8- or 16-byte aligned)
template <int N>
__device__ __forceinline__ void vload(const float *p, float *v) {
    if constexpr (N == 4) {
        const float4 x = *reinterpret_cast<const float4 *>(p);
        v[0] = x.x; v[1] = x.y; v[2] = x.z; v[3] = x.w;
    } else {
        const float2 x = *reinterpret_cast<const float2 *>(p);
        v[0] = x.x; v[1] = x.y;
    }
}
template <int N>
__device__ __forceinline__ void vatomic_add(float *p, const float *v) {
    if constexpr (N == 4) atomicAdd(reinterpret_cast<float4 *>(p), make_float4(v[0], v[1], v[2], v[3]));
    else atomicAdd(reinterpret_cast<float2 *>(p), make_float2(v[0], v[1]));
}

template <typename T, int D>
__global__ void __launch_bounds__(kBwThreads) bwd_attn_kernel(BwArgs a) {
    const Shape &s = a.s;
    constexpr int DP = D + 1;                       // padded rows for per-key access
    extern __shared__ float smem[];
    float *sq = smem;                                // [kRC][D]
    float *sdo = sq + kRC * D;                       // [kRC][D]
    float *sk = sdo + kRC * D;                       // [kKC][DP]
    float *sv = sk + kKC * DP;                       // [kKC][DP]
    float *sP = sv + kKC * DP;                       // [kRC][kKC + 1]
    float *sZ = sP + kRC * (kKC + 1);                // [kRC][kKC + 1]
    float *sD = sZ + kRC * (kKC + 1);                // [kRC]
    float *sL = sD + kRC;                            // [kRC] lse
    int *spos = reinterpret_cast<int *>(sL + kRC);   // [kRC] query position, -1 = no row
    float *sdg = reinterpret_cast<float *>(spos + kRC);   // [1]

    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    const int u = blockIdx.x / a.rchunks, rc = blockIdx.x % a.rchunks;
    const int j = u % s.nb, g = (u / s.nb) % s.Hkv, b = u / (s.nb * s.Hkv);
    const int R = s.G * s.bs;
    const T *Q = (const T *)a.Q, *K = (const T *)a.K, *V = (const T *)a.V, *O = (const T *)a.O,
            *dO = (const T *)a.dO;

    // ---- rows of this chunk: q, dO, D = <dO, O>, lse ------------------------
    for (int i = warp; i < kRC; i += kBwThreads / 32) {
        const int r = rc * kRC + i;
        const int h = g * s.G + r / s.bs, pos = j * s.bs + r % s.bs;
        const bool ok = r < R && pos < s.N;
        const size_t row = (((size_t)b * s.Hq + (ok ? h : 0)) * s.N + (ok ? pos : 0)) * D;
        float dsum = 0.f;
        for (int e = lane; e < D; e += 32) {
            const float qv = ok ? ld1(Q + row + e) : 0.f;
            const float dv = ok ? ld1(dO + row + e) : 0.f;
            const float ov = ok ? ld1(O + row + e) : 0.f;
            sq[i * D + e] = qv;
            sdo[i * D + e] = dv;
            dsum += dv * ov;
        }
#pragma unroll
        for (int o = 16; o > 0; o >>= 1) dsum += __shfl_xor_sync(0xffffffffu, dsum, o);
        if (lane == 0) {
            sD[i] = dsum;
            sL[i] = ok ? a.lse[((size_t)b * s.Hq + h) * s.N + pos] : -CUDART_INF_F;
            spos[i] = ok ? pos : -1;
        }
    }
    __syncthreads();

    constexpr int EPT = D / 32;                      // dQ columns per thread
    float dq[8][EPT];                                // rows warp + 8m, columns lane + 32c
#pragma unroll
    for (int m = 0; m < 8; ++m)
#pragma unroll
        for (int c = 0; c < EPT; ++c) dq[m][c] = 0.f;

    const size_t lu = ((size_t)b * s.Hkv + g) * s.nb + j;
    const int cnt = max(0, min(a.count[lu], s.cap));
    const int32_t *il = a.idx + lu * s.cap;
    const float *sl = a.score + lu * s.cap;
    const float s_loc = cnt > 0 ? sl[cnt - 1] : 0.f;
    const bool causal = s.flags & SA_CAUSAL;
    const size_t kvhead = ((size_t)b * s.Hkv + g) * s.N;

    for (int c = 0; c < cnt; ++c) {
        const int blk = il[c];
        if (!(blk >= 0 && blk <= j && (c == 0 || il[c - 1] < blk))) {
            if (tid == 0 && rc == 0) set_status(a.status, kStatusBadIndex);
            continue;
        }
        const bool forced = (blk == j && (s.flags & SA_LOCAL)) || (blk == 0 && (s.flags & SA_SINK));
        const float gate = ((s.flags & SA_GATE) && !forced) ? log_sigmoid(sl[c] - s_loc) : 0.f;
        const int t0 = blk * s.bs, t1 = min(t0 + s.bs, s.N);
        float dg = 0.f;
        for (int kc = t0; kc < t1; kc += kKC) {
            __syncthreads();                             // previous step's readers are done
            for (int x = tid; x < kKC * D; x += kBwThreads) {
                const int t = x / D, e = x % D;
                const int key = kc + t;
                const bool kok = key < t1;
                sk[t * DP + e] = kok ? ld1(K + (kvhead + key) * D + e) : 0.f;
                sv[t * DP + e] = kok ? ld1(V + (kvhead + key) * D + e) : 0.f;
            }
            __syncthreads();
            // z and dO.V for (row warp + 8m, key lane)
            {
                const int t = lane, key = kc + t;
                float z[8], dp[8];
#pragma unroll
                for (int m = 0; m < 8; ++m) z[m] = dp[m] = 0.f;
                // row operands as 16-byte broadcast loads, key operands per lane
                for (int e = 0; e < D; e += 4) {
                    float kv[4], vv[4];
#pragma unroll
                    for (int x = 0; x < 4; ++x) {
                        kv[x] = sk[t * DP + e + x];
                        vv[x] = sv[t * DP + e + x];
                    }
#pragma unroll
                    for (int m = 0; m < 8; ++m) {
                        const float4 q4 = *reinterpret_cast<const float4 *>(sq + (warp + 8 * m) * D + e);
                        const float4 d4 = *reinterpret_cast<const float4 *>(sdo + (warp + 8 * m) * D + e);
                        z[m] = fmaf(q4.x, kv[0], fmaf(q4.y, kv[1], fmaf(q4.z, kv[2], fmaf(q4.w, kv[3], z[m]))));
                        dp[m] = fmaf(d4.x, vv[0], fmaf(d4.y, vv[1], fmaf(d4.z, vv[2], fmaf(d4.w, vv[3], dp[m]))));
                    }
                }
#pragma unroll
                for (int m = 0; m < 8; ++m) {
                    const int i = warp + 8 * m;
                    const int pos = spos[i];
                    const bool vis = pos >= 0 && key < t1 && !(causal && blk == j && key > pos) &&
                                     sL[i] != -CUDART_INF_F;
                    const float p = vis ? expf(fmaf(s.scale, z[m], gate) - sL[i]) : 0.f;
                    const float dz = p * (dp[m] - sD[i]);
                    sP[i * (kKC + 1) + t] = p;
                    sZ[i * (kKC + 1) + t] = dz;
                    dg += dz;
                }
            }
            __syncthreads();
            // dQ (rows warp + 8m, columns lane + 32c) += scale dZ K
            for (int t = 0; t < kKC; ++t) {
#pragma unroll
                for (int m = 0; m < 8; ++m) {
                    const float w = sZ[(warp + 8 * m) * (kKC + 1) + t];
#pragma unroll
                    for (int cc = 0; cc < EPT; ++cc) dq[m][cc] = fmaf(w, sk[t * DP + lane + 32 * cc], dq[m][cc]);
                }
            }
            // dK, dV (keys warp + 8m', columns lane*EPT .. lane*EPT+EPT-1): each
            // row's q and dO slices are loaded once (vector loads) for the
            // thread's four keys; one vector atomic per key and lane at the end
            {
                constexpr int KT = kKC / 8;
                float ak[KT][EPT], av[KT][EPT];
#pragma unroll
                for (int m = 0; m < KT; ++m)
#pragma unroll
                    for (int cc = 0; cc < EPT; ++cc) ak[m][cc] = av[m][cc] = 0.f;
                for (int i = 0; i < kRC; ++i) {
                    float qv[EPT], dv[EPT];
                    vload<EPT>(sq + i * D + lane * EPT, qv);
                    vload<EPT>(sdo + i * D + lane * EPT, dv);
#pragma unroll
                    for (int m = 0; m < KT; ++m) {
                        const float wz = sZ[i * (kKC + 1) + warp + 8 * m], wp = sP[i * (kKC + 1) + warp + 8 * m];
#pragma unroll
                        for (int cc = 0; cc < EPT; ++cc) {
                            ak[m][cc] = fmaf(wz, qv[cc], ak[m][cc]);
                            av[m][cc] = fmaf(wp, dv[cc], av[m][cc]);
                        }
                    }
                }
#pragma unroll
                for (int m = 0; m < KT; ++m) {
                    const int key = kc + warp + 8 * m;
                    if (key < t1) {
#pragma unroll
                        for (int cc = 0; cc < EPT; ++cc) ak[m][cc] *= s.scale;
                        vatomic_add<EPT>(a.dK + (kvhead + key) * D + lane * EPT, ak[m]);
                        vatomic_add<EPT>(a.dV + (kvhead + key) * D + lane * EPT, av[m]);
                    }
                }
            }
        }
        // the entry's gate gradient: block sum, then one atomic per CTA
#pragma unroll
        for (int o = 16; o > 0; o >>= 1) dg += __shfl_xor_sync(0xffffffffu, dg, o);
        if (tid == 0) *sdg = 0.f;
        __syncthreads();
        if (lane == 0) atomicAdd(sdg, dg);
        __syncthreads();
        if (tid == 0) atomicAdd(a.dgate + lu * s.cap + c, *sdg);
    }
    // ---- dQ rows --------------------------------------------------------------
#pragma unroll
    for (int m = 0; m < 8; ++m) {
        const int i = warp + 8 * m;
        const int pos = spos[i];
        if (pos < 0) continue;
        const int r = rc * kRC + i;
        const int h = g * s.G + r / s.bs;
        float *dst = a.dQ + (((size_t)b * s.Hq + h) * s.N + pos) * D;
#pragma unroll
        for (int cc = 0; cc < EPT; ++cc) dst[lane + 32 * cc] = s.scale * dq[m][cc];
    }
}

// Kernel B: per unit, score gradients from the gate gradients.
__global__ void bwd_score_kernel(Shape s, const int32_t *idx, const float *score, const int32_t *count,
                                 const float *dgate, float *dscore, int units) {
    const int u = blockIdx.x * blockDim.x + threadIdx.x;
    if (u >= units) return;
    const int j = u % s.nb;
    const int cnt = max(0, min(count[u], s.cap));
    const int32_t *il = idx + (size_t)u * s.cap;
    const float *sl = score + (size_t)u * s.cap;
    float *ds = dscore + (size_t)u * s.cap;
    const float *dg = dgate + (size_t)u * s.cap;
    const float s_loc = cnt > 0 ? sl[cnt - 1] : 0.f;
    float sum = 0.f;
    int loc = -1;
    for (int c = 0; c < s.cap; ++c) {
        float v = 0.f;
        if (c < cnt) {
            const int blk = il[c];
            const bool forced = (blk == j && (s.flags & SA_LOCAL)) || (blk == 0 && (s.flags & SA_SINK));
            if (blk == j) loc = c;
            if ((s.flags & SA_GATE) && !forced) {
                const float x = sl[c] - s_loc;
                v = dg[c] / (1.f + expf(x));          // dg * sigmoid(-x)
                sum += v;
            }
        }
        ds[c] = v;
    }
    if (loc >= 0) ds[loc] -= sum;
}

// Kernel C: the selector chain of one unit (one warp per unit).
template <typename T, int D>
__global__ void sel_bwd_kernel(Shape s, const void *Qv, const void *Lv, const int32_t *idx, const float *dscore,
                               const int32_t *count, float *dQ, float *dL, int units) {
    constexpr int EPT = D / 32;
    const int u = blockIdx.x * (blockDim.x / 32) + (threadIdx.x >> 5);
    const int lane = threadIdx.x & 31;
    if (u >= units) return;
    const int j = u % s.nb, g = (u / s.nb) % s.Hkv, b = u / (s.nb * s.Hkv);
    const T *Q = (const T *)Qv, *L = (const T *)Lv;
    const int r0 = j * s.bs, nrows = min(s.bs, s.N - r0);
    const int R = s.G * nrows;
    float qb[EPT];
#pragma unroll
    for (int c = 0; c < EPT; ++c) qb[c] = 0.f;
    for (int h = g * s.G; h < (g + 1) * s.G; ++h)
        for (int r = 0; r < nrows; ++r) {
            const T *row = Q + (((size_t)b * s.Hq + h) * s.N + r0 + r) * D;
#pragma unroll
            for (int c = 0; c < EPT; ++c) qb[c] += to_f(row[lane + 32 * c]);
        }
#pragma unroll
    for (int c = 0; c < EPT; ++c) qb[c] /= (float)R;
    const int cnt = max(0, min(count[u], s.cap));
    const int32_t *il = idx + (size_t)u * s.cap;
    const float *ds = dscore + (size_t)u * s.cap;
    const size_t lbase = ((size_t)b * s.Hkv + g) * s.nb;
    float dqb[EPT];
#pragma unroll
    for (int c = 0; c < EPT; ++c) dqb[c] = 0.f;
    for (int e = 0; e < cnt; ++e) {
        const int blk = il[e];
        if (blk < 0 || blk > j) continue;
        const float w = s.scale * ds[e];
        if (w == 0.f) continue;
        const T *lrow = L + (lbase + blk) * D;
#pragma unroll
        for (int c = 0; c < EPT; ++c) {
            dqb[c] = fmaf(w, to_f(lrow[lane + 32 * c]), dqb[c]);
            atomicAdd(dL + (lbase + blk) * D + lane + 32 * c, w * qb[c]);
        }
    }
    for (int h = g * s.G; h < (g + 1) * s.G; ++h)
        for (int r = 0; r < nrows; ++r) {
            float *row = dQ + (((size_t)b * s.Hq + h) * s.N + r0 + r) * D;
#pragma unroll
            for (int c = 0; c < EPT; ++c) row[lane + 32 * c] += dqb[c] / (float)R;
        }
}

// Kernel D: dK[key] += dL[block of key] / (keys in that block).
__global__ void dl_to_dk_kernel(Shape s, const float *dL, float *dK, size_t total) {
    const size_t x = (size_t)blockIdx.x * blockDim.x + threadIdx.x;
    if (x >= total) return;
    const int e = (int)(x % s.d);
    const size_t row = x / s.d;                         // (b * Hkv + g) * N + t
    const int t = (int)(row % s.N);
    const size_t bg = row / s.N;
    const int blk = t / s.bs;
    const int n = min(s.bs, s.N - blk * s.bs);
    dK[x] += dL[(bg * s.nb + blk) * s.d + e] / (float)n;
}

template <typename T, int D>
cudaError_t run_attn_bwd(const BwArgs &a, cudaStream_t st) {
    const Shape &s = a.s;
    const size_t smem = sizeof(float) * ((size_t)2 * kRC * D + 2 * kKC * (D + 1) + 2 * kRC * (kKC + 1) + 2 * kRC) +
                        sizeof(int) * kRC + 16;
    cudaError_t e = cudaFuncSetAttribute(bwd_attn_kernel<T, D>, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    if (e != cudaSuccess) return e;
    const size_t units = (size_t)s.B * s.Hkv * s.nb;
    bwd_attn_kernel<T, D><<<(unsigned)(units * a.rchunks), kBwThreads, smem, st>>>(a);
    note_launch();
    return cudaGetLastError();
}

}  // namespace

bool backward_supported(const Shape &s) {
    if (s.flags & (SA_HIER | SA_SELECT_PER_QHEAD)) return false;
    return s.d == 64 || s.d == 128;
}

size_t select_backward_workspace(const Shape &s) { return (size_t)s.B * s.Hkv * s.nb * s.d * sizeof(float); }

size_t prefill_backward_workspace(const Shape &s) {
    const size_t simt = (size_t)s.B * s.Hkv * s.nb * s.cap * sizeof(float);
    // room for either path (SPARSE_ATTN_BACKWARD_PATH=simt selects the CUDA-core one)
    return backward_tc_shape_ok(s) ? std::max(simt, backward_tc_workspace(s)) : simt;
}

cudaError_t launch_prefill_backward(const Shape &s, const void *Q, const void *K, const void *V, const void *O,
                                    const float *lse, const void *dO, const int32_t *idx, const float *score,
                                    const int32_t *count, float *dQ, float *dK, float *dV, float *dscore,
                                    void *ws, cudaStream_t st) {
    if (backward_tc_supported(s))
        return launch_backward_tc(s, Q, K, V, O, lse, dO, idx, score, count, dQ, dK, dV, dscore, ws, st);
    const size_t kv_bytes = (size_t)s.B * s.Hkv * s.N * s.d * sizeof(float);
    float *dgate = reinterpret_cast<float *>(static_cast<unsigned char *>(ws) + ws_layout(s).scratch);
    const size_t units = (size_t)s.B * s.Hkv * s.nb;
    cudaError_t e;
    if ((e = cudaMemsetAsync(dK, 0, kv_bytes, st)) != cudaSuccess) return e;
    if ((e = cudaMemsetAsync(dV, 0, kv_bytes, st)) != cudaSuccess) return e;
    if ((e = cudaMemsetAsync(dgate, 0, prefill_backward_workspace(s), st)) != cudaSuccess) return e;
    BwArgs a{};
    a.s = s;
    a.Q = Q; a.K = K; a.V = V; a.O = O; a.dO = dO;
    a.lse = lse;
    a.idx = idx; a.score = score; a.count = count;
    a.dQ = dQ; a.dK = dK; a.dV = dV; a.dgate = dgate;
    a.status = static_cast<unsigned *>(ws);
    a.rchunks = (s.G * s.bs + kRC - 1) / kRC;
    if (s.dtype == SA_BF16) e = s.d == 128 ? run_attn_bwd<__nv_bfloat16, 128>(a, st) : run_attn_bwd<__nv_bfloat16, 64>(a, st);
    else e = s.d == 128 ? run_attn_bwd<float, 128>(a, st) : run_attn_bwd<float, 64>(a, st);
    if (e != cudaSuccess) return e;
    bwd_score_kernel<<<(unsigned)((units + 127) / 128), 128, 0, st>>>(s, idx, score, count, dgate, dscore, (int)units);
    note_launch();
    return cudaGetLastError();
}

cudaError_t launch_select_backward(const Shape &s, const void *Q, const void *L, const int32_t *idx,
                                   const float *dscore, const int32_t *count, float *dQ, float *dK, void *ws,
                                   cudaStream_t st) {
    float *dL = reinterpret_cast<float *>(static_cast<unsigned char *>(ws) + ws_layout(s).scratch);
    const size_t units = (size_t)s.B * s.Hkv * s.nb;
    cudaError_t e = cudaMemsetAsync(dL, 0, select_backward_workspace(s), st);
    if (e != cudaSuccess) return e;
    const unsigned grid = (unsigned)((units + 7) / 8);
    if (s.dtype == SA_BF16) {
        if (s.d == 128) sel_bwd_kernel<__nv_bfloat16, 128><<<grid, 256, 0, st>>>(s, Q, L, idx, dscore, count, dQ, dL, (int)units);
        else sel_bwd_kernel<__nv_bfloat16, 64><<<grid, 256, 0, st>>>(s, Q, L, idx, dscore, count, dQ, dL, (int)units);
    } else {
        if (s.d == 128) sel_bwd_kernel<float, 128><<<grid, 256, 0, st>>>(s, Q, L, idx, dscore, count, dQ, dL, (int)units);
        else sel_bwd_kernel<float, 64><<<grid, 256, 0, st>>>(s, Q, L, idx, dscore, count, dQ, dL, (int)units);
    }
    note_launch();
    if ((e = cudaGetLastError()) != cudaSuccess) return e;
    const size_t total = (size_t)s.B * s.Hkv * s.N * s.d;
    dl_to_dk_kernel<<<(unsigned)((total + 255) / 256), 256, 0, st>>>(s, dL, dK, total);
    note_launch();
    return cudaGetLastError();
}

}  // namespace sa
