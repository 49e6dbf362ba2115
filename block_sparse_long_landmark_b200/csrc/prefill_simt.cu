// prefill_simt.cu -- CUDA-core block-sparse prefill (fp32 and bf16, any
// supported shape).  The tensor-core kernel covers the bf16 d=128 workloads;
// this one serves fp32 (where TF32 tensor cores would break the 1e-4 bound)
// and shapes outside the tensor-core kernel's tiling.
//
// [SAS] "Ключевые факты" / "Как это применить": attention is computed
// blockwise, FlashAttention-style, without the square matrix; the gate is a
// log-domain term inside the softmax, normalised against the always-kept
// current block: gate_b = log_sigmoid(s_b - s_local) for selected blocks, 0
// for the forced sink and local blocks.  [HiLS] opening section: in
// hierarchical mode every kept block gets its own softmax and the block
// outputs are combined with weights softmax_b(s_b).
//
// CTA = 64 query rows of one q-head in one tile; TPR = d/32 threads per row,
// each holding 32 dims of q and of the accumulator.  Keys are streamed block
// by block through shared memory, 8 at a time: 8 partial dot products, a
// shuffle reduction across the row's threads, one online-softmax update.
#include <math_constants.h>

#include "bounds.cuh"
#include "common.cuh"

namespace sa {

constexpr int kRows = 64;
constexpr int kKeyChunk = 8;

struct PrefArgs {
    Shape s;
    const void *Q, *K, *V;
    const int32_t *idx;
    const float *score;
    const int32_t *count;
    void *O;
    float *lse;
    unsigned *status;
    int rchunks;   // 64-row chunks per tile
};

template <typename T, int TPR>
__global__ void __launch_bounds__(kRows *TPR) prefill_simt_kernel(PrefArgs a) {
    constexpr int D = TPR * 32;
    constexpr float kLog2e = 1.4426950408889634f;
    constexpr float kLn2 = 0.6931471805599453f;
    const Shape &s = a.s;
    extern __shared__ __align__(16) unsigned char smem_raw[];
    T *Ks = reinterpret_cast<T *>(smem_raw);
    T *Vs = Ks + (size_t)s.bs * D;

    // grid: ((b * Hq + h) * ntiles + j) * rchunks + rc
    int u = blockIdx.x;
    const int rc = u % a.rchunks;
    u /= a.rchunks;
    const int j = u % s.nb;
    u /= s.nb;
    const int h = u % s.Hq;
    const int b = u / s.Hq;
    const int g = h / s.G;
    const int hs = (s.flags & SA_SELECT_PER_QHEAD) ? h : g;
    const size_t lu = ((size_t)b * s.Hsel + hs) * s.nb + j;
    const int32_t *idx = a.idx + lu * s.cap;
    const float *sc = a.score + lu * s.cap;
    const int cnt = min(a.count[lu], s.cap);

    const int row = threadIdx.x / TPR, part = threadIdx.x % TPR;
    const int i = j * s.bs + rc * kRows + row;          // query position
    const bool row_ok = (rc * kRows + row) < s.bs && i < s.N;
    const int ic = row_ok ? i : min(s.N - 1, j * s.bs);

    const T *Qrow = (const T *)a.Q + (((size_t)b * s.Hq + h) * s.N + ic) * D + part * 32;
    float q[32];
#pragma unroll
    for (int v = 0; v < 32; v += Vec<T>::n) load16(Qrow + v, q + v);
    const float qscale = s.scale * kLog2e;   // logits in log2 units
#pragma unroll
    for (int v = 0; v < 32; ++v) q[v] *= qscale;

    const bool hier = s.flags & SA_HIER;
    const bool gate_on = s.flags & SA_GATE;
    const float s_local = cnt > 0 ? sc[cnt - 1] : 0.f;

    float acc[32], accb[32];
#pragma unroll
    for (int v = 0; v < 32; ++v) acc[v] = accb[v] = 0.f;
    float m = -CUDART_INF_F, l = 0.f;       // gated: running max / sum (log2 units)
    float M = -CUDART_INF_F, W = 0.f;       // hier: running max / sum of retrieval weights

    const T *Kg = (const T *)a.K + ((size_t)b * s.Hkv + g) * (size_t)s.N * D;
    const T *Vg = (const T *)a.V + ((size_t)b * s.Hkv + g) * (size_t)s.N * D;
    int prev = -1;
    for (int c = 0; c < cnt; ++c) {
        const int blk = idx[c];
        if (blk < 0 || blk > j || blk <= prev) {   // malformed list entry: skip it
            if (threadIdx.x == 0) set_status(a.status, kStatusBadIndex);
            continue;
        }
        prev = blk;
        const bool forced = (blk == j && (s.flags & SA_LOCAL)) || (blk == 0 && (s.flags & SA_SINK));
        const float gate = (gate_on && !forced) ? log_sigmoid(sc[c] - s_local) * kLog2e : 0.f;
        const int t0 = blk * s.bs, nk = min(s.bs, s.N - t0);
        SA_CHECK_START(a.status, t0, s.N);
        __syncthreads();
        {
            const int nvec = nk * D / Vec<T>::n;
            const T *ks = Kg + (size_t)t0 * D, *vs = Vg + (size_t)t0 * D;
            for (int e = threadIdx.x; e < nvec; e += blockDim.x) {
                reinterpret_cast<uint4 *>(Ks)[e] = reinterpret_cast<const uint4 *>(ks)[e];
                reinterpret_cast<uint4 *>(Vs)[e] = reinterpret_cast<const uint4 *>(vs)[e];
            }
        }
        __syncthreads();
        const int kend = (blk == j && (s.flags & SA_CAUSAL)) ? min(nk, i - t0 + 1) : nk;
        float mb = -CUDART_INF_F, lb = 0.f;   // hier: this block's softmax state
        if (hier) {
#pragma unroll
            for (int v = 0; v < 32; ++v) accb[v] = 0.f;
        }
        for (int k0 = 0; k0 < nk; k0 += kKeyChunk) {
            float z[kKeyChunk];
#pragma unroll
            for (int kk = 0; kk < kKeyChunk; ++kk) {
                const int t = min(k0 + kk, nk - 1);
                const T *kr = Ks + (size_t)t * D + part * 32;
                float dot = 0.f;
#pragma unroll
                for (int v = 0; v < 32; v += Vec<T>::n) {
                    float f[Vec<T>::n];
                    load16(kr + v, f);
#pragma unroll
                    for (int w = 0; w < Vec<T>::n; ++w) dot = fmaf(q[v + w], f[w], dot);
                }
#pragma unroll
                for (int o = 1; o < TPR; o <<= 1) dot += __shfl_xor_sync(0xffffffffu, dot, o);
                z[kk] = (k0 + kk < kend) ? dot + (hier ? 0.f : gate) : -CUDART_INF_F;
            }
            float cm = z[0];
#pragma unroll
            for (int kk = 1; kk < kKeyChunk; ++kk) cm = fmaxf(cm, z[kk]);
            float &rm = hier ? mb : m;
            float &rl = hier ? lb : l;
            float *ra = hier ? accb : acc;
            const float nm = fmaxf(rm, cm);
            if (nm == -CUDART_INF_F) continue;   // nothing visible yet
            const float corr = exp2f(rm - nm);
            rl *= corr;
#pragma unroll
            for (int v = 0; v < 32; ++v) ra[v] *= corr;
            rm = nm;
#pragma unroll
            for (int kk = 0; kk < kKeyChunk; ++kk) {
                const float p = exp2f(z[kk] - nm);
                rl += p;
                const T *vr = Vs + (size_t)min(k0 + kk, nk - 1) * D + part * 32;
#pragma unroll
                for (int v = 0; v < 32; v += Vec<T>::n) {
                    float f[Vec<T>::n];
                    load16(vr + v, f);
#pragma unroll
                    for (int w = 0; w < Vec<T>::n; ++w) ra[v + w] = fmaf(p, f[w], ra[v + w]);
                }
            }
        }
        if (hier && lb > 0.f) {
            // fold o_b = accb / lb into the retrieval-weighted sum
            const float sb = sc[c] * kLog2e;
            const float nM = fmaxf(M, sb);
            const float corr = exp2f(M - nM), wb = exp2f(sb - nM);
            W = W * corr + wb;
            const float f = wb / lb;
#pragma unroll
            for (int v = 0; v < 32; ++v) acc[v] = acc[v] * corr + f * accb[v];
            M = nM;
        }
    }
    if (!row_ok) return;
    const float den = hier ? W : l;
    const float inv = den > 0.f ? 1.f / den : 0.f;
    T *Orow = (T *)a.O + (((size_t)b * s.Hq + h) * s.N + i) * D + part * 32;
#pragma unroll
    for (int v = 0; v < 32; v += Vec<T>::n) {
        float f[Vec<T>::n];
#pragma unroll
        for (int w = 0; w < Vec<T>::n; ++w) f[w] = acc[v + w] * inv;
        store16(Orow + v, f);
    }
    if (part == 0) {
        const float mm = hier ? M : m;
        a.lse[((size_t)b * s.Hq + h) * s.N + i] = den > 0.f ? (mm + log2f(den)) * kLn2 : -CUDART_INF_F;
    }
}

template <typename T>
static cudaError_t run(const Shape &s, const PrefArgs &a0, cudaStream_t st) {
    PrefArgs a = a0;
    a.rchunks = (s.bs + kRows - 1) / kRows;
    const size_t smem = (size_t)2 * s.bs * s.d * sizeof(T);
    const unsigned grid = (unsigned)((size_t)s.B * s.Hq * s.nb * a.rchunks);
    void (*kern)(PrefArgs) = nullptr;
    int threads = 0;
    if (s.d == 64) { kern = prefill_simt_kernel<T, 2>; threads = kRows * 2; }
    else if (s.d == 128) { kern = prefill_simt_kernel<T, 4>; threads = kRows * 4; }
    else return cudaErrorInvalidValue;
    cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    if (e != cudaSuccess) return e;
    kern<<<grid, threads, smem, st>>>(a);
    note_launch();
    return cudaGetLastError();
}

cudaError_t launch_prefill_simt(const Shape &s, const void *Q, const void *K, const void *V, const int32_t *idx,
                                const float *score, const int32_t *count, void *O, float *lse, unsigned *status,
                                cudaStream_t st) {
    PrefArgs a{};
    a.s = s;
    a.Q = Q;
    a.K = K;
    a.V = V;
    a.idx = idx;
    a.score = score;
    a.count = count;
    a.O = O;
    a.lse = lse;
    a.status = status;
    return s.dtype == SA_BF16 ? run<__nv_bfloat16>(s, a, st) : run<float>(s, a, st);
}

}  // namespace sa
