// landmarks.cu -- block landmarks: the mean of each KV block's keys.
//
// [HiLS] (opening section) names the per-chunk summary a landmark; the Latent
// Sparse Attention post (section "Индекс перестаёт перебирать весь контекст")
// pools adjacent keys before they are scored.  The mean over the keys that
// exist (t < N) is summed in fp32 and stored in the KV dtype (round to nearest
// even), so a decode-time scan reads half the bytes of an fp32 copy.
//
// HBM-bound stream of K: one warp per block, 16-byte coalesced loads, several
// rows in flight per lane; algorithmic bytes = |K| + |L|.
#include "common.cuh"

namespace sa {

template <typename T, int VPR>
__global__ void __launch_bounds__(256) landmarks_kernel(const T *__restrict__ K, T *__restrict__ L, int N, int bs,
                                                        int nb, long long nunits, Shape s) {
    constexpr int EPV = Vec<T>::n;           // elements per 16-byte vector
    constexpr int RSTEP = 32 / VPR;          // rows a warp covers per step
    const int lane = threadIdx.x & 31;
    const long long unit = (long long)blockIdx.x * 8 + (threadIdx.x >> 5);
    if (unit >= nunits) return;
    const long long bg = unit / nb;
    const int blk = (int)(unit - bg * nb);
    const int d = VPR * EPV;
    const int t0 = blk * bs;
    // per-sequence length and first block to refresh (appends), when given
    const int bb = (int)(bg / s.Hkv);
    const int n = seq_n(s, bb);
    const int fb = s.first_block ? max(0, s.first_block[bb]) : 0;
    if (blk < fb || t0 >= n) return;   // the whole warp leaves together
    const int cnt = min(bs, n - t0);
    const int cv = lane % VPR, rs = lane / VPR;
    const T *base = K + ((size_t)bg * N + t0) * d + cv * EPV;
    float acc[EPV];
#pragma unroll
    for (int i = 0; i < EPV; ++i) acc[i] = 0.f;
    int r = rs;
    for (; r + 3 * RSTEP < cnt; r += 4 * RSTEP) {
        float f0[EPV], f1[EPV], f2[EPV], f3[EPV];
        load16(base + (size_t)r * d, f0);
        load16(base + (size_t)(r + RSTEP) * d, f1);
        load16(base + (size_t)(r + 2 * RSTEP) * d, f2);
        load16(base + (size_t)(r + 3 * RSTEP) * d, f3);
#pragma unroll
        for (int i = 0; i < EPV; ++i) acc[i] += (f0[i] + f1[i]) + (f2[i] + f3[i]);
    }
    for (; r < cnt; r += RSTEP) {
        float f0[EPV];
        load16(base + (size_t)r * d, f0);
#pragma unroll
        for (int i = 0; i < EPV; ++i) acc[i] += f0[i];
    }
#pragma unroll
    for (int o = VPR; o < 32; o <<= 1)
#pragma unroll
        for (int i = 0; i < EPV; ++i) acc[i] += __shfl_xor_sync(0xffffffffu, acc[i], o);
    if (rs == 0) {
        const float c = (float)cnt;
#pragma unroll
        for (int i = 0; i < EPV; ++i) acc[i] = __fdiv_rn(acc[i], c);
        store16(L + ((size_t)bg * nb + blk) * d + cv * EPV, acc);
    }
}

template <typename T>
static cudaError_t run(const Shape &s, const void *K, void *L, cudaStream_t st) {
    const long long nunits = (long long)s.B * s.Hkv * s.nb;
    const unsigned grid = (unsigned)((nunits + 7) / 8);
    const int vpr = s.d * (int)sizeof(T) / 16;
    auto k = (const T *)K;
    auto l = (T *)L;
    switch (vpr) {
        case 8: landmarks_kernel<T, 8><<<grid, 256, 0, st>>>(k, l, s.N, s.bs, s.nb, nunits, s); break;
        case 16: landmarks_kernel<T, 16><<<grid, 256, 0, st>>>(k, l, s.N, s.bs, s.nb, nunits, s); break;
        case 32: landmarks_kernel<T, 32><<<grid, 256, 0, st>>>(k, l, s.N, s.bs, s.nb, nunits, s); break;
        default: return cudaErrorInvalidValue;
    }
    note_launch();
    return cudaGetLastError();
}

cudaError_t launch_landmarks(const Shape &s, const void *K, void *L, cudaStream_t st) {
    return s.dtype == SA_BF16 ? run<__nv_bfloat16>(s, K, L, st) : run<float>(s, K, L, st);
}

}  // namespace sa
