// common.cuh -- shared device helpers and the internal launch interface of
// libsparse_attn.so.  sm_100a only.
#pragma once

#include <cuda_bf16.h>
#include <cuda_runtime.h>
#include <stdint.h>

#include "sparse_attn.h"

namespace sa {

// Launch that may start before the previous kernel on the stream has finished
// (programmatic dependent launch); the kernel waits for its inputs on the
// device (griddepcontrol.wait) before it reads what that kernel wrote.
template <typename... KArgs, typename... Args>
cudaError_t launch_pdl(void (*kern)(KArgs...), dim3 grid, dim3 block, size_t smem, cudaStream_t st, Args &&...args) {
    cudaLaunchConfig_t cfg{};
    cfg.gridDim = grid;
    cfg.blockDim = block;
    cfg.dynamicSmemBytes = smem;
    cfg.stream = st;
    cudaLaunchAttribute at[1];
    at[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    at[0].val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = at;
    cfg.numAttrs = 1;
    return cudaLaunchKernelEx(&cfg, kern, static_cast<Args &&>(args)...);
}

// Status word at the start of every workspace: bit 1 = index list entry out
// of range, bit 2 = NaN score, bit 4 = bounded wait expired.
constexpr unsigned kStatusBadIndex = 1u;
constexpr unsigned kStatusNaN = 2u;
constexpr unsigned kStatusTimeout = 4u;
constexpr size_t kStatusBytes = 256;   // keeps what follows 256-byte aligned

// Shape of one call, resolved on the host.
struct Shape {
    int B, Hq, Hkv, G, d, N, bs, nb, top_k, cap, flags, dtype;
    int Hsel;        // heads that own a selection list (Hkv, or Hq per q-head)
    int heads_per;   // query heads that share one list (G, or 1 per q-head)
    float scale;
    const int32_t *seq_len;      // decode / landmarks: per-sequence lengths [B] (device) or null = N
    const int32_t *first_block;  // landmarks: per-sequence first block to recompute [B] or null = 0
};

// Context length of sequence b: seq_len[b] clamped to [1, N], or N.
__device__ __forceinline__ int seq_n(const Shape &s, int b) {
    if (!s.seq_len) return s.N;
    const int n = s.seq_len[b];
    return n < 1 ? 1 : (n > s.N ? s.N : n);
}

__device__ __forceinline__ void set_status(unsigned *status, unsigned bit) {
    if (status) atomicOr(status, bit);
}

// fp32 -> uint32 key whose unsigned order is the float order (NaN -> 0).
__device__ __forceinline__ uint32_t ord_key(float f) {
    uint32_t u = __float_as_uint(f);
    if ((u & 0x7fffffffu) > 0x7f800000u) return 0u;
    return (u & 0x80000000u) ? ~u : (u | 0x80000000u);
}

__device__ __forceinline__ float key_to_float(uint32_t k) {
    uint32_t u = (k & 0x80000000u) ? (k & 0x7fffffffu) : ~k;
    return __uint_as_float(u);
}

__device__ __forceinline__ float log_sigmoid(float x) {
    return x >= 0.f ? -log1pf(expf(-x)) : x - log1pf(expf(x));
}

// 16-byte vector loads converted to fp32.
__device__ __forceinline__ void load16(const __nv_bfloat16 *p, float *f) {
    uint4 u = *reinterpret_cast<const uint4 *>(p);
    const __nv_bfloat162 *h = reinterpret_cast<const __nv_bfloat162 *>(&u);
#pragma unroll
    for (int i = 0; i < 4; ++i) {
        float2 t = __bfloat1622float2(h[i]);
        f[2 * i] = t.x;
        f[2 * i + 1] = t.y;
    }
}
__device__ __forceinline__ void load16(const float *p, float *f) {
    float4 u = *reinterpret_cast<const float4 *>(p);
    f[0] = u.x; f[1] = u.y; f[2] = u.z; f[3] = u.w;
}
__device__ __forceinline__ void store16(__nv_bfloat16 *p, const float *f) {
    uint4 u;
    __nv_bfloat162 *h = reinterpret_cast<__nv_bfloat162 *>(&u);
#pragma unroll
    for (int i = 0; i < 4; ++i) h[i] = __floats2bfloat162_rn(f[2 * i], f[2 * i + 1]);
    *reinterpret_cast<uint4 *>(p) = u;
}
__device__ __forceinline__ void store16(float *p, const float *f) {
    *reinterpret_cast<float4 *>(p) = make_float4(f[0], f[1], f[2], f[3]);
}
template <typename T> struct Vec { static constexpr int n = 16 / sizeof(T); };

__device__ __forceinline__ float to_f(float x) { return x; }
__device__ __forceinline__ float to_f(__nv_bfloat16 x) { return __bfloat162float(x); }
__device__ __forceinline__ void from_f(float &y, float x) { y = x; }
__device__ __forceinline__ void from_f(__nv_bfloat16 &y, float x) { y = __float2bfloat16_rn(x); }

// Packed two-wide fp32 arithmetic (sm_100): one instruction per pair.
__device__ __forceinline__ float2 ffma2(float2 a, float2 b, float2 c) {
    float2 d;
    asm("{\n\t.reg .b64 ra, rb, rc, rd;\n\t"
        "mov.b64 ra, {%2, %3};\n\tmov.b64 rb, {%4, %5};\n\tmov.b64 rc, {%6, %7};\n\t"
        "fma.rn.f32x2 rd, ra, rb, rc;\n\tmov.b64 {%0, %1}, rd;\n\t}"
        : "=f"(d.x), "=f"(d.y)
        : "f"(a.x), "f"(a.y), "f"(b.x), "f"(b.y), "f"(c.x), "f"(c.y));
    return d;
}
__device__ __forceinline__ float2 fadd2(float2 a, float2 b) {
    float2 d;
    asm("{\n\t.reg .b64 ra, rb, rd;\n\t"
        "mov.b64 ra, {%2, %3};\n\tmov.b64 rb, {%4, %5};\n\t"
        "add.rn.f32x2 rd, ra, rb;\n\tmov.b64 {%0, %1}, rd;\n\t}"
        : "=f"(d.x), "=f"(d.y)
        : "f"(a.x), "f"(a.y), "f"(b.x), "f"(b.y));
    return d;
}
// Inclusive scan over a CTA of 256 threads (8 warps); `tmp` holds 8 ints.
__device__ __forceinline__ int block_scan_incl(int v, int *tmp, int *total) {
    const int lane = threadIdx.x & 31, w = threadIdx.x >> 5;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
        int t = __shfl_up_sync(0xffffffffu, v, o);
        if (lane >= o) v += t;
    }
    if (lane == 31) tmp[w] = v;
    __syncthreads();
    int add = 0, tot = 0;
#pragma unroll
    for (int i = 0; i < 8; ++i) {
        int x = tmp[i];
        if (i < w) add += x;
        tot += x;
    }
    __syncthreads();
    if (total) *total = tot;
    return v + add;
}

// Workspace layout shared by every operation of a parameter set: the status
// word, then one completion-counter array per operation that keeps counters
// (each returned to zero by the call that uses it, and written by no other
// operation), then the scratch area that each operation reuses freely.
struct WsLayout {
    size_t sel_chunk;    // select.cu: [B * Hsel * nb] chunk CTAs finished per unit
    size_t sel_decode;   // select_decode.cu: [B * Hsel] CTAs finished per unit
    size_t sel_ready;    // select_decode.cu -> decode_mma.cu: [B * Hsel] epoch of the unit's latest list
    size_t dec;          // decode.cu: [B * Hsel] partial records written, [B * Hsel] merge CTAs done
    size_t bwd_kv;       // backward_kv.cu: [B * Hkv * key tiles * 8] splits finished per tile region
    size_t scratch;      // first byte of the scratch area
};
WsLayout ws_layout(const Shape &s);

// Decode with every scratch byte inside `scratch` (see decode_static.cu);
// *need receives the bytes this shape takes.
int decode_on_scratch(const sa_params *p, const void *q, const void *K, const void *V, const int32_t *idx,
                      const float *score, const int32_t *count, void *o, float *lse, void *scratch,
                      size_t scratch_bytes, size_t *need, cudaStream_t st);

// Process-wide count of kernels this library has launched (for reporting).
void note_launch();

// Streaming multiprocessors of the current device (0 on failure).
int sm_count();

// ---------------------------------------------------------------------------
// Internal launchers (return cudaError_t of the launch)
// ---------------------------------------------------------------------------
cudaError_t launch_landmarks(const Shape &s, const void *K, void *L, cudaStream_t st);
cudaError_t launch_select(const Shape &s, bool decode, const void *Q, const void *L, int32_t *idx, float *score,
                          int32_t *count, void *ws, size_t ws_bytes, cudaStream_t st);
size_t select_workspace(const Shape &s, bool decode);
bool select_tiles_supported(const Shape &s);
bool select_decode_supported(const Shape &s);
size_t select_decode_workspace(const Shape &s);
// With `ready` (the decode step's overlap), each unit's final list is
// published by storing `epoch` into ready[unit] once it is written.
cudaError_t launch_select_decode(const Shape &s, const void *q, const void *L, int32_t *idx, float *score,
                                 int32_t *count, void *ws, cudaStream_t st, unsigned *ready = nullptr,
                                 unsigned epoch = 0);
// SPARSE_ATTN_SELECT_PATH=chunked: decode selection by the CTA-per-chunk
// kernel of select.cu (a cross-check hook; both give the same lists)
bool select_force_chunked();
cudaError_t launch_select_tiles(const Shape &s, const void *Q, const void *L, int32_t *idx, float *score,
                                int32_t *count, unsigned *status, cudaStream_t st);
cudaError_t launch_prefill_simt(const Shape &s, const void *Q, const void *K, const void *V, const int32_t *idx,
                                const float *score, const int32_t *count, void *O, float *lse, unsigned *status,
                                cudaStream_t st);
bool prefill_tc_supported(const Shape &s);
cudaError_t launch_prefill_tc(const Shape &s, const void *Q, const void *K, const void *V, const int32_t *idx,
                              const float *score, const int32_t *count, void *O, float *lse, unsigned *status,
                              cudaStream_t st);
bool prefill_tc2_supported(const Shape &s);
cudaError_t launch_prefill_tc2(const Shape &s, const void *Q, const void *K, const void *V, const int32_t *idx,
                               const float *score, const int32_t *count, void *O, float *lse, unsigned *status,
                               cudaStream_t st);
bool decode_mma_supported(const Shape &s);
void decode_mma_geometry(const Shape &s, int &S, int &bps);
size_t decode_mma_partial_bytes(const Shape &s, int S);
int decode_mma_records(int S);
// Decode scratch passed explicitly: the status word, two completion counters
// per unit (zero on entry, zero again on exit) and the partial records
// (R_out per unit, combined by the caller's merge launch).
// With `ready` the launch does not wait for the previous launch as a whole:
// each item waits (bounded) until ready[unit] holds `epoch`.
cudaError_t launch_decode_mma(const Shape &s, const void *q, const void *K, const void *V, const int32_t *idx,
                              const float *score, const int32_t *count, unsigned *status, unsigned *ucnt,
                              float *part, cudaStream_t st, int &R_out, const unsigned *ready = nullptr,
                              unsigned epoch = 0);
cudaError_t launch_decode(const Shape &s, const void *q, const void *K, const void *V, const int32_t *idx,
                          const float *score, const int32_t *count, void *o, float *lse, unsigned *status,
                          unsigned *ucnt, float *part, cudaStream_t st, const unsigned *ready = nullptr,
                          unsigned epoch = 0);
size_t decode_workspace(const Shape &s);
bool backward_supported(const Shape &s);
size_t prefill_backward_workspace(const Shape &s);
size_t select_backward_workspace(const Shape &s);
cudaError_t launch_prefill_backward(const Shape &s, const void *Q, const void *K, const void *V, const void *O,
                                    const float *lse, const void *dO, const int32_t *idx, const float *score,
                                    const int32_t *count, float *dQ, float *dK, float *dV, float *dscore,
                                    void *ws, cudaStream_t st);
cudaError_t launch_select_backward(const Shape &s, const void *Q, const void *L, const int32_t *idx,
                                   const float *dscore, const int32_t *count, float *dQ, float *dK, void *ws,
                                   cudaStream_t st);

}  // namespace sa
