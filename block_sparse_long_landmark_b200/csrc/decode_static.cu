// decode_static.cu -- sparse_attn_decode_static: the decode entry point for
// callers that cannot allocate device memory.
//
// Who needs it: code that runs where cudaMalloc is off limits -- inside a
// custom allocator's own callbacks, in an inference server whose memory pool
// owns every device byte and forbids side allocations, or in plugins whose
// host framework hands them only the tensors of one call.  Such callers still
// pass the query, the cache, the kept lists and the outputs, but cannot give
// sparse_attn_decode its workspace.  This entry point uses instead a scratch
// array that lives inside the library itself:
//
//   * kStaticScratchBytes (2 MiB) of file-scope __device__ memory, present on
//     every GPU that loads the library until the process exits;
//   * its device address is looked up once per device with
//     cudaGetSymbolAddress, on the first call made while that device is
//     current -- make that first call before any stream capture;
//   * every call on a device shares the one array, so calls that overlap on
//     the GPU (different streams, or other host threads) race on it; order
//     them on one stream or serialise them;
//   * each call lays out, from the array's start, the status word and the
//     split partials, and clears the status word (cudaMemsetAsync on the
//     call's stream); the partials need no clearing because every split
//     writes its own slot before the merge reads it;
//   * problems whose split partials do not fit return SA_ERR_WORKSPACE before
//     anything is launched;
//   * nothing here calls cudaMalloc, cudaFree or an allocating library.
//
// The kernels are the ones sparse_attn_decode launches; only the scratch
// pointer differs.  Device-side list problems are skipped as there, but the
// status word that records them is internal to this entry point.
#include <mutex>

#include "common.cuh"

namespace {

constexpr size_t kStaticScratchBytes = size_t(2) << 20;
constexpr int kMaxDevices = 64;

static __device__ __align__(256) unsigned char g_decode_scratch[kStaticScratchBytes];

std::mutex g_mu;
void *g_addr[kMaxDevices] = {};

// Device address of the scratch array on the current device (set-up on the
// first call per device).  Returns nullptr on failure.
void *scratch_address() {
    int dev = -1;
    if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) return nullptr;
    std::lock_guard<std::mutex> lock(g_mu);
    if (!g_addr[dev]) {
        void *ptr = nullptr;
        if (cudaGetSymbolAddress(&ptr, g_decode_scratch) != cudaSuccess) return nullptr;
        g_addr[dev] = ptr;
    }
    return g_addr[dev];
}

}  // namespace

extern "C" int sparse_attn_decode_static(const sa_params *p, const void *q, const void *K, const void *V,
                                         const int32_t *idx, const float *score, const int32_t *count, void *o,
                                         float *lse, void *stream) {
    // size and argument checks first: too large a problem returns before any set-up or launch
    size_t need = 0;
    const int r = sa::decode_on_scratch(p, q, K, V, idx, score, count, o, lse, nullptr, 0, &need, nullptr);
    if (r != SA_ERR_WORKSPACE) return r;              // invalid parameters
    if (need > kStaticScratchBytes) return SA_ERR_WORKSPACE;
    if (!q || !K || !V || !idx || !score || !count || !o || !lse) return SA_ERR_ARG;
    void *ws = scratch_address();
    if (!ws) return SA_ERR_LAUNCH;
    return sa::decode_on_scratch(p, q, K, V, idx, score, count, o, lse, ws, kStaticScratchBytes, nullptr,
                                 (cudaStream_t)stream);
}
