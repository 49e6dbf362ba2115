// lsa.cuh -- internal interface of the flat clustered index (lsa.cu).
#pragma once

#include <cuda_runtime.h>
#include <stdint.h>

namespace sa {

// Shape of one flat-index call, resolved on the host.
struct LsaShape {
    int B, Hq, Hkv, G, d, N, pool, seg, clusters, top_clusters, sink, window, dtype;
    float scale;
    int nseg;        // complete segments: N / (pool * seg)
    int ctotal;      // clusters per (batch, kv-head): nseg * clusters
};

cudaError_t launch_lsa_build(const LsaShape &s, const void *K, double *centres, int32_t *members, int32_t *sizes,
                             cudaStream_t st);
cudaError_t launch_lsa_decode(const LsaShape &s, const void *q, const void *K, const void *V, const double *centres,
                              const int32_t *members, const int32_t *sizes, double *scores, unsigned *status, void *o,
                              float *lse, cudaStream_t st);

}  // namespace sa
