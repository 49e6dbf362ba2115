// backward_tc.cuh -- internal interface of the tensor-core backward
// (backward_tc.cu: row preparation, dQ and the gate gradients;
// backward_kv.cu: dK and dV by key tiles).
#pragma once

#include <cuda_runtime.h>
#include <stddef.h>
#include <stdint.h>

#include "common.cuh"

namespace sa {

// bf16, d = 128, block 64 or 128, 128-row query tiles, per-kv-head gated or plain lists
bool backward_tc_shape_ok(const Shape &s);
// the shape is supported and SPARSE_ATTN_BACKWARD_PATH does not ask for the CUDA-core path
bool backward_tc_supported(const Shape &s);
size_t backward_tc_workspace(const Shape &s);
cudaError_t launch_backward_tc(const Shape &s, const void *Q, const void *K, const void *V, const void *O,
                               const float *lse, const void *dO, const int32_t *idx, const float *score,
                               const int32_t *count, float *dQ, float *dK, float *dV, float *dscore, void *ws,
                               cudaStream_t st);

// dK, dV of every key tile from the rows that keep it.  `D` and `lse2` are
// the per-row values of bwd_rowprep_kernel; `work` is this step's part of
// the scratch area (backward_kv_workspace bytes); `rcnt` its completion
// counters ([tiles][8], zero between calls).
size_t backward_kv_workspace(const Shape &s);
cudaError_t launch_backward_kv(const Shape &s, const void *Q, const void *K, const void *V, const void *dO,
                               const float *D, const float *lse2, const int32_t *idx, const float *score,
                               const int32_t *count, float *dK, float *dV, void *work, int *rcnt,
                               unsigned *status, cudaStream_t st);

}  // namespace sa
