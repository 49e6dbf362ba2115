// bounds.cuh -- address checks of the debug build.  Built with
// -DSA_DEBUG_BOUNDS (python -m block_sparse_long_landmark_b200.build
// --debug-bounds, into lib/libsparse_attn_bounds.so), every gather checks that
// the first row it reads lies inside the slab of its tensor that the
// operation means to read (a kv-head's N keys, a query head's nb * block rows,
// a unit's landmarks; for the second 64-row half of a 128-key block, the
// sequence padded to whole blocks, whose rows past N are read and masked); a
// row outside sets status bit 8 (the copy still runs:
// the rows are clamped or masked downstream, so nothing faults).  The release
// build compiles every check to nothing.
#pragma once

#include "common.cuh"

namespace sa {

constexpr unsigned kStatusBounds = 8u;

#ifdef SA_DEBUG_BOUNDS
__device__ __forceinline__ void check_start(unsigned *status, long long start, long long extent) {
    if (start < 0 || start >= extent) set_status(status, kStatusBounds);
}
__device__ __forceinline__ void check_span(unsigned *status, long long start, long long count, long long extent) {
    if (start < 0 || count < 0 || start + count > extent) set_status(status, kStatusBounds);
}
#define SA_CHECK_START(status, start, extent) ::sa::check_start((status), (long long)(start), (long long)(extent))
#define SA_CHECK_SPAN(status, start, count, extent) \
    ::sa::check_span((status), (long long)(start), (long long)(count), (long long)(extent))
#else
#define SA_CHECK_START(status, start, extent) ((void)0)
#define SA_CHECK_SPAN(status, start, count, extent) ((void)0)
#endif

}  // namespace sa
