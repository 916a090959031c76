// noalloc.cu -- w4a4_linear_noalloc: the W4A4 layer GEMM for callers that
// cannot allocate device memory at call time.
//
// Some callers cannot provide device scratch when they call the layer:
// runtimes that plan every device buffer once at start-up and forbid
// allocation afterwards, or processes whose memory pool is already exhausted.
// Both GEMM kernels finish every output inside the CTA that owns it (the
// small-M kernel reduces its K-split partial sums in shared memory), so no
// call needs a workspace; this entry point takes the arguments of
// w4a4_linear minus the workspace and guarantees that it never asks for one.
#include <cstdint>
#include <cuda_runtime.h>

#include "../../include/hq.h"
#include "hq_gemm.cuh"

using namespace hq;

extern "C" hq_status w4a4_linear_noalloc(const uint8_t* Xq, const float* sx, int64_t M, int64_t K,
                                         const uint8_t* Wq, const uint16_t* sw, const uint16_t* zw, int64_t N,
                                         int32_t group, const uint8_t* A, const uint16_t* B,
                                         const int32_t* sal_idx, int32_t r, void* Y, hq_dtype yt, void* stream) {
    // every argument check first: a rejected call enqueues nothing
    const hq_status chk = check_linear(Xq, sx, M, K, Wq, sw, zw, N, group, A, B, sal_idx, r, Y, yt);
    if (chk != HQ_OK) return chk;
    if (M == 0 || N == 0) return HQ_OK;
    // a shape whose kernel would need scratch is not served here
    if (hq_linear_workspace_size(M, N, K, group) != 0) return HQ_ERR_UNSUPPORTED;
    return w4a4_linear(Xq, sx, M, K, Wq, sw, zw, N, group, A, B, sal_idx, r, Y, yt, nullptr, 0, stream);
}
