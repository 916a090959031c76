// noalloc.cu -- w4a4_linear_noalloc: the W4A4 layer GEMM for callers that
// cannot allocate device memory at call time.
//
// w4a4_linear needs a caller-provided workspace when it takes the small-M
// (decode) kernel: per-tile arrival counters and partial sums for the split
// weight tiles.  Some callers cannot provide one: runtimes that plan every
// device buffer once at start-up and forbid allocation afterwards, or
// processes whose memory pool is already exhausted.  This entry point keeps
// that scratch in a fixed file-scope device array instead, so the call itself
// allocates nothing.
#include <cstdint>
#include <mutex>
#include <cuda_runtime.h>

#include "../../include/hq.h"
#include "hq_gemm.cuh"

namespace hq {
namespace {

// Maximum scratch of the small-M kernel this entry point serves: 8 MiB
// (a decode-shaped 11008 x 4096 layer with 16 tokens needs about 2 MiB).  Every
// GPU that loads the library holds this array until the process exits.
constexpr size_t kNoAllocScratchBytes = 8u << 20;

static __device__ __align__(256) uint8_t g_noalloc_scratch[kNoAllocScratchBytes];

constexpr int kMaxDevices = 64;
std::mutex g_scratch_mutex;
void* g_scratch_ptr[kMaxDevices] = {};

// Device address of the scratch array on the current device.  The array's
// name in host code is only a host-side stand-in, so the address is looked up
// once per device (with that device current) and cached.
hq_status scratch_for_current_device(void** out) {
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess) return HQ_ERR_CUDA;
    if (dev < 0 || dev >= kMaxDevices) return HQ_ERR_UNSUPPORTED;
    std::lock_guard<std::mutex> lock(g_scratch_mutex);
    if (g_scratch_ptr[dev] == nullptr) {
        void* p = nullptr;
        if (cudaGetSymbolAddress(&p, g_noalloc_scratch) != cudaSuccess || p == nullptr) return HQ_ERR_CUDA;
        g_scratch_ptr[dev] = p;
    }
    *out = g_scratch_ptr[dev];
    return HQ_OK;
}

}  // namespace
}  // namespace hq

using namespace hq;

extern "C" hq_status w4a4_linear_noalloc(const uint8_t* Xq, const float* sx, int64_t M, int64_t K,
                                         const uint8_t* Wq, const uint16_t* sw, const uint16_t* zw, int64_t N,
                                         int32_t group, const uint8_t* A, const uint16_t* B,
                                         const int32_t* sal_idx, int32_t r, void* Y, hq_dtype yt, void* stream) {
    // every argument check first: a rejected call enqueues nothing
    const hq_status chk = check_linear(Xq, sx, M, K, Wq, sw, zw, N, group, A, B, sal_idx, r, Y, yt);
    if (chk != HQ_OK) return chk;
    if (M == 0 || N == 0) return HQ_OK;
    const size_t need = small_supported(M, group) ? hq_linear_workspace_size(M, N, K, group) : 0;
    if (need > kNoAllocScratchBytes) return HQ_ERR_UNSUPPORTED;   // beyond the fixed scratch
    if (need == 0)   // the large-M kernel needs no scratch
        return w4a4_linear(Xq, sx, M, K, Wq, sw, zw, N, group, A, B, sal_idx, r, Y, yt, nullptr, 0, stream);
    void* ws = nullptr;
    const hq_status s = scratch_for_current_device(&ws);
    if (s != HQ_OK) return s;
    // the per-tile arrival counters at the start of the scratch must be zero;
    // the array keeps whatever the previous call (of any shape) left in it
    if (cudaMemsetAsync(ws, 0, small_counter_bytes_for_n(N), static_cast<cudaStream_t>(stream)) != cudaSuccess)
        return HQ_ERR_CUDA;
    return w4a4_linear(Xq, sx, M, K, Wq, sw, zw, N, group, A, B, sal_idx, r, Y, yt, ws, kNoAllocScratchBytes,
                       stream);
}
